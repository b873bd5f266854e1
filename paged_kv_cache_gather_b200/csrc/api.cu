// C ABI entry points: argument checks on the host, then one or two kernel
// launches on the caller's stream. Nothing here allocates device memory or
// synchronises.
#include <cudaTypedefs.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "pkv_common.cuh"
#include "pkv_internal.h"

namespace pkv {

static thread_local char g_last_error[512] = "";

int fail(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return status;
}

void clear_last_error() { g_last_error[0] = 0; }

int device_sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

int check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(PKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return PKV_OK;
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_pool_tensor_map(void* map_out, const void* base, int64_t rows, int32_t head_dim,
                          int32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)head_dim * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(reinterpret_cast<CUtensorMap*>(map_out), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_pool_tensor_map_u8(void* map_out, const void* base, int64_t rows, int32_t head_dim,
                             int32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)head_dim};
  cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(reinterpret_cast<CUtensorMap*>(map_out), CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                  const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tensor_map_bf16(void* map_out, const void* base, int rank, const uint64_t* dims,
                          const uint64_t* strides_bytes, const uint32_t* box) {
  auto fn = encode_fn();
  if (!fn || rank < 1 || rank > 5) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) st[i] = strides_bytes[i];
  }
  CUresult r = fn(reinterpret_cast<CUtensorMap*>(map_out), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank,
                  const_cast<void*>(base), d, st, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int check_cache(const pkv_cache_desc& c, const char* fn) {
  if (c.num_blocks <= 0 || c.num_kv_heads <= 0 || c.head_dim <= 0 || c.block_size <= 0)
    return fail(PKV_ERR_INVALID_ARG, "%s: cache sizes must be positive", fn);
  if (c.block_size & (c.block_size - 1))
    return fail(PKV_ERR_INVALID_ARG, "%s: block_size %d is not a power of two", fn,
                c.block_size);
  if (c.dtype != PKV_F32 && c.dtype != PKV_BF16 && c.dtype != PKV_FP8_E4M3)
    return fail(PKV_ERR_UNSUPPORTED, "%s: dtype %d not supported", fn, c.dtype);
  if ((c.head_dim * dtype_size(c.dtype)) % 16 != 0)
    return fail(PKV_ERR_UNSUPPORTED, "%s: head_dim*elem_size must be a multiple of 16 bytes",
                fn);
  const int64_t rows = (int64_t)c.num_blocks * c.num_kv_heads * c.block_size;
  if (rows >= (int64_t(1) << 31))
    return fail(PKV_ERR_UNSUPPORTED, "%s: pool of %lld rows exceeds 2^31", fn, (long long)rows);
  return PKV_OK;
}

int check_mask(const pkv_mask_mod& m, const char* fn) {
  if (m.kind < PKV_MASK_NONE || m.kind > PKV_MASK_DOCUMENT)
    return fail(PKV_ERR_INVALID_ARG, "%s: unknown mask kind %d", fn, m.kind);
  if (m.kind == PKV_MASK_PREFIX_LM && !m.prefix_len)
    return fail(PKV_ERR_INVALID_ARG, "%s: prefix-LM mask needs prefix_len", fn);
  if (m.kind == PKV_MASK_DOCUMENT && (!m.doc_offsets || !m.doc_starts))
    return fail(PKV_ERR_INVALID_ARG, "%s: document mask needs doc_offsets and doc_starts", fn);
  return PKV_OK;
}

}  // namespace pkv

using namespace pkv;

extern "C" {

int pkv_version(void) { return PKV_VERSION; }

const char* pkv_last_error(void) { return g_last_error; }

const char* pkv_status_string(int status) {
  switch (status) {
    case PKV_OK: return "PKV_OK";
    case PKV_ERR_INVALID_ARG: return "PKV_ERR_INVALID_ARG";
    case PKV_ERR_UNSUPPORTED: return "PKV_ERR_UNSUPPORTED";
    case PKV_ERR_CUDA: return "PKV_ERR_CUDA";
    case PKV_ERR_WORKSPACE_TOO_SMALL: return "PKV_ERR_WORKSPACE_TOO_SMALL";
    case PKV_ERR_BAD_INDEX: return "PKV_ERR_BAD_INDEX";
    default: return "PKV_ERR_UNKNOWN";
  }
}

int paged_kv_append(const void* k, const void* v, const int64_t* slot_mapping, int32_t num_tokens,
                    void* k_cache, void* v_cache, pkv_cache_desc cache, int32_t* dbg_err,
                    void* stream) {
  g_last_error[0] = 0;
  if (int st = check_cache(cache, "paged_kv_append")) return st;
  if (cache.dtype == PKV_FP8_E4M3)
    return fail(PKV_ERR_UNSUPPORTED, "paged_kv_append: E4M3 pools take paged_kv_append_fp8");
  if (num_tokens < 0) return fail(PKV_ERR_INVALID_ARG, "paged_kv_append: num_tokens < 0");
  if (num_tokens == 0) return PKV_OK;
  if (!k || !v || !slot_mapping || !k_cache || !v_cache)
    return fail(PKV_ERR_INVALID_ARG, "paged_kv_append: null pointer");
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PKV_ERR_INVALID_ARG, "paged_kv_append: tensors must be 16-byte aligned");
  return launch_append(k, v, slot_mapping, num_tokens, k_cache, v_cache, cache, dbg_err,
                       static_cast<cudaStream_t>(stream));
}

int paged_kv_gather(const void* k_cache, const void* v_cache, pkv_cache_desc cache,
                    const int32_t* block_tables, int32_t max_blocks_per_seq,
                    const int32_t* seq_lens, int32_t batch, int32_t out_max_len, void* k_out,
                    void* v_out, int32_t* dbg_err, void* stream) {
  g_last_error[0] = 0;
  if (int st = check_cache(cache, "paged_kv_gather")) return st;
  if (batch < 0 || out_max_len < 0 || max_blocks_per_seq <= 0)
    return fail(PKV_ERR_INVALID_ARG, "paged_kv_gather: bad batch/out_max_len/max_blocks");
  if (batch == 0 || out_max_len == 0) return PKV_OK;
  if (!k_cache || !v_cache || !block_tables || !seq_lens || !k_out || !v_out)
    return fail(PKV_ERR_INVALID_ARG, "paged_kv_gather: null pointer");
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_out) || !aligned16(v_out))
    return fail(PKV_ERR_INVALID_ARG, "paged_kv_gather: tensors must be 16-byte aligned");
  return launch_gather(k_cache, v_cache, cache, block_tables, max_blocks_per_seq, seq_lens, batch,
                       out_max_len, k_out, v_out, dbg_err, static_cast<cudaStream_t>(stream));
}

int paged_kv_copy_blocks(void* k_cache, void* v_cache, pkv_cache_desc cache,
                         const int32_t* block_pairs, int32_t num_pairs, int32_t* dbg_err,
                         void* stream) {
  g_last_error[0] = 0;
  if (int st = check_cache(cache, "paged_kv_copy_blocks")) return st;
  if (cache.dtype == PKV_FP8_E4M3)
    return fail(PKV_ERR_UNSUPPORTED, "paged_kv_copy_blocks: E4M3 pools (row scales) not supported");
  if (num_pairs < 0) return fail(PKV_ERR_INVALID_ARG, "paged_kv_copy_blocks: num_pairs < 0");
  if (num_pairs == 0) return PKV_OK;
  if (!k_cache || !v_cache || !block_pairs)
    return fail(PKV_ERR_INVALID_ARG, "paged_kv_copy_blocks: null pointer");
  if (!aligned16(k_cache) || !aligned16(v_cache))
    return fail(PKV_ERR_INVALID_ARG, "paged_kv_copy_blocks: pools must be 16-byte aligned");
  return launch_copy_blocks(k_cache, v_cache, cache, block_pairs, num_pairs, dbg_err,
                            static_cast<cudaStream_t>(stream));
}

int paged_kv_copy_blocks_fp8(void* k_cache, void* v_cache, float* k_scale, float* v_scale,
                             pkv_cache_desc cache, const int32_t* block_pairs, int32_t num_pairs,
                             int32_t* dbg_err, void* stream) {
  g_last_error[0] = 0;
  const char* fn = "paged_kv_copy_blocks_fp8";
  if (int st = check_cache(cache, fn)) return st;
  if (cache.dtype != PKV_FP8_E4M3)
    return fail(PKV_ERR_UNSUPPORTED, "%s: E4M3 pools only (others take paged_kv_copy_blocks)", fn);
  const int64_t scale_bytes = (int64_t)cache.num_kv_heads * cache.block_size * 4;
  if (scale_bytes % 16)
    return fail(PKV_ERR_UNSUPPORTED, "%s: num_kv_heads * block_size must be a multiple of 4", fn);
  if (num_pairs < 0) return fail(PKV_ERR_INVALID_ARG, "%s: num_pairs < 0", fn);
  if (num_pairs == 0) return PKV_OK;
  if (!k_cache || !v_cache || !k_scale || !v_scale || !block_pairs)
    return fail(PKV_ERR_INVALID_ARG, "%s: null pointer", fn);
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_scale) || !aligned16(v_scale))
    return fail(PKV_ERR_INVALID_ARG, "%s: pools and scales must be 16-byte aligned", fn);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (int st = launch_copy_blocks(k_cache, v_cache, cache, block_pairs, num_pairs, dbg_err, s))
    return st;
  return launch_copy_spans(k_scale, v_scale, scale_bytes, cache.num_blocks, block_pairs,
                           num_pairs, dbg_err, s);
}

size_t paged_attention_decode_workspace_size(int32_t batch, int32_t num_q_heads,
                                             pkv_cache_desc cache) {
  if (check_cache(cache, "paged_attention_decode_workspace_size") != PKV_OK) return 0;
  if (batch < 0 || num_q_heads <= 0 || num_q_heads % cache.num_kv_heads) return 0;
  return decode_workspace_size(batch, num_q_heads, cache);
}

static int decode_entry(const char* fn, const void* q, const void* k_cache, const void* v_cache,
                        const float* k_scale, const float* v_scale, const void* k_new,
                        const void* v_new, pkv_cache_desc cache,
                        const int32_t* block_tables, int32_t max_blocks_per_seq,
                        const int32_t* seq_lens, int32_t batch, int32_t num_q_heads, float scale,
                        pkv_mask_mod mask, void* out, float* lse, void* workspace,
                        size_t workspace_bytes, int32_t* dbg_err, void* stream) {
  g_last_error[0] = 0;
  if (int st = check_cache(cache, fn)) return st;
  if (int st = check_mask(mask, fn)) return st;
  const bool fp8 = cache.dtype == PKV_FP8_E4M3;
  if (fp8 != (k_scale != nullptr))
    return fail(fp8 ? PKV_ERR_INVALID_ARG : PKV_ERR_UNSUPPORTED,
                fp8 ? "%s: E4M3 pools need row scales" : "%s: %s", fn,
                "row scales belong to E4M3 pools (paged_attention_decode_fp8)");
  if (batch < 0 || max_blocks_per_seq <= 0)
    return fail(PKV_ERR_INVALID_ARG, "%s: bad batch or max_blocks_per_seq", fn);
  if (num_q_heads <= 0 || num_q_heads % cache.num_kv_heads)
    return fail(PKV_ERR_INVALID_ARG, "%s: num_q_heads %d not a multiple of num_kv_heads %d", fn,
                num_q_heads, cache.num_kv_heads);
  if (!(scale == scale)) return fail(PKV_ERR_INVALID_ARG, "%s: scale is NaN", fn);
  if (batch == 0) return PKV_OK;
  if (!q || !k_cache || !v_cache || !block_tables || !seq_lens || !out ||
      (fp8 && (!k_scale || !v_scale)))
    return fail(PKV_ERR_INVALID_ARG, "%s: null pointer", fn);
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      !aligned16(workspace) || (fp8 && (!aligned16(k_scale) || !aligned16(v_scale))) ||
      !aligned16(k_new) || !aligned16(v_new))
    return fail(PKV_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", fn);
  const size_t need = decode_workspace_size(batch, num_q_heads, cache);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need))
    return fail(PKV_ERR_WORKSPACE_TOO_SMALL, "%s: workspace needs %zu bytes, got %zu", fn, need,
                workspace_bytes);
  DecodeArgs a{q,         k_cache, v_cache,    cache, block_tables, max_blocks_per_seq,
               seq_lens,  batch,   num_q_heads, scale, mask,         out,
               lse,       workspace, workspace_bytes, dbg_err, static_cast<cudaStream_t>(stream)};
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.k_new = k_new;
  a.v_new = v_new;
  return launch_decode(a);
}

int paged_attention_decode(const void* q, const void* k_cache, const void* v_cache,
                           pkv_cache_desc cache, const int32_t* block_tables,
                           int32_t max_blocks_per_seq, const int32_t* seq_lens, int32_t batch,
                           int32_t num_q_heads, float scale, pkv_mask_mod mask, void* out,
                           float* lse, void* workspace, size_t workspace_bytes,
                           int32_t* dbg_err, void* stream) {
  return decode_entry("paged_attention_decode", q, k_cache, v_cache, nullptr, nullptr, nullptr,
                      nullptr, cache,
                      block_tables, max_blocks_per_seq, seq_lens, batch, num_q_heads, scale, mask,
                      out, lse, workspace, workspace_bytes, dbg_err, stream);
}

int paged_attention_decode_fp8(const void* q, const void* k_cache, const void* v_cache,
                               const float* k_scale, const float* v_scale, pkv_cache_desc cache,
                               const int32_t* block_tables, int32_t max_blocks_per_seq,
                               const int32_t* seq_lens, int32_t batch, int32_t num_q_heads,
                               float scale, pkv_mask_mod mask, void* out, float* lse,
                               void* workspace, size_t workspace_bytes, int32_t* dbg_err,
                               void* stream) {
  const char* fn = "paged_attention_decode_fp8";
  if (cache.dtype != PKV_FP8_E4M3) {
    g_last_error[0] = 0;
    return fail(PKV_ERR_INVALID_ARG, "%s: the pool must be E4M3", fn);
  }
  return decode_entry(fn, q, k_cache, v_cache, k_scale, v_scale, nullptr, nullptr, cache,
                      block_tables,
                      max_blocks_per_seq, seq_lens, batch, num_q_heads, scale, mask, out, lse,
                      workspace, workspace_bytes, dbg_err, stream);
}

int paged_attention_decode_append(const void* q, const void* k_new, const void* v_new,
                                  void* k_cache, void* v_cache, pkv_cache_desc cache,
                                  const int32_t* block_tables, int32_t max_blocks_per_seq,
                                  const int32_t* seq_lens, int32_t batch, int32_t num_q_heads,
                                  float scale, pkv_mask_mod mask, void* out, float* lse,
                                  void* workspace, size_t workspace_bytes, int32_t* dbg_err,
                                  void* stream) {
  const char* fn = "paged_attention_decode_append";
  g_last_error[0] = 0;
  if (int st = check_cache(cache, fn)) return st;
  if (cache.dtype != PKV_BF16)
    return fail(PKV_ERR_UNSUPPORTED, "%s: bf16 pools only", fn);
  if (batch > 0 && (!k_new || !v_new)) return fail(PKV_ERR_INVALID_ARG, "%s: null pointer", fn);
  return decode_entry(fn, q, k_cache, v_cache, nullptr, nullptr, k_new, v_new, cache,
                      block_tables, max_blocks_per_seq, seq_lens, batch, num_q_heads, scale, mask,
                      out, lse, workspace, workspace_bytes, dbg_err, stream);
}

int paged_kv_append_fp8(const void* k, const void* v, const int64_t* slot_mapping,
                        int32_t num_tokens, void* k_cache, void* v_cache, float* k_scale,
                        float* v_scale, pkv_cache_desc cache, int32_t* dbg_err, void* stream) {
  g_last_error[0] = 0;
  const char* fn = "paged_kv_append_fp8";
  if (int st = check_cache(cache, fn)) return st;
  if (cache.dtype != PKV_FP8_E4M3 || cache.head_dim != 128)
    return fail(PKV_ERR_UNSUPPORTED, "%s: E4M3 pools with head_dim 128 only", fn);
  if (num_tokens < 0) return fail(PKV_ERR_INVALID_ARG, "%s: num_tokens < 0", fn);
  if (num_tokens == 0) return PKV_OK;
  if (!k || !v || !slot_mapping || !k_cache || !v_cache || !k_scale || !v_scale)
    return fail(PKV_ERR_INVALID_ARG, "%s: null pointer", fn);
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PKV_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", fn);
  return launch_append_fp8(k, v, slot_mapping, num_tokens, k_cache, v_cache, k_scale, v_scale,
                           cache, dbg_err, static_cast<cudaStream_t>(stream));
}

int paged_attention_prefill(const void* q, const void* k_new, const void* v_new,
                            const void* k_cache, const void* v_cache, pkv_cache_desc cache,
                            const int32_t* block_tables, int32_t max_blocks_per_seq,
                            const int32_t* ctx_lens, const int32_t* q_lens, int32_t batch,
                            int32_t total_q, int32_t num_q_heads, float scale, pkv_mask_mod mask,
                            void* out, float* lse, int32_t* dbg_err, void* stream) {
  g_last_error[0] = 0;
  const char* fn = "paged_attention_prefill";
  if (int st = check_cache(cache, fn)) return st;
  if (int st = check_mask(mask, fn)) return st;
  if (batch < 0 || total_q < 0 || max_blocks_per_seq <= 0)
    return fail(PKV_ERR_INVALID_ARG, "%s: bad batch, total_q or max_blocks_per_seq", fn);
  if (num_q_heads <= 0 || num_q_heads % cache.num_kv_heads)
    return fail(PKV_ERR_INVALID_ARG, "%s: num_q_heads %d not a multiple of num_kv_heads %d", fn,
                num_q_heads, cache.num_kv_heads);
  if (!(scale == scale)) return fail(PKV_ERR_INVALID_ARG, "%s: scale is NaN", fn);
  if (batch == 0 || total_q == 0) return PKV_OK;
  if (!q || !k_new || !v_new || !k_cache || !v_cache || !block_tables || !ctx_lens || !q_lens ||
      !out)
    return fail(PKV_ERR_INVALID_ARG, "%s: null pointer", fn);
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) ||
      !aligned16(v_cache) || !aligned16(out))
    return fail(PKV_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", fn);
  PrefillArgs a{q,        k_new,  v_new, k_cache, v_cache, cache, block_tables, max_blocks_per_seq,
                ctx_lens, q_lens, batch, total_q, num_q_heads, scale, mask, out,
                lse,      dbg_err, static_cast<cudaStream_t>(stream)};
  return launch_prefill(a);
}

// One warp waits on an mbarrier that nothing arrives on, through the same
// bounded wait every kernel of the library uses (bursts of try_wait, a
// globaltimer check between bursts, 4 s limit); when the wait gives up it sets
// PKV_DBG_TIMEOUT and the kernel returns normally.
__global__ void __launch_bounds__(32) debug_wait_timeout_kernel(int32_t* dbg, uint64_t* elapsed_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncwarp();
  const uint64_t t0 = global_ns();
  const bool ok = mbar_wait(smem_u32(&bar), 0);
  const uint64_t t1 = global_ns();
  if (threadIdx.x == 0) {
    if (!ok) flag_error(dbg, PKV_DBG_TIMEOUT);
    if (elapsed_ns) *elapsed_ns = t1 - t0;
  }
}

int pkv_debug_wait_timeout(int32_t* dbg_err, uint64_t* elapsed_ns, void* stream) {
  g_last_error[0] = 0;
  if (!dbg_err) return fail(PKV_ERR_INVALID_ARG, "pkv_debug_wait_timeout: null debug word");
  debug_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(dbg_err, elapsed_ns);
  return check_launch("pkv_debug_wait_timeout");
}

}  // extern "C"
