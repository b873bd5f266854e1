// Slot-mapped KV append and block-table gather.
//
// Both are exact byte copies, HBM-bound: every thread moves one 16-byte
// vector of K and one of V (128-bit loads and stores, consecutive threads on
// consecutive vectors of a head row), grid-stride over a grid sized to a
// multiple of the SM count.
//
// Append follows "Ultimate Guide to PagedAttention", dynamic growth: the new
// token goes to slot = block * block_size + row and nothing else moves.
// Gather follows the block-table section of the same page: position p of
// sequence b lives in block table[b][p / bs], row p % bs.
#include <cuda_fp8.h>

#include "pkv_common.cuh"
#include "pkv_internal.h"

namespace pkv {

__global__ void __launch_bounds__(256) kv_append_kernel(
    const int4* __restrict__ k, const int4* __restrict__ v, const int64_t* __restrict__ slots,
    int64_t num_vec, int32_t vec_per_row, int32_t num_kv_heads, int32_t block_shift,
    int64_t pool_slots, int4* __restrict__ k_cache, int4* __restrict__ v_cache, int32_t* dbg) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t vec_per_tok = (int64_t)vec_per_row * num_kv_heads;
  const int32_t bs_mask = (1 << block_shift) - 1;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < num_vec; i += stride) {
    const int64_t t = i / vec_per_tok;
    const int64_t rem = i - t * vec_per_tok;
    const int64_t h = rem / vec_per_row;
    const int64_t c = rem - h * vec_per_row;
    const int64_t slot = __ldg(slots + t);
    if (slot < 0) continue;
    if (slot >= pool_slots) {
      flag_error(dbg, PKV_DBG_SLOT);
      continue;
    }
    const int64_t blk = slot >> block_shift;
    const int64_t row = slot & bs_mask;
    const int64_t dst = (((blk * num_kv_heads + h) << block_shift) + row) * vec_per_row + c;
    const int4 kv = __ldg(k + i);
    const int4 vv = __ldg(v + i);
    // streaming stores: the written rows leave L2 soon instead of lingering
    // dirty until a later kernel's traffic evicts them
    __stcs(k_cache + dst, kv);
    __stcs(v_cache + dst, vv);
  }
}

__global__ void __launch_bounds__(256) kv_gather_kernel(
    const int4* __restrict__ k_cache, const int4* __restrict__ v_cache,
    const int32_t* __restrict__ tables, int32_t max_blocks, const int32_t* __restrict__ lens,
    int64_t num_vec, int32_t vec_per_row, int32_t num_kv_heads, int32_t block_shift,
    int32_t num_blocks, int32_t out_max_len, int4* __restrict__ k_out, int4* __restrict__ v_out,
    int32_t* dbg) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int32_t bs_mask = (1 << block_shift) - 1;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < num_vec; i += stride) {
    // output index i = ((b * Hkv + h) * out_max_len + p) * vec_per_row + c
    int64_t r = i / vec_per_row;
    const int64_t c = i - r * vec_per_row;
    const int64_t p = r % out_max_len;
    r /= out_max_len;
    const int64_t h = r % num_kv_heads;
    const int64_t b = r / num_kv_heads;
    int4 kv = make_int4(0, 0, 0, 0), vv = kv;
    const int32_t L = __ldg(lens + b);
    if (p < L) {
      const int64_t j = p >> block_shift;
      if (j >= max_blocks) {
        flag_error(dbg, PKV_DBG_LENGTH);
      } else {
        const int32_t blk = __ldg(tables + b * max_blocks + j);
        if (blk < 0 || blk >= num_blocks) {
          flag_error(dbg, PKV_DBG_BLOCK_ID);
        } else {
          const int64_t src =
              ((((int64_t)blk * num_kv_heads + h) << block_shift) + (p & bs_mask)) * vec_per_row +
              c;
          kv = __ldg(k_cache + src);
          vv = __ldg(v_cache + src);
        }
      }
    }
    k_out[i] = kv;
    v_out[i] = vv;
  }
}

// Copy-on-write: block pairs (src, dst); every KV head's rows of block src
// are copied to block dst, K and V. One thread per 16-byte vector.
// With `skip_unset`, pairs (-1, -1) are holes in the list and copy nothing.
__global__ void __launch_bounds__(256) kv_copy_blocks_kernel(
    int4* __restrict__ k_cache, int4* __restrict__ v_cache, const int32_t* __restrict__ pairs,
    int64_t num_vec, int64_t vec_per_block, int32_t num_blocks, bool skip_unset, int32_t* dbg) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < num_vec; i += stride) {
    const int64_t pr = i / vec_per_block;
    const int64_t off = i - pr * vec_per_block;
    const int32_t src = __ldg(pairs + 2 * pr), dst = __ldg(pairs + 2 * pr + 1);
    if (skip_unset && src == -1 && dst == -1) continue;
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
      if (off == 0) flag_error(dbg, PKV_DBG_BLOCK_ID);
      continue;
    }
    k_cache[(int64_t)dst * vec_per_block + off] = k_cache[(int64_t)src * vec_per_block + off];
    v_cache[(int64_t)dst * vec_per_block + off] = v_cache[(int64_t)src * vec_per_block + off];
  }
}

// E4M3 append: one warp per (token, KV head) row of K and of V; each lane
// holds 4 of the 128 values. The row's scale is amax / 448 (IEEE float32
// division; 1 for an all-zero row), each value is divided by it (IEEE) and
// rounded to the nearest E4M3 code, ties to even, saturating at +-448.
__device__ __forceinline__ uint32_t quantize4_e4m3(const uint2 w, float s) {
  const float x0 = __uint_as_float(w.x << 16), x1 = __uint_as_float(w.x & 0xffff0000u);
  const float x2 = __uint_as_float(w.y << 16), x3 = __uint_as_float(w.y & 0xffff0000u);
  const __nv_fp8x2_storage_t lo =
      __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(x0, s), __fdiv_rn(x1, s)), __NV_SATFINITE,
                               __NV_E4M3);
  const __nv_fp8x2_storage_t hi =
      __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(x2, s), __fdiv_rn(x3, s)), __NV_SATFINITE,
                               __NV_E4M3);
  return (uint32_t)lo | ((uint32_t)hi << 16);
}

__device__ __forceinline__ float row_amax(const uint2 w) {
  float a = fmaxf(fmaxf(fabsf(__uint_as_float(w.x << 16)), fabsf(__uint_as_float(w.x & 0xffff0000u))),
                  fmaxf(fabsf(__uint_as_float(w.y << 16)), fabsf(__uint_as_float(w.y & 0xffff0000u))));
#pragma unroll
  for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  return a;
}

__global__ void __launch_bounds__(256) kv_append_fp8_kernel(
    const uint2* __restrict__ k, const uint2* __restrict__ v, const int64_t* __restrict__ slots,
    int64_t rows, int32_t num_kv_heads, int32_t block_shift, int64_t pool_slots,
    uint32_t* __restrict__ k_cache, uint32_t* __restrict__ v_cache, float* __restrict__ k_scale,
    float* __restrict__ v_scale, int32_t* dbg) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int32_t bs_mask = (1 << block_shift) - 1;
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += warps) {
    const int64_t t = r / num_kv_heads;
    const int64_t h = r - t * num_kv_heads;
    const int64_t slot = __ldg(slots + t);
    if (slot < 0) continue;
    if (slot >= pool_slots) {
      if (lane == 0) flag_error(dbg, PKV_DBG_SLOT);
      continue;
    }
    const int64_t dst = (((slot >> block_shift) * num_kv_heads + h) << block_shift) + (slot & bs_mask);
    // 128 bf16 values = 32 uint2 per row; 128 codes = 32 uint32 per row
    const uint2 wk = __ldg(k + r * 32 + lane);
    const uint2 wv = __ldg(v + r * 32 + lane);
    const float ak = row_amax(wk), av = row_amax(wv);
    const float sk = ak > 0.f ? __fdiv_rn(ak, 448.f) : 1.f;
    const float sv = av > 0.f ? __fdiv_rn(av, 448.f) : 1.f;
    __stcs(k_cache + dst * 32 + lane, quantize4_e4m3(wk, sk));
    __stcs(v_cache + dst * 32 + lane, quantize4_e4m3(wv, sv));
    if (lane == 0) {
      k_scale[dst] = sk;
      v_scale[dst] = sv;
    }
  }
}

static int grid_for(int64_t work, int threads) {
  const int sms = device_sm_count();
  int64_t blocks = (work + threads - 1) / threads;
  const int64_t cap = (int64_t)sms * 8;  // 8 resident 256-thread CTAs per SM
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return (int)blocks;
}

int launch_append(const void* k, const void* v, const int64_t* slots, int32_t num_tokens,
                  void* k_cache, void* v_cache, const pkv_cache_desc& c, int32_t* dbg,
                  cudaStream_t s) {
  const int es = dtype_size(c.dtype);
  const int32_t vec_per_row = c.head_dim * es / 16;
  const int64_t num_vec = (int64_t)num_tokens * c.num_kv_heads * vec_per_row;
  if (num_vec == 0) return PKV_OK;
  const int threads = 256;
  kv_append_kernel<<<grid_for(num_vec, threads), threads, 0, s>>>(
      static_cast<const int4*>(k), static_cast<const int4*>(v), slots, num_vec, vec_per_row,
      c.num_kv_heads, log2_int(c.block_size), (int64_t)c.num_blocks * c.block_size,
      static_cast<int4*>(k_cache), static_cast<int4*>(v_cache), dbg);
  return check_launch("paged_kv_append");
}

int launch_append_fp8(const void* k, const void* v, const int64_t* slots, int32_t num_tokens,
                      void* k_cache, void* v_cache, float* k_scale, float* v_scale,
                      const pkv_cache_desc& c, int32_t* dbg, cudaStream_t s) {
  const int64_t rows = (int64_t)num_tokens * c.num_kv_heads;
  if (rows == 0) return PKV_OK;
  const int threads = 256;
  kv_append_fp8_kernel<<<grid_for(rows * 32, threads), threads, 0, s>>>(
      static_cast<const uint2*>(k), static_cast<const uint2*>(v), slots, rows, c.num_kv_heads,
      log2_int(c.block_size), (int64_t)c.num_blocks * c.block_size,
      static_cast<uint32_t*>(k_cache), static_cast<uint32_t*>(v_cache), k_scale, v_scale, dbg);
  return check_launch("paged_kv_append_fp8");
}

int launch_gather(const void* k_cache, const void* v_cache, const pkv_cache_desc& c,
                  const int32_t* tables, int32_t max_blocks, const int32_t* lens, int32_t batch,
                  int32_t out_max_len, void* k_out, void* v_out, int32_t* dbg, cudaStream_t s) {
  const int es = dtype_size(c.dtype);
  const int32_t vec_per_row = c.head_dim * es / 16;
  const int64_t num_vec = (int64_t)batch * c.num_kv_heads * out_max_len * vec_per_row;
  if (num_vec == 0) return PKV_OK;
  const int threads = 256;
  kv_gather_kernel<<<grid_for(num_vec, threads), threads, 0, s>>>(
      static_cast<const int4*>(k_cache), static_cast<const int4*>(v_cache), tables, max_blocks,
      lens, num_vec, vec_per_row, c.num_kv_heads, log2_int(c.block_size), c.num_blocks,
      out_max_len, static_cast<int4*>(k_out), static_cast<int4*>(v_out), dbg);
  return check_launch("paged_kv_gather");
}

int launch_copy_spans(void* a, void* b, int64_t bytes_per_block, int32_t num_blocks,
                      const int32_t* pairs, int32_t num_pairs, int32_t* dbg, cudaStream_t s,
                      bool skip_unset) {
  const int64_t vec_per_block = bytes_per_block / 16;
  const int64_t num_vec = (int64_t)num_pairs * vec_per_block;
  if (num_vec == 0) return PKV_OK;
  const int threads = 256;
  kv_copy_blocks_kernel<<<grid_for(num_vec, threads), threads, 0, s>>>(
      static_cast<int4*>(a), static_cast<int4*>(b), pairs, num_vec, vec_per_block, num_blocks,
      skip_unset, dbg);
  return check_launch("paged_kv_copy_blocks");
}

int launch_copy_blocks(void* k_cache, void* v_cache, const pkv_cache_desc& c,
                       const int32_t* pairs, int32_t num_pairs, int32_t* dbg, cudaStream_t s,
                       bool skip_unset) {
  const int64_t bytes = (int64_t)c.num_kv_heads * c.block_size * c.head_dim * dtype_size(c.dtype);
  return launch_copy_spans(k_cache, v_cache, bytes, c.num_blocks, pairs, num_pairs, dbg, s,
                           skip_unset);
}

}  // namespace pkv
