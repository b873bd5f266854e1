// Shared-prefix (cascade) decode: beams or samples that share a prompt read
// its KV blocks once per group instead of once per sequence.
//
// Source: "Ultimate Guide to PagedAttention", sections on memory sharing and
// beam search (requests with a common prefix point at the same physical
// blocks, stored once); the split into a shared part and a private part is
// exact because softmax attention over a union of key sets is the
// log-sum-exp merge of the attention over each part ("FlashAttention",
// abstract: exact attention computed tile by tile).
//
// Three launches on the caller's stream:
//  1. prefix: the tensor-core prefill kernel in group mode; a unit is (group,
//     KV head) with every member's query heads as the rows of one query tile
//     (8 beams x 4 heads = 32 rows), so each shared block is loaded once per
//     group and KV head; float32 partials (o, lse) per (sequence, head);
//  2. suffix: the regular paged decode over each sequence's keys from its
//     shared length on (per-sequence key start), written to out and to an
//     internal lse;
//  3. merge: o = w_p o_p + w_s o_s with w = exp(lse_part - lse),
//     lse = log(exp(lse_p) + exp(lse_s)), in place over out.
#include <cmath>

#include "pkv_common.cuh"
#include "pkv_internal.h"

namespace pkv {

namespace {

constexpr int kD = 128;

__global__ void __launch_bounds__(128) shared_prefix_merge_kernel(
    __nv_bfloat16* __restrict__ out, float* __restrict__ lse_out, const float* __restrict__ part_o,
    const float* __restrict__ part_lse, const float* __restrict__ lse_s,
    const int32_t* __restrict__ shared_len, int32_t batch, int32_t num_q_heads) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);  // (sequence, head)
  if (row >= (int64_t)batch * num_q_heads) return;
  const int b = (int)(row / num_q_heads);
  const float ls = lse_s[row];
  float lse = ls;
  if (shared_len[b] > 0) {
    const float lp = part_lse[row];
    const float m = fmaxf(lp, ls);
    if (m != -INFINITY) {
      const float wp = expf(lp - m), ws = expf(ls - m);
      const float inv = 1.f / (wp + ws);
      lse = m + logf(wp + ws);
      const float4 po = reinterpret_cast<const float4*>(part_o + row * kD)[lane];
      uint2 sv = reinterpret_cast<const uint2*>(out + row * kD)[lane];
      const float s0 = __uint_as_float(sv.x << 16), s1 = __uint_as_float(sv.x & 0xffff0000u);
      const float s2 = __uint_as_float(sv.y << 16), s3 = __uint_as_float(sv.y & 0xffff0000u);
      const float a = wp * inv, c = ws * inv;
      uint2 r;
      r.x = pack_bf16x2(a * po.x + c * s0, a * po.y + c * s1);
      r.y = pack_bf16x2(a * po.z + c * s2, a * po.w + c * s3);
      reinterpret_cast<uint2*>(out + row * kD)[lane] = r;
    }
  }
  if (lse_out && lane == 0) lse_out[row] = lse;
}

struct Layout {
  size_t dec, part_o, part_lse, lse_s, total;
};

Layout layout(int32_t batch, int32_t num_q_heads, const pkv_cache_desc& c) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  Layout l;
  l.dec = up(decode_workspace_size(batch, num_q_heads, c));
  const size_t rows = (size_t)batch * num_q_heads;
  l.part_o = l.dec;
  l.part_lse = l.part_o + up(rows * kD * 4);
  l.lse_s = l.part_lse + up(rows * 4);
  l.total = l.lse_s + up(rows * 4);
  return l;
}

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" {

PKV_API size_t paged_attention_decode_shared_prefix_workspace_size(int32_t batch,
                                                                   int32_t num_q_heads,
                                                                   pkv_cache_desc cache) {
  if (check_cache(cache, "paged_attention_decode_shared_prefix_workspace_size") != PKV_OK)
    return 0;
  if (batch <= 0 || num_q_heads <= 0 || num_q_heads % cache.num_kv_heads) return 0;
  return layout(batch, num_q_heads, cache).total;
}

PKV_API int paged_attention_decode_shared_prefix(
    const void* q, const void* k_cache, const void* v_cache, pkv_cache_desc cache,
    const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
    int32_t batch, int32_t num_q_heads, float scale, pkv_mask_mod mask,
    const int32_t* group_start, int32_t num_groups, int32_t max_group_size,
    const int32_t* shared_len, void* out, float* lse, void* workspace, size_t workspace_bytes,
    int32_t* dbg_err, void* stream) {
  const char* fn = "paged_attention_decode_shared_prefix";
  clear_last_error();
  if (int st = check_cache(cache, fn)) return st;
  if (int st = check_mask(mask, fn)) return st;
  if (cache.dtype != PKV_BF16 || cache.head_dim != kD)
    return fail(PKV_ERR_UNSUPPORTED, "%s: bf16 pools with head_dim 128 only", fn);
  if (mask.kind == PKV_MASK_SLIDING)
    return fail(PKV_ERR_UNSUPPORTED, "%s: mask must be none or causal", fn);
  if (batch < 0 || max_blocks_per_seq <= 0)
    return fail(PKV_ERR_INVALID_ARG, "%s: bad batch or max_blocks_per_seq", fn);
  if (num_q_heads <= 0 || num_q_heads % cache.num_kv_heads)
    return fail(PKV_ERR_INVALID_ARG, "%s: num_q_heads %d not a multiple of num_kv_heads %d", fn,
                num_q_heads, cache.num_kv_heads);
  if (!(scale == scale)) return fail(PKV_ERR_INVALID_ARG, "%s: scale is NaN", fn);
  if (batch == 0) return PKV_OK;
  if (num_groups <= 0 || max_group_size <= 0)
    return fail(PKV_ERR_INVALID_ARG, "%s: num_groups and max_group_size must be positive", fn);
  const int g = num_q_heads / cache.num_kv_heads;
  if (max_group_size > batch) max_group_size = batch;  // no group is larger than the batch
  if ((int64_t)max_group_size * g > 128)
    return fail(PKV_ERR_UNSUPPORTED, "%s: max_group_size * (num_q_heads / num_kv_heads) = %lld"
                " exceeds 128 rows", fn, (long long)max_group_size * g);
  if (!q || !k_cache || !v_cache || !block_tables || !seq_lens || !group_start || !shared_len ||
      !out || !workspace)
    return fail(PKV_ERR_INVALID_ARG, "%s: null pointer", fn);
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      !aligned16(workspace))
    return fail(PKV_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", fn);
  const Layout l = layout(batch, num_q_heads, cache);
  if (workspace_bytes < l.total)
    return fail(PKV_ERR_WORKSPACE_TOO_SMALL, "%s: workspace needs %zu bytes, got %zu", fn, l.total,
                workspace_bytes);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* part_o = reinterpret_cast<float*>(ws + l.part_o);
  float* part_lse = reinterpret_cast<float*>(ws + l.part_lse);
  float* lse_s = reinterpret_cast<float*>(ws + l.lse_s);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // 1. shared prefixes, once per (group, KV head)
  GroupPrefixArgs ga{q,        k_cache,        v_cache,    cache,  block_tables, max_blocks_per_seq,
                     seq_lens, batch,          num_q_heads, scale, group_start,  num_groups,
                     max_group_size, shared_len, part_o,    part_lse, dbg_err,   s};
  if (int st = launch_prefix_groups(ga)) return st;
  // 2. each sequence's own keys, from its shared length on
  DecodeArgs a{q,        k_cache, v_cache,     cache, block_tables, max_blocks_per_seq,
               seq_lens, batch,   num_q_heads, scale, mask,         out,
               lse_s,    ws,      l.dec,       dbg_err, s};
  a.key_start = shared_len;
  if (int st = launch_decode(a)) return st;
  // 3. merge in place
  const int64_t rows = (int64_t)batch * num_q_heads;
  shared_prefix_merge_kernel<<<(unsigned)((rows + 3) / 4), 128, 0, s>>>(
      static_cast<__nv_bfloat16*>(out), lse, part_o, part_lse, lse_s, shared_len, batch,
      num_q_heads);
  return check_launch(fn);
}

}  // extern "C"
