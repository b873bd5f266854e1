// Block-sparse view of a mask modifier: for every (sequence, query head,
// query tile, key tile), whether no query-key pair of the tile is visible
// (the attention kernels skip it), some are (masked element by element), or
// all are (no per-element mask).
//
// Source: "Paged Attention Meets FlexAttention" (abstract) — FlexAttention's
// mask modifiers inside the paged kernel; FlexAttention turns a mask into
// such a per-block table so that fully masked blocks cost nothing.
//
// Every supported mask gives the query at position q the keys [lo(q), hi(q))
// with lo and hi non-decreasing in q and lo(q+1) <= hi(q) (a query always sees
// itself unless the mask is none), so for a tile of queries [q0, q1] the union
// of the rows' intervals is [lo(q0), hi(q1)) and their intersection
// [lo(q1), hi(q0)): a key tile [k0, k1] is skipped if it misses the union and
// full if it lies inside the intersection.
#include "pkv_common.cuh"
#include "pkv_internal.h"

namespace pkv {

namespace {

__global__ void __launch_bounds__(256) block_mask_kernel(
    const int32_t* __restrict__ ctx_lens, const int32_t* __restrict__ q_lens, int32_t batch,
    int32_t num_q_heads, pkv_mask_mod mask, int32_t q_tile, int32_t k_tile, int32_t n_q_tiles,
    int32_t n_k_tiles, uint8_t* __restrict__ out) {
  const int64_t total = (int64_t)batch * num_q_heads * n_q_tiles * n_k_tiles;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    int64_t r = i;
    const int kt = (int)(r % n_k_tiles);
    r /= n_k_tiles;
    const int qt = (int)(r % n_q_tiles);
    r /= n_q_tiles;
    const int h = (int)(r % num_q_heads);
    const int b = (int)(r / num_q_heads);
    const int C = max(0, __ldg(ctx_lens + b));
    const int Q = max(0, __ldg(q_lens + b));
    const int n = C + Q;
    const int q0 = C + qt * q_tile, q1 = min(q0 + q_tile, C + Q) - 1;
    const int k0 = kt * k_tile, k1 = min(k0 + k_tile, n) - 1;
    uint8_t cls = PKV_BLOCK_SKIP;
    if (q0 <= q1 && k0 <= k1) {
      const int any_lo = mask_lo(mask, b, h, q0), any_hi = mask_hi(mask, b, q1, n);
      if (k0 < any_hi && k1 >= any_lo) {
        const int all_lo = mask_lo(mask, b, h, q1), all_hi = mask_hi(mask, b, q0, n);
        cls = (k0 >= all_lo && k1 < all_hi) ? PKV_BLOCK_FULL : PKV_BLOCK_PARTIAL;
      }
    }
    out[i] = cls;
  }
}

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" {

PKV_API int paged_attention_block_mask(const int32_t* ctx_lens, const int32_t* q_lens,
                                       int32_t batch, int32_t num_q_heads, pkv_mask_mod mask,
                                       int32_t q_tile, int32_t k_tile, int32_t n_q_tiles,
                                       int32_t n_k_tiles, uint8_t* out, void* stream) {
  const char* fn = "paged_attention_block_mask";
  clear_last_error();
  if (int st = check_mask(mask, fn)) return st;
  if (batch < 0 || num_q_heads <= 0 || q_tile <= 0 || k_tile <= 0 || n_q_tiles < 0 ||
      n_k_tiles < 0)
    return fail(PKV_ERR_INVALID_ARG, "%s: bad sizes", fn);
  const int64_t total = (int64_t)batch * num_q_heads * n_q_tiles * n_k_tiles;
  if (total == 0) return PKV_OK;
  if (!ctx_lens || !q_lens || !out) return fail(PKV_ERR_INVALID_ARG, "%s: null pointer", fn);
  const int64_t blocks = (total + 255) / 256;
  const int grid = (int)(blocks < (int64_t)device_sm_count() * 8 ? blocks
                                                                 : (int64_t)device_sm_count() * 8);
  block_mask_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      ctx_lens, q_lens, batch, num_q_heads, mask, q_tile, k_tile, n_q_tiles, n_k_tiles, out);
  return check_launch(fn);
}

}  // extern "C"
