// Pieces of the paged chunked-prefill kernel: the parameters, the unit of
// work and its key tiles, bounded waits, named barriers and TMA helpers. Method: "Paged Attention Meets FlexAttention"
// (abstract) with the exact tiled softmax of "FlashAttention" (abstract).
#pragma once

#include <cmath>

#include "pkv_common.cuh"
#include "pkv_internal.h"

namespace pkv {
namespace pf {

constexpr int kD = 128;                   // head dim
constexpr int kM = 128;                   // query rows per tile
constexpr int kN = 128;                   // keys per tile
constexpr int kTileBytes = kN * kD * 2;   // 32 KB (K or V or Q tile)
constexpr int kHalfBytes = kTileBytes / 2;
constexpr int kMaxBatch = 4096;
constexpr float kRescaleThreshold = 8.f;  // log2 units

struct PrefillParams {
  const int32_t* tables;
  int32_t max_blocks;
  const int32_t* ctx_lens;
  const int32_t* q_lens;
  int32_t batch;
  int32_t total_q;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t group;
  int32_t pairs;        // units per KV head and query tile: group/2 (two heads) or group (one head)
  int32_t two_heads;    // 1 when a unit holds two query heads
  int32_t bs_shift;
  int32_t box_rows;     // rows of one paged TMA box (min(block_size, 16))
  int32_t num_blocks;
  int32_t pool_rows;    // num_blocks * Hkv * block_size (first out-of-bounds row)
  float scale_log2;
  pkv_mask_mod mask;
  __nv_bfloat16* out;
  float* lse;
  int32_t* dbg;
};

struct Unit {
  bool valid;
  int b, kvh, hp, qt;
  int C, Q, qoff;
  int ctx_lo, n_ctx;   // context tiles [ctx_lo, ctx_lo + n_ctx)
  int ch_lo, n_ch;     // chunk tiles   [ch_lo, ch_lo + n_ch)
  __device__ int n() const { return n_ctx + n_ch; }
};

__device__ __forceinline__ Unit unit_of(const PrefillParams& p, const int32_t* qoff, int max_qt,
                                        int64_t u) {
  // (sequence, KV head) major: the units that stream the same K/V (every
  // query tile and head pair of a KV head) are consecutive, so the CTAs of a
  // wave share a few K/V streams through L2; within them, the last (longest)
  // query tile first
  Unit x;
  const int64_t per_kv = (int64_t)max_qt * p.pairs;
  const int64_t sh = u / per_kv;
  const int64_t rem = u - sh * per_kv;
  x.b = (int)(sh / p.num_kv_heads);
  x.kvh = (int)(sh % p.num_kv_heads);
  const int qt_rev = (int)(rem / p.pairs);
  x.hp = (int)(rem % p.pairs);
  x.qt = max_qt - 1 - qt_rev;
  x.Q = qoff[x.b + 1] - qoff[x.b];
  x.qoff = qoff[x.b];
  x.valid = x.qt >= 0 && x.qt * kM < x.Q;
  if (!x.valid) return x;
  int C = p.ctx_lens[x.b];
  if (C < 0) C = 0;
  const int cap = p.max_blocks << p.bs_shift;
  if (C > cap) {
    flag_error(p.dbg, PKV_DBG_LENGTH);
    C = cap;
  }
  x.C = C;
  const int qmin = C + x.qt * kM;                        // position of the tile's first row
  const int qlast = min(qmin + kM - 1, C + x.Q - 1);     // and of its last real row
  const int ctx_tiles = (C + kN - 1) / kN;
  // keys any row of the tile can see: [lowest start over the unit's heads at
  // its first row, end at its last row) (both ends grow with the position)
  const int h0 = x.kvh * p.group + x.hp * (p.two_heads ? 2 : 1);
  int lo_key = mask_lo(p.mask, x.b, h0, qmin);
  if (p.two_heads) lo_key = min(lo_key, mask_lo(p.mask, x.b, h0 + 1, qmin));
  const int hi_key = mask_hi(p.mask, x.b, qlast, C + x.Q);
  x.ctx_lo = min(lo_key / kN, ctx_tiles);
  x.n_ctx = ctx_tiles - x.ctx_lo;
  const int ch_hi = hi_key > C ? (hi_key - 1 - C) / kN : -1;
  x.ch_lo = (lo_key > C) ? (lo_key - C) / kN : 0;
  x.n_ch = max(0, ch_hi - x.ch_lo + 1);
  return x;
}

// Tile j of a unit: is it a context tile, and the position of its first key.
__device__ __forceinline__ void tile_of(const Unit& x, int j, bool& ctx, int& idx, int& kp0) {
  if (j < x.n_ctx) {
    ctx = true;
    idx = x.ctx_lo + j;
    kp0 = idx * kN;
  } else {
    ctx = false;
    idx = x.ch_lo + (j - x.n_ctx);
    kp0 = x.C + idx * kN;
  }
}

// A context tile whose 16-row box straddles the context end holds rows past
// it that come from the pool (stale, possibly non-finite); they are zeroed in
// shared memory before the MMAs read the tile.
__device__ __forceinline__ bool needs_fix(const Unit& x, bool ctx, int kp0, int box_rows) {
  return ctx && kp0 < x.C && kp0 + kN > x.C && (x.C % box_rows) != 0;
}

// Warp-collective bounded wait: every lane of the warp calls it and gets the
// same answer, so the warp never splits around the warp-wide tcgen05
// instructions that follow. With `all_lanes` false only lane 0 polls (the
// warp's other lanes are ordered after it by the warp barrier). On a timeout
// (or an abort raised by another warp) it records PKV_DBG_TIMEOUT and tells
// every role to stop.
__device__ __forceinline__ bool wait_or_flag(uint32_t bar, uint32_t parity, int32_t* dbg,
                                             int* abort_flag, bool all_lanes = false) {
  bool ok = true;
  if (all_lanes || (threadIdx.x & 31) == 0)
    ok = *reinterpret_cast<volatile int*>(abort_flag) == 0 && mbar_wait(bar, parity);
  ok = __all_sync(0xffffffffu, ok);
  __syncwarp();
  if (!ok && (threadIdx.x & 31) == 0) {
    flag_error(dbg, PKV_DBG_TIMEOUT);
    *reinterpret_cast<volatile int*>(abort_flag) = 1;
  }
  return ok;
}

// Named barrier of `n` threads; the `and` form also returns whether `pred`
// held in all of them (every arriving thread gets the same answer).
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ bool named_and(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// 3-D TMA tile load (inner coordinate first).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int32_t c0,
                                            int32_t c1, int32_t c2, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

struct Maps {
  CUtensorMap q;       // 3-D {D, Hq, total_q}, box {64, 1, 128}
  CUtensorMap knew;    // 3-D {D, Hkv, total_q}, box {64, 1, 128}
  CUtensorMap vnew;
  CUtensorMap kpool;   // 2-D {D, pool rows}, box {64, box_rows}
  CUtensorMap vpool;
};

// 18 warps: five on two of the SM's four sub-partitions, whose 16K-register
// files then allow at most 96 registers a thread

// Exclusive prefix of q_lens over the batch into qoff[0..batch] and the
// largest number of query tiles of a sequence into *max_qt (one warp; lane 0
// writes the totals). Flags PKV_DBG_QLEN_SUM (block 0) when the lengths do not
// add up to total_q.
__device__ __forceinline__ void query_offsets(const PrefillParams& p, int lane, int32_t* qoff,
                                              int32_t* max_qt) {
  int run = 0, mq = 0;
  for (int base = 0; base < p.batch; base += 32) {
    const int b = base + lane;
    int q = b < p.batch ? max(0, p.q_lens[b]) : 0;
    mq = max(mq, (q + kM - 1) / kM);
    int incl = q;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (b < p.batch) qoff[b] = run + incl - q;
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) mq = max(mq, __shfl_xor_sync(0xffffffffu, mq, o));
  if (lane == 0) {
    qoff[p.batch] = run;
    *max_qt = mq;
    if (run != p.total_q && blockIdx.x == 0) flag_error(p.dbg, PKV_DBG_QLEN_SUM);
  }
}

}  // namespace pf


}  // namespace pkv
