// Paged decode attention: one query token per sequence over its paged KV.
//
// Method: "Paged Attention Meets FlexAttention" (abstract) — a fused kernel
// that gathers the scattered KV blocks through the block table and applies
// the mask modifier inside the kernel — with the exact, tiled online softmax
// of "FlashAttention" (abstract). Layout and indexing: "Ultimate Guide to
// PagedAttention", KV-block and block-table sections.
//
// B200 design (bf16):
//  * Work is a flat list of 16-token tiles: for every (sequence b, KV head)
//    segment, the tiles that hold visible keys (a sliding window drops whole
//    tiles before it). Each worker (one warp) takes one contiguous range of
//    that list, so every worker streams the same number of bytes whatever
//    the length mix; a segment cut between workers leaves (o, lse) partials
//    that a second kernel merges by log-sum-exp. The split depends only on
//    the lengths and the window, never on block ids, so the result is
//    bit-identical under any placement of the blocks.
//  * 12 workers per CTA, one CTA per SM: each warp is one serial stream of
//    dependent MMA/shuffle work, so the SM needs several warps per
//    sub-partition to issue every cycle (4 warps reached 59% of HBM peak,
//    12 warps 86%). Each warp runs its own NSTAGE-deep TMA ring: a 16-row x 64-column box
//    per 128-byte half of the head row, 128-byte swizzled, so the tensor-core
//    fragment loads (ldmatrix) are bank-conflict free. Block ids are loaded
//    one tile ahead of the copy that needs them.
//  * The query-head group of a KV head (g <= 8) is the N=8 side of
//    mma.sync m16n8k16 (bf16 in, fp32 accumulate): S^T = K Q^T puts the 16
//    tokens of a tile on M, so every KV byte is read once for the whole
//    group. P^T is turned into the B operand of O^T += V^T P^T with
//    movmatrix, without a trip through shared memory.
//  * fp32 pools use a plain CUDA-core kernel (one CTA per (b, q head)).
#include <cmath>

#include "pkv_common.cuh"
#include "pkv_internal.h"

namespace pkv {

constexpr int kTile = 16;            // tokens per tile
constexpr int kMinTilesPerWorker = 2;
constexpr int kMaxWarpsPerCta = 12;  // largest built bf16 variant (sizes the workspace)

struct DecodeParams {
  const __nv_bfloat16* q;
  const int32_t* tables;
  int32_t max_blocks;
  const int32_t* seq_lens;
  int32_t batch;
  int32_t num_kv_heads;
  int32_t group;       // query heads per KV head
  int32_t num_q_heads;
  int32_t bs_shift;    // log2(block_size)
  int32_t num_blocks;
  float scale_log2;    // scale * log2(e)
  pkv_mask_mod mask;
  const float* k_scale;  // E4M3 pools: float32 scale of each stored row [pool rows]
  const float* v_scale;
  // fused append: each sequence's newest token [batch, num_kv_heads, D], written
  // into the pools at position seq_lens[b]-1 of its block table
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k_pool;
  __nv_bfloat16* v_pool;
  __nv_bfloat16* out;
  float* lse;
  float* ws_o;         // [2 * workers, group, D] partial outputs (normalised)
  float* ws_lse;       // [2 * workers, group] partial lse (natural log)
  int32_t* ws_prefix;  // [batch + 1] tiles per KV head before sequence b
  int32_t workers;     // warps launched
  int32_t* dbg;
};

// Visible range and tile span of sequence b.
struct SeqSpan {
  int lo, hi;      // visible keys [lo, hi)
  int t0;          // first tile (in 16-token units of position)
  int n;           // tiles
};

__device__ __forceinline__ SeqSpan seq_span(const DecodeParams& p, int b) {
  SeqSpan s;
  int L = __ldg(p.seq_lens + b);
  if (L < 0) L = 0;
  const int cap = p.max_blocks << p.bs_shift;
  if (L > cap) {
    flag_error(p.dbg, PKV_DBG_LENGTH);
    L = cap;
  }
  decode_key_range(p.mask, p.num_q_heads, b, L, s.lo, s.hi);
  s.t0 = s.lo / kTile;
  s.n = s.hi > s.lo ? (s.hi + kTile - 1) / kTile - s.t0 : 0;
  return s;
}

// Tiles per KV head summed over all sequences (warp-cooperative; every lane
// gets the result). If `prefix` is not null, also writes the exclusive
// prefix over sequences (batch + 1 entries).
__device__ __forceinline__ int total_tiles(const DecodeParams& p, int lane, int32_t* prefix) {
  int run = 0;
  for (int base = 0; base < p.batch; base += 32) {
    const int b = base + lane;
    int n = b < p.batch ? seq_span(p, b).n : 0;
    int incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int x = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += x;
    }
    if (prefix && b < p.batch) prefix[b] = run + incl - n;
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (prefix && lane == 0) prefix[p.batch] = run;
  return run;
}

// Sequence holding global tile x (x < total): returns b and the number of
// tiles (over all KV heads) before sequence b.
__device__ __forceinline__ void find_seq(const DecodeParams& p, int lane, int64_t x, int& b_out,
                                         int64_t& before) {
  const int H = p.num_kv_heads;
  int64_t run = 0;
  for (int base = 0; base < p.batch; base += 32) {
    const int b = base + lane;
    int n = b < p.batch ? seq_span(p, b).n : 0;
    int incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    // first lane whose inclusive end (over all heads) passes x
    const bool hit = b < p.batch && run + (int64_t)incl * H > x;
    const unsigned m = __ballot_sync(0xffffffffu, hit);
    if (m) {
      const int src = __ffs(m) - 1;
      const int excl = __shfl_sync(0xffffffffu, incl - n, src);
      b_out = base + src;
      before = run + (int64_t)excl * H;
      return;
    }
    run += (int64_t)__shfl_sync(0xffffffffu, incl, 31) * H;
  }
  b_out = p.batch;
  before = run;
}

__device__ __forceinline__ int workers_for(int64_t total, int launched) {
  // a list that fits half the launched warps one tile each takes one tile per
  // warp (shortest latency for small batches); longer lists give every warp
  // at least kMinTilesPerWorker, which halves the pieces the merge reads
  // (batch 1 at 2048 tokens: 24 us with two tiles per warp, 28 us with one)
  if (2 * total <= launched) return total > 0 ? (int)total : 1;
  int64_t w = total / kMinTilesPerWorker;
  return (int)(w < launched ? w : launched);
}

// Cursor over the flat tile list (uniform across the warp).
struct Cursor {
  int b, kvh;
  SeqSpan s;
  int64_t seg_first;  // global index of the segment's first tile
  int64_t t;          // global tile index
};

__device__ __forceinline__ void cursor_next_seq(const DecodeParams& p, Cursor& c) {
  // move to the next sequence with tiles (caller has set seg_first)
  do {
    ++c.b;
    if (c.b >= p.batch) return;
    c.s = seq_span(p, c.b);
  } while (c.s.n == 0);
  c.kvh = 0;
}

__device__ __forceinline__ void cursor_advance(const DecodeParams& p, Cursor& c) {
  ++c.t;
  if (c.t == c.seg_first + c.s.n) {
    c.seg_first += c.s.n;
    if (c.kvh + 1 < p.num_kv_heads) {
      ++c.kvh;
    } else {
      cursor_next_seq(p, c);
    }
  }
}

// Shared-memory layout. bf16 pools: a stage is a K tile then a V tile (16
// rows x D, 128-byte-swizzled halves of 64 columns). E4M3 pools (KV8, D = 128):
// a stage is a K tile then a V tile of 16 rows x 128 one-byte codes (one
// swizzled 128-byte row per token), plus 128 bytes of row scales (K then V)
// per stage.
template <int D, bool KV8 = false>
struct Cfg {
  static constexpr int kHalves = KV8 ? 1 : D / 64;            // TMA boxes per row
  static constexpr int kTileBytes = kTile * D * (KV8 ? 1 : 2);  // K (or V) bytes of one tile
  static constexpr int kStageBytes = 2 * kTileBytes;           // K then V
  static constexpr int kScaleBytes = KV8 ? 2 * kTile * 4 : 0;
};

// PH: per-head sliding windows (each head column masks keys below its own
// start); the instance without them carries none of that code.
// KV8: E4M3 pools with a float32 scale per stored row (D = 128). Codes are
// decoded exactly to f16 (cvt.rn.f16x2.e4m3x2) in registers and the MMAs run
// in f16. K: each ldmatrix word holds four codes of one token, decoded into
// the A fragments of two k16 steps whose k order the query fragments follow.
// V: the codes are read transposed (ldmatrix .trans on byte pairs), each word
// regrouped per head_dim column with a byte permute, so one word gives the
// A-fragment pairs of two head_dim columns (2r and 2r + 1 of the 16-column
// block: an accumulator row r holds the column 2r, row r + 8 the column
// 2r + 1). K's row scales multiply the scores, V's row scales (times 256,
// which keeps the products clear of f16 subnormals and is divided out at the
// end) multiply P.
// APPEND: the decode step's append is fused in. The worker that holds the last
// tile of a (sequence, KV head) segment writes that sequence's new token
// (k_new/v_new) into the pools at position seq_lens[b]-1 of its block table
// and into the tile it has just loaded, over the row the pool held before; no
// other worker reads that row, so the result is that of an append followed by
// a decode.
template <int D, int NSTAGE, int WPC, bool PH, bool KV8, bool APPEND = false>
__global__ void __launch_bounds__(WPC * 32, 1)
    decode_bf16_kernel(const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap, const DecodeParams p) {
  using C = Cfg<D, KV8>;
  static_assert(!KV8 || D == 128, "E4M3 pools are built for head_dim 128");
  constexpr float kVScale = 256.f;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzle atoms
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  uint8_t* ring = smem + warp * NSTAGE * C::kStageBytes;
  float* scl = reinterpret_cast<float*>(smem + WPC * NSTAGE * C::kStageBytes) +
               warp * NSTAGE * (C::kScaleBytes / 4);
  uint64_t* bars = reinterpret_cast<uint64_t*>(
                       smem + WPC * NSTAGE * (C::kStageBytes + C::kScaleBytes)) +
                   warp * NSTAGE;

  const int gw = blockIdx.x * WPC + warp;
  const bool writer = (gw == 0);
  const int64_t T = (int64_t)total_tiles(p, lane, writer ? p.ws_prefix : nullptr) * p.num_kv_heads;
  const int W = workers_for(T, p.workers);
  if (gw >= W || T == 0) return;
  const int64_t start = (int64_t)gw * T / W;
  const int64_t end = (int64_t)(gw + 1) * T / W;
  if (start >= end) return;

  if (lane == 0) {
    prefetch_tmap(&kmap);
    prefetch_tmap(&vmap);
    for (int i = 0; i < NSTAGE; ++i) mbar_init(smem_u32(bars + i), 1);
    fence_barrier_init();
  }
  __syncwarp();

  // locate the first tile
  Cursor cur;
  {
    int b;
    int64_t before;
    find_seq(p, lane, start, b, before);
    cur.b = b;
    cur.s = seq_span(p, b);
    const int64_t off = start - before;
    cur.kvh = (int)(off / cur.s.n);
    cur.seg_first = before + (int64_t)cur.kvh * cur.s.n;
    cur.t = start;
  }
  Cursor pc = cur;  // producer cursor

  const int bs_mask = (1 << p.bs_shift) - 1;
  const int box_rows = p.bs_shift >= 4 ? kTile : (1 << p.bs_shift);  // 8 or 16
  const int pieces = kTile / box_rows;                                // 1 or 2
  const uint64_t evict_first = policy_evict_first();

  // block ids of the producer's next tile (lane 0 only), loaded one step ahead
  int pid0 = 0, pid1 = 0;
  auto load_ids = [&](const Cursor& c) {
    if (lane != 0 || c.b >= p.batch) return;
    const int tok0 = (c.s.t0 + (int)(c.t - c.seg_first)) * kTile;
    const int j = tok0 >> p.bs_shift;
    const int32_t* row = p.tables + (int64_t)c.b * p.max_blocks;
    pid0 = j < p.max_blocks ? __ldg(row + j) : -1;
    if (pieces == 2) pid1 = (j + 1 < p.max_blocks && tok0 + 8 < c.s.hi) ? __ldg(row + j + 1) : -1;
  };
  auto issue = [&](const Cursor& c, int stage) {
    if (lane != 0) return;
    const int tok0 = (c.s.t0 + (int)(c.t - c.seg_first)) * kTile;
    const uint32_t bar = smem_u32(bars + stage);
    const uint32_t kdst = smem_u32(ring + stage * C::kStageBytes);
    const uint32_t vdst = kdst + C::kTileBytes;
    int ids[2] = {pid0, pid1};
    bool need[2];
    uint32_t bytes = 0;
    for (int pi = 0; pi < pieces; ++pi) {
      const int a = tok0 + pi * box_rows;
      need[pi] = a < c.s.hi && a + box_rows > c.s.lo;
      if (need[pi]) {
        if (ids[pi] < 0 || ids[pi] >= p.num_blocks) {
          flag_error(p.dbg, PKV_DBG_BLOCK_ID);
          ids[pi] = 0;
        }
        bytes += KV8 ? 2u * box_rows * (D + 4) : 2u * box_rows * D * 2;
      }
    }
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar, bytes);
    for (int pi = 0; pi < pieces; ++pi) {
      if (!need[pi]) continue;
      const int row = ((ids[pi] * p.num_kv_heads + c.kvh) << p.bs_shift) +
                      ((tok0 + pi * box_rows) & bs_mask);
#pragma unroll
      for (int h = 0; h < C::kHalves; ++h) {
        const uint32_t o = h * (kTile * 128) + pi * box_rows * 128;
        tma_load_2d_hint(kdst + o, &kmap, h * (KV8 ? 128 : 64), row, bar, evict_first);
        tma_load_2d_hint(vdst + o, &vmap, h * (KV8 ? 128 : 64), row, bar, evict_first);
      }
      if constexpr (KV8) {
        const uint32_t sdst = smem_u32(scl + stage * 2 * kTile) + pi * box_rows * 4;
        bulk_load_1d(sdst, p.k_scale + row, box_rows * 4, bar);
        bulk_load_1d(sdst + kTile * 4, p.v_scale + row, box_rows * 4, bar);
      }
    }
  };

  const int64_t ntiles = end - start;
  // prologue: fill NSTAGE-1 stages
  load_ids(pc);
  int64_t issued = 0;
  for (; issued < NSTAGE - 1 && issued < ntiles; ++issued) {
    issue(pc, (int)(issued % NSTAGE));
    cursor_advance(p, pc);
    if (issued + 1 < ntiles) load_ids(pc);
  }

  // lane roles in the mma fragments
  const int g4 = lane >> 2;        // row (token) within 8, or head column for B
  const int c4 = lane & 3;
  const int mi = lane >> 3, mr = lane & 7;
  const int krow = mr + ((mi & 1) << 3);   // K tile row this lane addresses
  const int kco = mi >> 1;                 // +0/+1 chunk for k 0-7 / 8-15
  const int vtok = mr + ((mi >> 1) << 3);  // V tile row (token) this lane addresses
  const int vco = mi & 1;
  // head_dim columns of accumulator rows g4 and g4 + 8 within a 16-column block
  const int dlo = KV8 ? 2 * g4 : g4, dhi = KV8 ? 2 * g4 + 1 : g4 + 8;

  uint32_t qf[D / 16][2];
  float o[D / 16][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  int piece = 0;  // 0 for the worker's first piece, 1 afterwards
  int64_t piece_start = start;
  // per-head windows: the segment spans the union of the heads' ranges and
  // each of this lane's two head columns masks keys below its own start
  constexpr bool per_head = PH;
  int lo_h0 = 0, lo_h1 = 0;

  for (int64_t k = 0; k < ntiles; ++k) {
    // producer: refill the stage consumed in the previous iteration
    if (issued < ntiles) {
      issue(pc, (int)(issued % NSTAGE));
      cursor_advance(p, pc);
      ++issued;
      if (issued < ntiles) load_ids(pc);
    }
    const bool seg_begin = (k == 0) || (cur.t == cur.seg_first);
    if (seg_begin) {
      piece_start = cur.t;
      // query fragments of this (b, kv head): B operand, column = head g4
      const int hq = cur.kvh * p.group + g4;
      const __nv_bfloat16* qrow = p.q + ((int64_t)cur.b * p.num_q_heads + hq) * D;
      if constexpr (KV8) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          if (g4 < p.group) {
            // f16 B fragments in the k order of the E4M3 A fragments: step kk
            // covers columns 16kk..16kk+15, this lane's four at 16kk + 4*c4
            const uint2 w = __ldg(reinterpret_cast<const uint2*>(qrow + kk * 16 + 4 * c4));
            qf[kk][0] = pack_f16x2(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u));
            qf[kk][1] = pack_f16x2(__uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
          } else {
            qf[kk][0] = qf[kk][1] = 0u;
          }
        }
      } else {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          if (g4 < p.group) {
            qf[kk][0] = __ldg(reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * c4));
            qf[kk][1] = __ldg(reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 8 + 2 * c4));
          } else {
            qf[kk][0] = qf[kk][1] = 0u;
          }
        }
      }
      if (per_head) {
        const int L = cur.s.hi;
        const int hb = cur.kvh * p.group + 2 * c4;
        lo_h0 = 2 * c4 < p.group ? mask_lo(p.mask, cur.b, hb, L - 1) : 0;
        lo_h1 = 2 * c4 + 1 < p.group ? mask_lo(p.mask, cur.b, hb + 1, L - 1) : 0;
      }
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
    }

    const int stage = (int)(k % NSTAGE);
    const uint32_t parity = (uint32_t)((k / NSTAGE) & 1);
    uint8_t* kst = ring + stage * C::kStageBytes;
    const uint32_t kbase = smem_u32(kst);
    const uint32_t vbase = kbase + C::kTileBytes;
    if (!mbar_wait(smem_u32(bars + stage), parity)) {
      flag_error(p.dbg, PKV_DBG_TIMEOUT);
      return;
    }
    const int tok0 = (cur.s.t0 + (int)(cur.t - cur.seg_first)) * kTile;
    const bool partial = tok0 < cur.s.lo || tok0 + kTile > cur.s.hi;
    if constexpr (APPEND) {
      const int last = cur.s.hi - 1;  // the new token's position
      if (last >= tok0 && last < tok0 + kTile) {
        // 16-byte chunks of the new K row (lanes 0..D/8-1) and V row (the next D/8)
        constexpr int kChunks = D / 8;
        const int r = last - tok0;
        if (lane < 2 * kChunks) {
          const bool isv = lane >= kChunks;
          const int ch = isv ? lane - kChunks : lane;
          const int64_t src = ((int64_t)cur.b * p.num_kv_heads + cur.kvh) * D;
          const uint4 val =
              __ldg(reinterpret_cast<const uint4*>((isv ? p.v_new : p.k_new) + src) + ch);
          *reinterpret_cast<uint4*>(kst + (isv ? C::kTileBytes : 0) + (ch >> 3) * (kTile * 128) +
                                    r * 128 + (((ch & 7) ^ (r & 7)) << 4)) = val;
          const int j = last >> p.bs_shift;
          const int blk = j < p.max_blocks ? __ldg(p.tables + (int64_t)cur.b * p.max_blocks + j) : -1;
          if (blk >= 0 && blk < p.num_blocks) {
            const int64_t grow = ((int64_t)(blk * p.num_kv_heads + cur.kvh) << p.bs_shift) +
                                 (last & bs_mask);
            *(reinterpret_cast<uint4*>((isv ? p.v_pool : p.k_pool) + grow * D) + ch) = val;
          }  // an invalid id was flagged when the tile was loaded
        }
        // these generic writes precede the next TMA write of this stage
        fence_proxy_async_smem();
        __syncwarp();
      }
    }
    if (partial) {
      // rows outside [lo, hi) may hold stale or non-finite data: zero them in V
      for (int i = lane; i < kTile * C::kHalves * 8; i += 32) {
        const int h = i / (kTile * 8);
        const int r = (i / 8) % kTile;
        const int ch = i % 8;
        const int pos = tok0 + r;
        if (pos < cur.s.lo || pos >= cur.s.hi)
          *reinterpret_cast<int4*>(kst + C::kTileBytes + h * (kTile * 128) + r * 128 + ch * 16) =
              make_int4(0, 0, 0, 0);
      }
      // these generic writes precede the next TMA write of this stage
      fence_proxy_async_smem();
      __syncwarp();
    }

    // S^T (16 tokens x 8 heads) = K (16 x D) * Q^T (D x 8)
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
    if constexpr (KV8) {
      // one ldmatrix covers 32 codes of 16 rows; each 16-bit unit holds two
      // codes, decoded into the f16 A fragments of two k16 steps whose k
      // order the query fragments follow
#pragma unroll
      for (int s2 = 0; s2 < D / 32; ++s2) {
        const int chunk = 2 * s2 + kco;
        uint32_t r[4];
        ldmatrix_x4(r, kbase + krow * 128 + ((chunk ^ (krow & 7)) << 4));
        uint32_t a[4];
        a[0] = e4m3x2_to_f16x2(r[0]);
        a[1] = e4m3x2_to_f16x2(r[1]);
        a[2] = e4m3x2_to_f16x2(r[0] >> 16);
        a[3] = e4m3x2_to_f16x2(r[1] >> 16);
        mma_f16_16816(sa, a, qf[2 * s2][0], qf[2 * s2][1]);
        a[0] = e4m3x2_to_f16x2(r[2]);
        a[1] = e4m3x2_to_f16x2(r[3]);
        a[2] = e4m3x2_to_f16x2(r[2] >> 16);
        a[3] = e4m3x2_to_f16x2(r[3] >> 16);
        mma_f16_16816(sb, a, qf[2 * s2 + 1][0], qf[2 * s2 + 1][1]);
      }
    } else {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int chunk = 2 * kk + kco;
        const uint32_t addr = kbase + (chunk >> 3) * (kTile * 128) + krow * 128 +
                              (((chunk & 7) ^ (krow & 7)) << 4);
        uint32_t a[4];
        ldmatrix_x4(a, addr);
        if (kk & 1)
          mma_bf16_16816(sb, a, qf[kk][0], qf[kk][1]);
        else
          mma_bf16_16816(sa, a, qf[kk][0], qf[kk][1]);
      }
    }
    // element e: token g4 (+8 for e >= 2), head 2*c4 + (e & 1)
    float x[4];
    if constexpr (KV8) {
      const float* ks = scl + stage * 2 * kTile;  // this tile's K row scales
      const float k0 = ks[g4] * p.scale_log2, k1 = ks[g4 + 8] * p.scale_log2;
      x[0] = (sa[0] + sb[0]) * k0;
      x[1] = (sa[1] + sb[1]) * k0;
      x[2] = (sa[2] + sb[2]) * k1;
      x[3] = (sa[3] + sb[3]) * k1;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) x[e] = (sa[e] + sb[e]) * p.scale_log2;
    }
    if (partial) {
      const int p0 = tok0 + g4, p1 = p0 + 8;
      if (p0 < cur.s.lo || p0 >= cur.s.hi) x[0] = x[1] = -INFINITY;
      if (p1 < cur.s.lo || p1 >= cur.s.hi) x[2] = x[3] = -INFINITY;
    }
    if (per_head) {
      const int p0 = tok0 + g4, p1 = p0 + 8;
      if (p0 < lo_h0) x[0] = -INFINITY;
      if (p0 < lo_h1) x[1] = -INFINITY;
      if (p1 < lo_h0) x[2] = -INFINITY;
      if (p1 < lo_h1) x[3] = -INFINITY;
    }
    float mx0 = fmaxf(x[0], x[2]), mx1 = fmaxf(x[1], x[3]);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    // every tile of a piece holds a key visible to all heads of the group, so
    // the new maxima are finite; with per-head windows a head may have seen
    // none yet (maximum -inf), and 0 stands in as the reference then
    const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
    float r0 = n0, r1 = n1;
    if (per_head) {
      r0 = n0 == -INFINITY ? 0.f : n0;
      r1 = n1 == -INFINITY ? 0.f : n1;
    }
    const float al0 = fast_exp2(m0 - r0), al1 = fast_exp2(m1 - r1);
    m0 = n0;
    m1 = n1;
    const float p00 = fast_exp2(x[0] - r0), p01 = fast_exp2(x[1] - r1);
    const float p10 = fast_exp2(x[2] - r0), p11 = fast_exp2(x[3] - r1);
    l0 = l0 * al0 + p00 + p10;
    l1 = l1 * al1 + p01 + p11;
    if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        o[mt][0] *= al0;
        o[mt][1] *= al1;
        o[mt][2] *= al0;
        o[mt][3] *= al1;
      }
    }
    // P^T rows (tokens) -> B operand (k = token, n = head) via 8x8 transposes
    uint32_t pb0, pb1;
    if constexpr (KV8) {
      // V's row scale (x 256) joins P; rows outside [lo, hi) get 0, whatever
      // their stored scale holds
      const float* vs = scl + stage * 2 * kTile + kTile;
      const int q0 = tok0 + g4, q1 = q0 + 8;
      const float v0 = (q0 >= cur.s.lo && q0 < cur.s.hi) ? vs[g4] * kVScale : 0.f;
      const float v1 = (q1 >= cur.s.lo && q1 < cur.s.hi) ? vs[g4 + 8] * kVScale : 0.f;
      pb0 = movmatrix_trans(pack_f16x2(p00 * v0, p01 * v0));
      pb1 = movmatrix_trans(pack_f16x2(p10 * v1, p11 * v1));
    } else {
      pb0 = movmatrix_trans(pack_bf16x2(p00, p01));
      pb1 = movmatrix_trans(pack_bf16x2(p10, p11));
    }
    // O^T (D x 8) += V^T (D x 16 tokens) * P^T (16 x 8)
    if constexpr (KV8) {
      // one transposed load covers two 16-code column blocks: r[0] / r[1] the
      // first block's tokens 0-7 / 8-15, r[2] / r[3] the second's; each word
      // holds columns 2g4, 2g4 + 1 of tokens 2c4, 2c4 + 1, regrouped per column
#pragma unroll
      for (int cp = 0; cp < D / 32; ++cp) {
        const int chunk = 2 * cp + (mi >> 1);
        uint32_t r[4];
        ldmatrix_x4_trans(r, vbase + krow * 128 + ((chunk ^ (krow & 7)) << 4));
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint32_t x0 = byte_perm(r[2 * hh], 0u, 0x3120u);
          const uint32_t x1 = byte_perm(r[2 * hh + 1], 0u, 0x3120u);
          uint32_t a[4];
          a[0] = e4m3x2_to_f16x2(x0);
          a[1] = e4m3x2_to_f16x2(x0 >> 16);
          a[2] = e4m3x2_to_f16x2(x1);
          a[3] = e4m3x2_to_f16x2(x1 >> 16);
          mma_f16_16816(o[2 * cp + hh], a, pb0, pb1);
        }
      }
    } else {
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        const int chunk = 2 * mt + vco;
        const uint32_t addr = vbase + (chunk >> 3) * (kTile * 128) + vtok * 128 +
                              (((chunk & 7) ^ (vtok & 7)) << 4);
        uint32_t a[4];
        ldmatrix_x4_trans(a, addr);
        mma_bf16_16816(o[mt], a, pb0, pb1);
      }
    }
    __syncwarp();

    // end of this worker's piece of the segment?
    const int64_t seg_end = cur.seg_first + cur.s.n;
    const bool piece_end = (k == ntiles - 1) || (cur.t + 1 == seg_end);
    if (piece_end) {
      float s0 = l0, s1 = l1;
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        s0 += __shfl_xor_sync(0xffffffffu, s0, off);
        s1 += __shfl_xor_sync(0xffffffffu, s1, off);
      }
      // a head that saw no key in this piece (per-head windows) gives 0, -inf
      const float un = KV8 ? 1.f / kVScale : 1.f;  // E4M3: O carries V's extra factor
      const float inv0 = s0 > 0.f ? un / s0 : 0.f, inv1 = s1 > 0.f ? un / s1 : 0.f;
      const float lse0 = s0 > 0.f ? m0 * kLn2 + logf(s0) : -INFINITY;
      const float lse1 = s1 > 0.f ? m1 * kLn2 + logf(s1) : -INFINITY;
      const int h0 = 2 * c4, h1 = h0 + 1;
      const bool whole = (piece_start == cur.seg_first) && (cur.t + 1 == seg_end);
      if (whole) {
        const int64_t obase = ((int64_t)cur.b * p.num_q_heads + cur.kvh * p.group) * D;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          const int d0 = mt * 16 + dlo, d1 = mt * 16 + dhi;
          if (h0 < p.group) {
            p.out[obase + h0 * D + d0] = __float2bfloat16_rn(o[mt][0] * inv0);
            p.out[obase + h0 * D + d1] = __float2bfloat16_rn(o[mt][2] * inv0);
          }
          if (h1 < p.group) {
            p.out[obase + h1 * D + d0] = __float2bfloat16_rn(o[mt][1] * inv1);
            p.out[obase + h1 * D + d1] = __float2bfloat16_rn(o[mt][3] * inv1);
          }
        }
        if (p.lse && g4 == 0) {
          const int64_t lb = (int64_t)cur.b * p.num_q_heads + cur.kvh * p.group;
          if (h0 < p.group) p.lse[lb + h0] = lse0;
          if (h1 < p.group) p.lse[lb + h1] = lse1;
        }
      } else {
        const int64_t slot = (int64_t)gw * 2 + piece;
        float* wo = p.ws_o + slot * p.group * D;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          const int d0 = mt * 16 + dlo, d1 = mt * 16 + dhi;
          if (h0 < p.group) {
            wo[h0 * D + d0] = o[mt][0] * inv0;
            wo[h0 * D + d1] = o[mt][2] * inv0;
          }
          if (h1 < p.group) {
            wo[h1 * D + d0] = o[mt][1] * inv1;
            wo[h1 * D + d1] = o[mt][3] * inv1;
          }
        }
        if (g4 == 0) {
          if (h0 < p.group) p.ws_lse[slot * p.group + h0] = lse0;
          if (h1 < p.group) p.ws_lse[slot * p.group + h1] = lse1;
        }
      }
      piece = 1;
    }
    cursor_advance(p, cur);
  }
}

// Merges the partials of segments split between workers, and writes zeros /
// -inf for empty sequences. A CTA has kCombineWarps warps. SPLIT = false: one
// warp per (segment, query head) item, four items per CTA; SPLIT = true: one
// CTA per item, warp w taking pieces w, w + kCombineWarps, ... and the warps'
// results merged through shared memory (for few, long segments, which a
// single warp would merge over many rounds). Each warp keeps a running
// maximum, sum and weighted output (lanes over head_dim) with eight pieces'
// LSEs and partial outputs in flight at a time.
constexpr int kCombineWarps = 4;
template <int D, bool SPLIT>
__global__ void __launch_bounds__(kCombineWarps * 32) decode_combine_kernel(const DecodeParams p) {
  constexpr int V = D / 32;  // floats per lane
  constexpr int kBatch = 8;  // pieces in flight per warp
  constexpr int kStride = SPLIT ? kCombineWarps : 1;
  static_assert(D <= kCombineWarps * 32, "one thread per output element");
  __shared__ float sm_m[kCombineWarps], sm_s[kCombineWarps];
  __shared__ float sm_acc[SPLIT ? kCombineWarps : 1][D];
  // launched as a programmatic dependent of the main kernel: wait until its
  // grid has completed and its partials, prefix and outputs are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t item = SPLIT ? (int64_t)blockIdx.x : (int64_t)blockIdx.x * kCombineWarps + warp;
  const int H = p.num_kv_heads;
  if (item >= (int64_t)p.batch * H * p.group) return;
  const int h = (int)(item % p.group);
  const int64_t seg = item / p.group;
  const int b = (int)(seg / H);
  const int kvh = (int)(seg % H);
  const int n = p.ws_prefix[b + 1] - p.ws_prefix[b];
  const int64_t orow = ((int64_t)b * p.num_q_heads + kvh * p.group + h);
  if (n == 0) {
    if (SPLIT ? threadIdx.x < D : lane < D / V) {
      const int t = SPLIT ? threadIdx.x : lane;
      for (int i = 0; i < (SPLIT ? 1 : V); ++i)
        p.out[orow * D + (SPLIT ? t : t * V + i)] = __float2bfloat16_rn(0.f);
    }
    if (p.lse && (SPLIT ? threadIdx.x == 0 : lane == 0)) p.lse[orow] = -INFINITY;
    return;
  }
  const int64_t T = (int64_t)p.ws_prefix[p.batch] * H;
  const int W = workers_for(T, p.workers);
  const int64_t s0 = (int64_t)p.ws_prefix[b] * H + (int64_t)kvh * n;
  const int64_t s1 = s0 + n;
  auto owner = [&](int64_t x) { return (int)(((x + 1) * W - 1) / T); };
  const int wf = owner(s0), wl = owner(s1 - 1);
  if (wf == wl) return;  // written whole by one worker
  // slot of worker w's piece of this segment, or -1 if w has no tiles
  auto slot_of = [&](int w) -> int64_t {
    const int64_t st = (int64_t)w * T / W, en = (int64_t)(w + 1) * T / W;
    if (st == en) return -1;
    return (int64_t)w * 2 + ((w == wf && st < s0) ? 1 : 0);
  };
  float m = -INFINITY, sum = 0.f, acc[V];
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.f;
  for (int w0 = wf + (SPLIT ? warp : 0); w0 <= wl; w0 += kStride * kBatch) {
    float x[kBatch], v[kBatch][V];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int w = w0 + u * kStride;
      const int64_t sl = w <= wl ? slot_of(w) : -1;
      x[u] = sl >= 0 ? __ldcg(p.ws_lse + sl * p.group + h) : -INFINITY;
      const float* src = p.ws_o + ((sl >= 0 ? sl : 0) * p.group + h) * D + lane * V;
      if constexpr (V == 4) {
        const float4 y = sl >= 0 ? __ldcg(reinterpret_cast<const float4*>(src))
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
        v[u][0] = y.x;
        v[u][1] = y.y;
        v[u][2] = y.z;
        v[u][3] = y.w;
      } else {
#pragma unroll
        for (int i = 0; i < V; ++i) v[u][i] = sl >= 0 ? __ldcg(src + i) : 0.f;
      }
    }
    float nm = m;
#pragma unroll
    for (int u = 0; u < kBatch; ++u) nm = fmaxf(nm, x[u]);
    if (nm == -INFINITY) continue;
    const float c = m == -INFINITY ? 0.f : __expf(m - nm);
    sum *= c;
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] *= c;
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const float e = x[u] == -INFINITY ? 0.f : __expf(x[u] - nm);
      sum += e;
#pragma unroll
      for (int i = 0; i < V; ++i) acc[i] += e * v[u][i];
    }
    m = nm;
  }
  if constexpr (!SPLIT) {
    const float inv = sum > 0.f ? 1.f / sum : 0.f;
#pragma unroll
    for (int i = 0; i < V; ++i) p.out[orow * D + lane * V + i] = __float2bfloat16_rn(acc[i] * inv);
    if (p.lse && lane == 0) p.lse[orow] = sum > 0.f ? m + logf(sum) : -INFINITY;
  } else {
    if (lane == 0) {
      sm_m[warp] = m;
      sm_s[warp] = sum;
    }
#pragma unroll
    for (int i = 0; i < V; ++i) sm_acc[warp][lane * V + i] = acc[i];
    __syncthreads();
    if (threadIdx.x < D) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kCombineWarps; ++w) M = fmaxf(M, sm_m[w]);
      float S = 0.f, A = 0.f;
#pragma unroll
      for (int w = 0; w < kCombineWarps; ++w) {
        if (sm_m[w] == -INFINITY) continue;
        const float c = __expf(sm_m[w] - M);
        S += sm_s[w] * c;
        A += sm_acc[w][threadIdx.x] * c;
      }
      p.out[orow * D + threadIdx.x] = __float2bfloat16_rn(S > 0.f ? A / S : 0.f);
      if (p.lse && threadIdx.x == 0) p.lse[orow] = S > 0.f ? M + logf(S) : -INFINITY;
    }
  }
}

// ---------------------------------------------------------------- fp32 path

// One CTA per (sequence, query head); keys in chunks of blockDim.x, one key
// per thread for the dot product, one output element per thread for P.V.
__global__ void __launch_bounds__(128) decode_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ kc, const float* __restrict__ vc,
    const int32_t* __restrict__ tables, int32_t max_blocks, const int32_t* __restrict__ seq_lens,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t bs_shift,
    int32_t num_blocks, float scale, pkv_mask_mod mask, float* __restrict__ out,
    float* __restrict__ lse, int32_t* dbg) {
  constexpr int NT = 128;
  __shared__ float qs[256];
  __shared__ float ps[NT];
  __shared__ float red[NT / 32];
  const int b = blockIdx.x / num_q_heads;
  const int h = blockIdx.x % num_q_heads;
  const int kvh = h / (num_q_heads / num_kv_heads);
  const int tid = threadIdx.x;
  int L = seq_lens[b];
  if (L < 0) L = 0;
  if (L > (max_blocks << bs_shift)) {
    flag_error(dbg, PKV_DBG_LENGTH);
    L = max_blocks << bs_shift;
  }
  int lo, hi;
  hi = L;
  lo = L > 0 ? mask_lo(mask, b, h, L - 1) : 0;
  for (int d = tid; d < head_dim; d += NT) qs[d] = q[((int64_t)b * num_q_heads + h) * head_dim + d];
  __syncthreads();
  float m = -INFINITY, l = 0.f;
  float acc[2] = {0.f, 0.f};  // head_dim <= 256
  const int bs_mask = (1 << bs_shift) - 1;
  for (int base = lo; base < hi; base += NT) {
    const int j = base + tid;
    float s = -INFINITY;
    if (j < hi) {
      int blk = tables[(int64_t)b * max_blocks + (j >> bs_shift)];
      if (blk < 0 || blk >= num_blocks) {
        flag_error(dbg, PKV_DBG_BLOCK_ID);
      } else {
        const float* kr = kc + ((((int64_t)blk * num_kv_heads + kvh) << bs_shift) + (j & bs_mask)) *
                                   head_dim;
        float dot = 0.f;
        for (int d = 0; d < head_dim; ++d) dot = fmaf(qs[d], kr[d], dot);
        s = dot * scale;
      }
    }
    // chunk max
    float cm = s;
    for (int off = 16; off; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
    if ((tid & 31) == 0) red[tid >> 5] = cm;
    __syncthreads();
    cm = red[0];
    for (int i = 1; i < NT / 32; ++i) cm = fmaxf(cm, red[i]);
    __syncthreads();
    const float mn = fmaxf(m, cm);
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - mn);
    const float pj = (s == -INFINITY) ? 0.f : expf(s - mn);
    ps[tid] = pj;
    float cs = pj;
    for (int off = 16; off; off >>= 1) cs += __shfl_xor_sync(0xffffffffu, cs, off);
    if ((tid & 31) == 0) red[tid >> 5] = cs;
    __syncthreads();
    cs = 0.f;
    for (int i = 0; i < NT / 32; ++i) cs += red[i];
    l = l * alpha + cs;
    m = mn;
    const int nk = min(NT, hi - base);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int d = tid + r * NT;
      if (d < head_dim) {
        float a = acc[r] * alpha;
        for (int i = 0; i < nk; ++i) {
          const int jj = base + i;
          const int blk = tables[(int64_t)b * max_blocks + (jj >> bs_shift)];
          if (blk < 0 || blk >= num_blocks) continue;
          const float* vr =
              vc + ((((int64_t)blk * num_kv_heads + kvh) << bs_shift) + (jj & bs_mask)) * head_dim;
          a = fmaf(ps[i], vr[d], a);
        }
        acc[r] = a;
      }
    }
    __syncthreads();
  }
  const float inv = (l > 0.f) ? 1.f / l : 0.f;
  for (int r = 0; r < 2; ++r) {
    const int d = tid + r * NT;
    if (d < head_dim) out[((int64_t)b * num_q_heads + h) * head_dim + d] = acc[r] * inv;
  }
  if (lse && tid == 0) lse[(int64_t)b * num_q_heads + h] = (l > 0.f) ? m + logf(l) : -INFINITY;
}

// ---------------------------------------------------------------- host side

namespace {

template <int D, int NSTAGE, int WPC, bool PH, bool KV8 = false, bool APPEND = false>
int launch_bf16_impl(const DecodeArgs& a) {
  using Cf = Cfg<D, KV8>;
  const int sms = device_sm_count();
  const int workers = sms * WPC;
  const int g = a.num_q_heads / a.cache.num_kv_heads;
  const size_t smem =
      (size_t)WPC * NSTAGE * (Cf::kStageBytes + Cf::kScaleBytes) + WPC * NSTAGE * 8 + 1024;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(decode_bf16_kernel<D, NSTAGE, WPC, PH, KV8, APPEND>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return check_launch("paged_attention_decode: smem attribute");
    attr_set[dev] = true;
  }
  const int box_rows = a.cache.block_size >= kTile ? kTile : a.cache.block_size;
  const int64_t rows = (int64_t)a.cache.num_blocks * a.cache.num_kv_heads * a.cache.block_size;
  alignas(64) CUtensorMap kmap, vmap;
  const bool maps_ok =
      KV8 ? (make_pool_tensor_map_u8(&kmap, a.k_cache, rows, D, box_rows) &&
             make_pool_tensor_map_u8(&vmap, a.v_cache, rows, D, box_rows))
          : (make_pool_tensor_map(&kmap, a.k_cache, rows, D, box_rows) &&
             make_pool_tensor_map(&vmap, a.v_cache, rows, D, box_rows));
  if (!maps_ok) return fail(PKV_ERR_CUDA, "paged_attention_decode: tensor map encoding failed");

  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.tables = a.tables;
  p.max_blocks = a.max_blocks;
  p.seq_lens = a.seq_lens;
  p.batch = a.batch;
  p.num_kv_heads = a.cache.num_kv_heads;
  p.group = g;
  p.num_q_heads = a.num_q_heads;
  p.bs_shift = log2_int(a.cache.block_size);
  p.num_blocks = a.cache.num_blocks;
  p.scale_log2 = a.scale * kLog2e;
  p.mask = a.mask;
  p.k_scale = a.k_scale;
  p.v_scale = a.v_scale;
  p.k_new = static_cast<const __nv_bfloat16*>(a.k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(a.v_new);
  p.k_pool = static_cast<__nv_bfloat16*>(const_cast<void*>(a.k_cache));
  p.v_pool = static_cast<__nv_bfloat16*>(const_cast<void*>(a.v_cache));
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  const size_t o_bytes = (size_t)2 * workers * g * D * 4;
  const size_t l_bytes = ((size_t)2 * workers * g * 4 + 255) & ~size_t(255);
  p.ws_o = reinterpret_cast<float*>(ws);
  p.ws_lse = reinterpret_cast<float*>(ws + o_bytes);
  p.ws_prefix = reinterpret_cast<int32_t*>(ws + o_bytes + l_bytes);
  p.workers = workers;
  p.dbg = a.dbg;

  decode_bf16_kernel<D, NSTAGE, WPC, PH, KV8, APPEND><<<sms, WPC * 32, smem, a.stream>>>(kmap, vmap,
                                                                                         p);
  if (int st = check_launch("paged_attention_decode")) return st;
  const int64_t items = (int64_t)a.batch * a.cache.num_kv_heads * g;
  // segments are split into workers / segments pieces on average: below
  // eight segments per worker's worth, one warp merges an item in one round
  const bool split = (int64_t)a.batch * a.cache.num_kv_heads * 8 < workers;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(split ? items : (items + kCombineWarps - 1) / kCombineWarps));
  cfg.blockDim = dim3(kCombineWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (split)
    cudaLaunchKernelEx(&cfg, decode_combine_kernel<D, true>, p);
  else
    cudaLaunchKernelEx(&cfg, decode_combine_kernel<D, false>, p);
  return check_launch("paged_attention_decode: combine");
}

// Warps per CTA (one CTA per SM) and ring depth per warp, the fastest
// measured on B200: 12 warps with 2-stage rings for bf16 head_dim 128 (192 KB
// of ring per CTA; 4, 6 and 8 warps with deeper rings were slower), 16 warps
// with 3-stage rings for E4M3 pools (2 stages: within noise; 20 warps spill).
template <int D>
int launch_bf16(const DecodeArgs& a) {
  const bool per_head = a.mask.kind == PKV_MASK_SLIDING && a.mask.window_per_head;
  if constexpr (D == 128) {
    // E4M3 pools: 4 KB stages (+ 128 B of row scales) per warp
    if (a.cache.dtype == PKV_FP8_E4M3) {
      if (per_head) return launch_bf16_impl<D, 3, 12, true, true>(a);
      return launch_bf16_impl<D, 3, 16, false, true>(a);
    }
  }
  if (a.k_new) {
    if (per_head) return launch_bf16_impl<D, (D == 128 ? 2 : 4), 12, true, false, true>(a);
    return launch_bf16_impl<D, (D == 128 ? 2 : 4), 12, false, false, true>(a);
  }
  if (per_head) return launch_bf16_impl<D, (D == 128 ? 2 : 4), 12, true>(a);
  return launch_bf16_impl<D, (D == 128 ? 2 : 4), 12, false>(a);
}

}  // namespace

size_t decode_workspace_size(int32_t batch, int32_t num_q_heads, const pkv_cache_desc& c) {
  if (c.dtype == PKV_F32) return 0;
  // the E4M3 decode has a 16-warp variant
  const int workers = device_sm_count() * (c.dtype == PKV_FP8_E4M3 ? 16 : kMaxWarpsPerCta);
  const int g = num_q_heads / c.num_kv_heads;
  const size_t o_bytes = (size_t)2 * workers * g * c.head_dim * 4;
  const size_t l_bytes = ((size_t)2 * workers * g * 4 + 255) & ~size_t(255);
  const size_t p_bytes = ((size_t)(batch + 1) * 4 + 255) & ~size_t(255);
  return o_bytes + l_bytes + p_bytes;
}

int launch_decode(const DecodeArgs& a) {
  const int g = a.num_q_heads / a.cache.num_kv_heads;
  if (a.cache.dtype == PKV_F32) {
    if (a.cache.head_dim > 256)
      return fail(PKV_ERR_UNSUPPORTED, "paged_attention_decode: fp32 head_dim > 256");
    const int64_t grid = (int64_t)a.batch * a.num_q_heads;
    decode_f32_kernel<<<(unsigned)grid, 128, 0, a.stream>>>(
        static_cast<const float*>(a.q), static_cast<const float*>(a.k_cache),
        static_cast<const float*>(a.v_cache), a.tables, a.max_blocks, a.seq_lens, a.num_q_heads,
        a.cache.num_kv_heads, a.cache.head_dim, log2_int(a.cache.block_size), a.cache.num_blocks,
        a.scale, a.mask, static_cast<float*>(a.out),
        a.lse, a.dbg);
    return check_launch("paged_attention_decode (fp32)");
  }
  if (a.cache.dtype == PKV_FP8_E4M3 && (a.cache.head_dim != 128 || !a.k_scale || !a.v_scale))
    return fail(PKV_ERR_UNSUPPORTED,
                "paged_attention_decode: E4M3 pools need head_dim 128 and row scales");
  if (g < 1 || g > 8)
    return fail(PKV_ERR_UNSUPPORTED, "paged_attention_decode: bf16 group size %d not in 1..8", g);
  if (a.cache.block_size < 8)
    return fail(PKV_ERR_UNSUPPORTED, "paged_attention_decode: bf16 needs block_size >= 8");
  if (a.cache.head_dim == 128) return launch_bf16<128>(a);
  if (a.cache.head_dim == 64) return launch_bf16<64>(a);
  return fail(PKV_ERR_UNSUPPORTED, "paged_attention_decode: bf16 head_dim %d (64 or 128)",
              a.cache.head_dim);
}

}  // namespace pkv
