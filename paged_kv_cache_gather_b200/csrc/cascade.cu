// Shared-prefix (cascade) decode: sequences that share a prompt (beams,
// parallel samples) read its KV blocks once per group instead of once each.
//
// Source: "Ultimate Guide to PagedAttention", sections on memory sharing and
// beam search (sequences of one request point their common prefix at the same
// physical blocks, stored once). Splitting each sequence's keys into the
// shared prefix and its own keys is exact: softmax attention over a union of
// key sets is the log-sum-exp merge of the attention over each set, the same
// identity the tiled exact softmax of "FlashAttention" (abstract) rests on.
//
// B200 design (bf16, head_dim 128):
//  * One persistent launch of `grouped_decode_kernel` over a flat list of
//    16-token tiles, as in the paged decode kernel. An item of the list is
//    either a prefix item (one group, a block of up to 16 query rows, or 32
//    when a KV head has more than 16 query heads: every member's query heads
//    of a KV head, row = member * g + head; keys: the group's shared prefix
//    through its first member's block table) or an own-key item
//    (one sequence, its g query heads; keys from its shared length to its
//    end). Each (item, KV head) segment is a run of tiles; warps take equal
//    contiguous ranges of the whole list, so the work is balanced whatever the
//    group sizes and lengths are.
//  * The query rows of a segment are the N side of mma.sync m16n8k16 (two or
//    four n-tiles of 8 rows), so a KV tile, loaded once by TMA into the warp's
//    ring, serves all the segment's rows; a group's row blocks read the same
//    prefix tiles, the later ones from L2. S^T = K Q^T puts tokens on M; P^T is
//    transposed in registers (movmatrix) into the B operand of O^T += V^T P^T.
//    The query tile of a segment is staged in the warp's shared memory
//    (128-byte XOR swizzle) and read with ldmatrix. The path is HBM-bound: a
//    tile of 8 KB carries up to 64 small MMAs.
//  * Results leave the main kernel normalised, in float32: a segment one warp
//    did whole goes to a per-(sequence, head) buffer (one for prefixes, one for
//    own keys); a segment cut between warps leaves pieces in per-warp slots.
//    `grouped_combine_kernel` (a programmatic dependent launch) gives each
//    (sequence, head) one warp that finds the sequence's group, merges the
//    pieces of its prefix segment and of its own-key segment by log-sum-exp,
//    merges the two, and writes bf16 out and the LSE.
#include <algorithm>
#include <climits>
#include <cmath>

#include "pkv_common.cuh"
#include "pkv_internal.h"

namespace pkv {

namespace {

constexpr int kD = 128;
constexpr int kTile = 16;            // tokens per tile
// Rows per segment and warps per CTA (one CTA per SM). The kernel is
// latency-bound: 16-row segments (168 registers) let 10 warps fit where 32-row
// segments (252 registers) allowed 8, 94 us per call on the beams workload
// against 111 us (11 warps: 97 us). Groups of more than 16 query heads per KV
// head need 32-row segments.
constexpr int kSmallRows = 16, kSmallWarps = 10;
constexpr int kLargeRows = 32, kLargeWarps = 8;
constexpr int kStages = 2;           // TMA ring depth per warp
constexpr int kMinTilesPerWorker = 2;
constexpr int kTileBytes = kTile * kD * 2;            // K (or V) bytes of one tile
constexpr int kStageBytes = 2 * kTileBytes;           // K then V
// shared memory of one warp: its TMA ring and its segment's staged query rows
__host__ __device__ constexpr int warp_smem(int rows) { return kStages * kStageBytes + rows * kD * 2; }

struct GroupedParams {
  const __nv_bfloat16* q;      // [batch, Hq, D]
  const int32_t* tables;
  int32_t max_blocks;
  const int32_t* seq_lens;
  const int32_t* group_start;  // [num_groups + 1]
  const int32_t* shared_len;   // [batch]
  int32_t batch;
  int32_t num_groups;
  int32_t seg_rows;            // query rows per segment (16 or 32)
  int32_t row_blocks;          // prefix items per group: ceil(max_members * g / seg_rows)
  int32_t max_members;
  int32_t items;               // num_groups * row_blocks + batch
  int32_t num_kv_heads;
  int32_t group;               // query heads per KV head
  int32_t num_q_heads;
  int32_t bs_shift;
  int32_t num_blocks;
  float scale_log2;
  __nv_bfloat16* out;
  float* lse;
  float* ws_o;                 // [2 * workers, seg_rows, D] pieces of split segments
  float* ws_lse;               // [2 * workers, seg_rows]
  float* whole_o;              // [2, batch * Hq, D]: prefix (0) / own keys (1), whole segments
  float* whole_lse;            // [2, batch * Hq]
  int32_t* ws_prefix;          // [items + 1] tiles per KV head before item i
  int32_t workers;
  int32_t* dbg;
};

// One entry of the work list.
struct Item {
  int lo, hi;    // keys [lo, hi)
  int t0, n;     // first tile (16-token units of position) and number of tiles
  int lead;      // sequence whose block table holds the keys (and first query row)
  int rows;      // query rows of the segment
  int rb;        // row block within the group (prefix items)
  bool prefix;
};

__device__ __forceinline__ int clamp_len(const GroupedParams& p, int L) {
  const int cap = p.max_blocks << p.bs_shift;
  if (L > cap) {
    flag_error(p.dbg, PKV_DBG_LENGTH);
    L = cap;
  }
  return max(L, 0);
}

template <int TILE>
__device__ __forceinline__ Item item_of(const GroupedParams& p, int i) {
  Item it;
  const int np = p.num_groups * p.row_blocks;
  if (i < np) {
    const int gi = i / p.row_blocks;
    it.rb = i - gi * p.row_blocks;
    it.prefix = true;
    int b0 = __ldg(p.group_start + gi), b1 = __ldg(p.group_start + gi + 1);
    b0 = min(max(b0, 0), p.batch);
    b1 = min(max(b1, b0), min(p.batch, b0 + p.max_members));
    it.lead = b0;
    it.rows = min(p.seg_rows, (b1 - b0) * p.group - it.rb * p.seg_rows);
    it.lo = 0;
    it.hi = it.rows > 0 ? clamp_len(p, __ldg(p.shared_len + b0)) : 0;
  } else {
    const int b = i - np;
    it.rb = 0;
    it.prefix = false;
    it.lead = b;
    it.rows = p.group;
    it.hi = clamp_len(p, __ldg(p.seq_lens + b));
    it.lo = min(max(__ldg(p.shared_len + b), 0), it.hi);
  }
  it.t0 = it.lo / TILE;
  it.n = it.hi > it.lo ? (it.hi + TILE - 1) / TILE - it.t0 : 0;
  return it;
}

// Tiles per KV head summed over all items (warp-cooperative; every lane gets
// the result); with `prefix`, also the exclusive prefix over items.
template <int TILE>
__device__ __forceinline__ int total_tiles(const GroupedParams& p, int lane, int32_t* prefix) {
  int run = 0;
  for (int base = 0; base < p.items; base += 32) {
    const int i = base + lane;
    const int n = i < p.items ? item_of<TILE>(p, i).n : 0;
    int incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (prefix && i < p.items) prefix[i] = run + incl - n;
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (prefix && lane == 0) prefix[p.items] = run;
  return run;
}

// Item holding global tile x, and the number of tiles (all KV heads) before it.
template <int TILE>
__device__ __forceinline__ void find_item(const GroupedParams& p, int lane, int64_t x, int& i_out,
                                          int64_t& before) {
  const int H = p.num_kv_heads;
  int64_t run = 0;
  for (int base = 0; base < p.items; base += 32) {
    const int i = base + lane;
    const int n = i < p.items ? item_of<TILE>(p, i).n : 0;
    int incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const bool hit = i < p.items && run + (int64_t)incl * H > x;
    const unsigned m = __ballot_sync(0xffffffffu, hit);
    if (m) {
      const int src = __ffs(m) - 1;
      const int excl = __shfl_sync(0xffffffffu, incl - n, src);
      i_out = base + src;
      before = run + (int64_t)excl * H;
      return;
    }
    run += (int64_t)__shfl_sync(0xffffffffu, incl, 31) * H;
  }
  i_out = p.items;
  before = run;
}

__device__ __forceinline__ int workers_for(int64_t total, int launched) {
  int64_t w = total / kMinTilesPerWorker;
  if (w < 1) w = 1;
  return (int)(w < launched ? w : launched);
}

// Cursor over the flat tile list (uniform across the warp).
struct Cursor {
  int i, kvh;
  Item it;
  int64_t seg_first;  // global index of the segment's first tile
  int64_t t;          // global tile index
};

template <int TILE>
__device__ __forceinline__ void cursor_advance(const GroupedParams& p, Cursor& c) {
  ++c.t;
  if (c.t == c.seg_first + c.it.n) {
    c.seg_first += c.it.n;
    if (c.kvh + 1 < p.num_kv_heads) {
      ++c.kvh;
    } else {
      do {
        ++c.i;
        if (c.i >= p.items) return;
        c.it = item_of<TILE>(p, c.i);
      } while (c.it.n == 0);
      c.kvh = 0;
    }
  }
}

// (sequence, query head) of row r of a segment.
__device__ __forceinline__ void row_target(const GroupedParams& p, const Item& it, int kvh, int r,
                                           int& b, int& h) {
  if (it.prefix) {
    const int R = it.rb * p.seg_rows + r;
    b = it.lead + R / p.group;
    h = kvh * p.group + R % p.group;
  } else {
    b = it.lead;
    h = kvh * p.group + r;
  }
}

// Byte offset of 16-byte chunk `c` (0..15) of row `r` in a swizzled tile of
// `rows` rows: two 64-column halves, 128-byte rows, chunk index XOR row % 8.
__device__ __forceinline__ uint32_t swz(int rows, int r, int c) {
  return (uint32_t)((c >> 3) * (rows * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

}  // namespace

// NT: n-tiles of 8 query rows per segment; WARPS: warps per CTA.
template <int NT, int WARPS>
__global__ void __launch_bounds__(WARPS * 32, 1)
    grouped_decode_kernel(const __grid_constant__ CUtensorMap kmap,
                          const __grid_constant__ CUtensorMap vmap, const GroupedParams p) {
  constexpr int kNT = NT;
  constexpr int kRows = NT * 8;
  constexpr int kWarps = WARPS;
  constexpr int kWarpSmem = warp_smem(kRows);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  uint8_t* ring = smem + warp * kWarpSmem;
  uint8_t* qs = ring + kStages * kStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWarps * kWarpSmem) + warp * kStages;

  const int gw = blockIdx.x * kWarps + warp;
  const int64_t T =
      (int64_t)total_tiles<kTile>(p, lane, gw == 0 ? p.ws_prefix : nullptr) * p.num_kv_heads;
  const int W = workers_for(T, p.workers);
  if (gw >= W || T == 0) return;
  const int64_t start = (int64_t)gw * T / W;
  const int64_t end = (int64_t)(gw + 1) * T / W;
  if (start >= end) return;

  if (lane == 0) {
    prefetch_tmap(&kmap);
    prefetch_tmap(&vmap);
    for (int i = 0; i < kStages; ++i) mbar_init(smem_u32(bars + i), 1);
    fence_barrier_init();
  }
  __syncwarp();

  Cursor cur;
  {
    int i;
    int64_t before;
    find_item<kTile>(p, lane, start, i, before);
    cur.i = i;
    cur.it = item_of<kTile>(p, i);
    const int64_t off = start - before;
    cur.kvh = (int)(off / cur.it.n);
    cur.seg_first = before + (int64_t)cur.kvh * cur.it.n;
    cur.t = start;
  }
  Cursor pc = cur;  // producer cursor

  const int bs_mask = (1 << p.bs_shift) - 1;
  const int box_rows = p.bs_shift >= 4 ? kTile : (1 << p.bs_shift);  // 8 or 16
  const int pieces = kTile / box_rows;                                // 1 or 2
  const uint64_t evict_first = policy_evict_first();

  // block ids of the producer's next tile (lane 0), loaded one step ahead
  int pid0 = 0, pid1 = 0;
  auto load_ids = [&](const Cursor& c) {
    if (lane != 0 || c.i >= p.items) return;
    const int tok0 = (c.it.t0 + (int)(c.t - c.seg_first)) * kTile;
    const int j = tok0 >> p.bs_shift;
    const int32_t* row = p.tables + (int64_t)c.it.lead * p.max_blocks;
    pid0 = j < p.max_blocks ? __ldg(row + j) : -1;
    if (pieces == 2) pid1 = (j + 1 < p.max_blocks && tok0 + 8 < c.it.hi) ? __ldg(row + j + 1) : -1;
  };
  auto issue = [&](const Cursor& c, int stage) {
    if (lane != 0) return;
    const int tok0 = (c.it.t0 + (int)(c.t - c.seg_first)) * kTile;
    const uint32_t bar = smem_u32(bars + stage);
    const uint32_t kdst = smem_u32(ring + stage * kStageBytes);
    const uint32_t vdst = kdst + kTileBytes;
    int ids[2] = {pid0, pid1};
    bool need[2];
    uint32_t bytes = 0;
    for (int pi = 0; pi < pieces; ++pi) {
      const int a = tok0 + pi * box_rows;
      need[pi] = a < c.it.hi && a + box_rows > c.it.lo;
      if (need[pi]) {
        if (ids[pi] < 0 || ids[pi] >= p.num_blocks) {
          flag_error(p.dbg, PKV_DBG_BLOCK_ID);
          ids[pi] = 0;
        }
        bytes += 2u * box_rows * kD * 2;
      }
    }
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar, bytes);
    for (int pi = 0; pi < pieces; ++pi) {
      if (!need[pi]) continue;
      const int row = ((ids[pi] * p.num_kv_heads + c.kvh) << p.bs_shift) +
                      ((tok0 + pi * box_rows) & bs_mask);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t o = h * (kTile * 128) + pi * box_rows * 128;
        tma_load_2d_hint(kdst + o, &kmap, h * 64, row, bar, evict_first);
        tma_load_2d_hint(vdst + o, &vmap, h * 64, row, bar, evict_first);
      }
    }
  };

  const int64_t ntiles = end - start;
  load_ids(pc);
  int64_t issued = 0;
  for (; issued < kStages - 1 && issued < ntiles; ++issued) {
    issue(pc, (int)(issued % kStages));
    cursor_advance<kTile>(p, pc);
    if (issued + 1 < ntiles) load_ids(pc);
  }

  // lane roles in the mma fragments
  const int g4 = lane >> 2;
  const int c4 = lane & 3;
  const int mi = lane >> 3, mr = lane & 7;
  const int krow = mr + ((mi & 1) << 3);   // K tile row (token) this lane addresses
  const int kco = mi >> 1;
  const int vtok = mr + ((mi >> 1) << 3);  // V tile row (token) this lane addresses
  const int vco = mi & 1;
  const int qrow = mr + ((mi >> 1) << 3);  // query row (within an n-tile pair) of this lane
  const int qco = mi & 1;

  float o[kNT][kD / 16][4];
  float m0[kNT], m1[kNT], l0[kNT], l1[kNT];
  int piece = 0;
  int64_t piece_start = start;
  int ntv = kNT;  // n-tiles holding rows of the current segment

  for (int64_t k = 0; k < ntiles; ++k) {
    if (issued < ntiles) {
      issue(pc, (int)(issued % kStages));
      cursor_advance<kTile>(p, pc);
      ++issued;
      if (issued < ntiles) load_ids(pc);
    }
    const bool seg_begin = (k == 0) || (cur.t == cur.seg_first);
    if (seg_begin) {
      piece_start = cur.t;
      ntv = (cur.it.rows + 7) >> 3;
      // stage the segment's query rows (zero past its last row), swizzled
      for (int x = lane; x < kRows * 16; x += 32) {
        const int r = x >> 4, c = x & 15;
        int4 v = make_int4(0, 0, 0, 0);
        if (r < cur.it.rows) {
          int b, h;
          row_target(p, cur.it, cur.kvh, r, b, h);
          v = __ldg(reinterpret_cast<const int4*>(p.q + ((int64_t)b * p.num_q_heads + h) * kD) +
                    c);
        }
        *reinterpret_cast<int4*>(qs + swz(kRows, r, c)) = v;
      }
      __syncwarp();
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt) {
#pragma unroll
        for (int mt = 0; mt < kD / 16; ++mt) o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
        m0[nt] = m1[nt] = -INFINITY;
        l0[nt] = l1[nt] = 0.f;
      }
    }

    const int stage = (int)(k % kStages);
    const uint32_t parity = (uint32_t)((k / kStages) & 1);
    uint8_t* kst = ring + stage * kStageBytes;
    const uint32_t kbase = smem_u32(kst);
    const uint32_t vbase = kbase + kTileBytes;
    const uint32_t qbase = smem_u32(qs);
    if (!mbar_wait(smem_u32(bars + stage), parity)) {
      flag_error(p.dbg, PKV_DBG_TIMEOUT);
      return;
    }
    const int tok0 = (cur.it.t0 + (int)(cur.t - cur.seg_first)) * kTile;
    const bool partial = tok0 < cur.it.lo || tok0 + kTile > cur.it.hi;
    if (partial) {
      // rows outside [lo, hi) may hold stale or non-finite data: zero them in V
      for (int x = lane; x < kTile * 16; x += 32) {
        const int r = x >> 4, c = x & 15;
        const int pos = tok0 + r;
        if (pos < cur.it.lo || pos >= cur.it.hi)
          *reinterpret_cast<int4*>(kst + kTileBytes + swz(kTile, r, c)) = make_int4(0, 0, 0, 0);
      }
      fence_proxy_async_smem();
      __syncwarp();
    }

    // S^T (16 tokens x 32 rows) = K (16 x D) * Q^T (D x 32)
    float s[kNT][4];
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk) {
      uint32_t a[4];
      ldmatrix_x4(a, kbase + swz(kTile, krow, 2 * kk + kco));
#pragma unroll
      for (int np = 0; np < kNT / 2; ++np) {
        if (2 * np < ntv) {
          // B fragments of n-tiles 2np, 2np+1: rows (n) x 16 columns (k) of the query tile
          uint32_t bq[4];
          ldmatrix_x4(bq, qbase + swz(kRows, np * 16 + qrow, 2 * kk + qco));
          mma_bf16_16816(s[2 * np], a, bq[0], bq[1]);
          if (2 * np + 1 < ntv) mma_bf16_16816(s[2 * np + 1], a, bq[2], bq[3]);
        }
      }
    }
    // element e of s[nt]: token g4 (+8 for e >= 2), row nt*8 + 2*c4 + (e & 1)
    bool bad0 = false, bad1 = false;
    if (partial) {
      const int p0 = tok0 + g4, p1 = p0 + 8;
      bad0 = p0 < cur.it.lo || p0 >= cur.it.hi;
      bad1 = p1 < cur.it.lo || p1 >= cur.it.hi;
    }
    uint32_t pb0[kNT], pb1[kNT];
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) {
      if (nt < ntv) {
        float x0 = s[nt][0] * p.scale_log2, x1 = s[nt][1] * p.scale_log2;
        float x2 = s[nt][2] * p.scale_log2, x3 = s[nt][3] * p.scale_log2;
        if (bad0) x0 = x1 = -INFINITY;
        if (bad1) x2 = x3 = -INFINITY;
        float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
        }
        // every tile of a segment holds a visible key: the new maxima are finite
        const float n0 = fmaxf(m0[nt], mx0), n1 = fmaxf(m1[nt], mx1);
        const float al0 = fast_exp2(m0[nt] - n0), al1 = fast_exp2(m1[nt] - n1);
        m0[nt] = n0;
        m1[nt] = n1;
        const float p00 = fast_exp2(x0 - n0), p01 = fast_exp2(x1 - n1);
        const float p10 = fast_exp2(x2 - n0), p11 = fast_exp2(x3 - n1);
        l0[nt] = l0[nt] * al0 + p00 + p10;
        l1[nt] = l1[nt] * al1 + p01 + p11;
        if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
          for (int mt = 0; mt < kD / 16; ++mt) {
            o[nt][mt][0] *= al0;
            o[nt][mt][1] *= al1;
            o[nt][mt][2] *= al0;
            o[nt][mt][3] *= al1;
          }
        }
        pb0[nt] = movmatrix_trans(pack_bf16x2(p00, p01));
        pb1[nt] = movmatrix_trans(pack_bf16x2(p10, p11));
      }
    }
    // O^T (D x 32) += V^T (D x 16 tokens) * P^T (16 x 32)
#pragma unroll
    for (int mt = 0; mt < kD / 16; ++mt) {
      uint32_t a[4];
      ldmatrix_x4_trans(a, vbase + swz(kTile, vtok, 2 * mt + vco));
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt)
        if (nt < ntv) mma_bf16_16816(o[nt][mt], a, pb0[nt], pb1[nt]);
    }
    __syncwarp();

    const int64_t seg_end = cur.seg_first + cur.it.n;
    const bool piece_end = (k == ntiles - 1) || (cur.t + 1 == seg_end);
    if (piece_end) {
      const bool whole = (piece_start == cur.seg_first) && (cur.t + 1 == seg_end);
      const int64_t slot = (int64_t)gw * 2 + piece;
      const int kind = cur.it.prefix ? 0 : 1;
      const int64_t rows_all = (int64_t)p.batch * p.num_q_heads;
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt) {
        if (nt < ntv) {
          float s0 = l0[nt], s1 = l1[nt];
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) {
            s0 += __shfl_xor_sync(0xffffffffu, s0, off);
            s1 += __shfl_xor_sync(0xffffffffu, s1, off);
          }
          const float inv[2] = {1.f / s0, 1.f / s1};
          const float ls[2] = {m0[nt] * kLn2 + logf(s0), m1[nt] * kLn2 + logf(s1)};
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int r = nt * 8 + 2 * c4 + j;
            if (r >= cur.it.rows) continue;
            float* dst;
            float* dl;
            if (whole) {
              int b, h;
              row_target(p, cur.it, cur.kvh, r, b, h);
              const int64_t orow = kind * rows_all + (int64_t)b * p.num_q_heads + h;
              dst = p.whole_o + orow * kD;
              dl = p.whole_lse + orow;
            } else {
              dst = p.ws_o + (slot * kRows + r) * kD;
              dl = p.ws_lse + slot * kRows + r;
            }
#pragma unroll
            for (int mt = 0; mt < kD / 16; ++mt) {
              dst[mt * 16 + g4] = o[nt][mt][j] * inv[j];
              dst[mt * 16 + g4 + 8] = o[nt][mt][2 + j] * inv[j];
            }
            if (g4 == 0) *dl = ls[j];
          }
        }
      }
      piece = 1;  // the worker's later piece, if split, is its last: slot 1
    }
    cursor_advance<kTile>(p, cur);
  }
}

namespace {

// Group of sequence b: the last gi with group_start[gi] <= b, by a 32-way
// search across the warp (every lane gets the answer; -1 if b precedes all).
__device__ __forceinline__ int find_group(const GroupedParams& p, int lane, int b) {
  int lo = 0, hi = p.num_groups;
  while (true) {
    const int step = (hi - lo + 31) / 32;
    const int idx = lo + lane * step;
    const bool le = idx < hi && __ldg(p.group_start + idx) <= b;
    const unsigned m = __ballot_sync(0xffffffffu, le);
    if (!m) return -1;
    lo += (31 - __clz(m)) * step;
    if (step == 1) return lo;
    hi = min(hi, lo + step);
  }
}

// Result of segment (item i, KV head kvh) for its row r: this lane's four
// output columns (normalised) and the LSE (-inf for an empty segment). A
// segment one worker did whole is read from whole_o / whole_lse at
// `whole_row`; a split one merges its workers' pieces by log-sum-exp.
__device__ __forceinline__ float segment_result(const GroupedParams& p, int lane, int i, int kvh,
                                                int r, int64_t whole_row, float (&acc)[4]) {
  acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
  const int H = p.num_kv_heads;
  const int n = p.ws_prefix[i + 1] - p.ws_prefix[i];
  if (n <= 0) return -INFINITY;
  const int64_t T = (int64_t)p.ws_prefix[p.items] * H;
  const int W = workers_for(T, p.workers);
  const int64_t s0 = (int64_t)p.ws_prefix[i] * H + (int64_t)kvh * n;
  const int64_t s1 = s0 + n;
  auto owner = [&](int64_t x) { return (int)(((x + 1) * W - 1) / T); };
  const int wf = owner(s0), wl = owner(s1 - 1);
  if (wf == wl) {
    const float4 v = __ldcg(reinterpret_cast<const float4*>(p.whole_o + whole_row * kD) + lane);
    acc[0] = v.x;
    acc[1] = v.y;
    acc[2] = v.z;
    acc[3] = v.w;
    return __ldcg(p.whole_lse + whole_row);
  }
  // slot of worker w's piece of this segment, or -1 if w has no tiles
  auto slot_of = [&](int w) -> int64_t {
    const int64_t st = (int64_t)w * T / W, en = (int64_t)(w + 1) * T / W;
    if (st == en) return -1;
    return (int64_t)w * 2 + ((w == wf && st < s0) ? 1 : 0);
  };
  // running maximum, sum and weighted output over the pieces, eight pieces'
  // LSEs and partial outputs in flight per round (the loop is latency-bound)
  float m = -INFINITY, sum = 0.f;
  for (int w0 = wf; w0 <= wl; w0 += 8) {
    float x[8];
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int w = w0 + u;
      const int64_t sl = w <= wl ? slot_of(w) : -1;
      x[u] = sl >= 0 ? __ldcg(p.ws_lse + sl * p.seg_rows + r) : -INFINITY;
      v[u] = sl >= 0 ? __ldcg(reinterpret_cast<const float4*>(p.ws_o + (sl * p.seg_rows + r) * kD) +
                              lane)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float nm = m;
#pragma unroll
    for (int u = 0; u < 8; ++u) nm = fmaxf(nm, x[u]);
    if (nm == -INFINITY) continue;
    const float c = m == -INFINITY ? 0.f : __expf(m - nm);
    sum *= c;
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[j] *= c;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float e = x[u] == -INFINITY ? 0.f : __expf(x[u] - nm);
      sum += e;
      acc[0] += e * v[u].x;
      acc[1] += e * v[u].y;
      acc[2] += e * v[u].z;
      acc[3] += e * v[u].w;
    }
    m = nm;
  }
  if (!(sum > 0.f)) {
    acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
    return -INFINITY;
  }
  const float inv = 1.f / sum;
#pragma unroll
  for (int j = 0; j < 4; ++j) acc[j] *= inv;
  return m + logf(sum);
}

}  // namespace

// One warp per (sequence, query head): prefix result and own-key result,
// each merged from its pieces, then merged with each other.
__global__ void __launch_bounds__(128) grouped_combine_kernel(const GroupedParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int64_t rows_all = (int64_t)p.batch * p.num_q_heads;
  if (row >= rows_all) return;
  const int b = (int)(row / p.num_q_heads);
  const int h = (int)(row % p.num_q_heads);
  const int kvh = h / p.group, hh = h % p.group;
  if (row == 0 && lane == 0 &&
      (p.group_start[0] != 0 || p.group_start[p.num_groups] != p.batch))
    flag_error(p.dbg, PKV_DBG_LENGTH);

  // the sequence's group and its row in the group's prefix items
  float op[4], os[4];
  float lp = -INFINITY;
  const int gi = find_group(p, lane, b);
  bool ok = gi >= 0 && gi < p.num_groups;
  int b0 = 0;
  if (ok) {
    b0 = __ldg(p.group_start + gi);
    const int b1 = __ldg(p.group_start + gi + 1);
    const int sl = __ldg(p.shared_len + b);
    ok = b0 >= 0 && b < b1 && b1 - b0 <= p.max_members && sl == __ldg(p.shared_len + b0) &&
         sl >= 0 && sl <= __ldg(p.seq_lens + b);
  }
  if (!ok) {
    if (lane == 0) flag_error(p.dbg, PKV_DBG_LENGTH);
    op[0] = op[1] = op[2] = op[3] = 0.f;
  } else {
    const int R = (b - b0) * p.group + hh;
    lp = segment_result(p, lane, gi * p.row_blocks + R / p.seg_rows, kvh, R % p.seg_rows, row, op);
  }
  const float ls = segment_result(p, lane, p.num_groups * p.row_blocks + b, kvh, hh,
                                  rows_all + row, os);
  const float m = fmaxf(lp, ls);
  float v[4] = {0.f, 0.f, 0.f, 0.f};
  float lse = -INFINITY;
  if (m != -INFINITY) {
    const float wp = lp == -INFINITY ? 0.f : __expf(lp - m);
    const float ws = ls == -INFINITY ? 0.f : __expf(ls - m);
    const float inv = 1.f / (wp + ws);
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = (wp * op[j] + ws * os[j]) * inv;
    lse = m + logf(wp + ws);
  }
  uint2 packed;
  packed.x = pack_bf16x2(v[0], v[1]);
  packed.y = pack_bf16x2(v[2], v[3]);
  reinterpret_cast<uint2*>(p.out + row * kD)[lane] = packed;
  if (p.lse && lane == 0) p.lse[row] = lse;
}

namespace {

// One launch of the main kernel with NT n-tiles of rows per segment and WARPS
// warps per CTA (one CTA per SM).
template <int NT, int WARPS>
int launch_grouped(GroupedParams& p, const CUtensorMap& kmap, const CUtensorMap& vmap, int sms,
                   cudaStream_t s) {
  const size_t smem = (size_t)WARPS * warp_smem(NT * 8) + WARPS * kStages * 8 + 1024;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(grouped_decode_kernel<NT, WARPS>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return check_launch("paged_attention_decode_shared_prefix: smem attribute");
    attr_set[dev] = true;
  }
  p.workers = sms * WARPS;
  grouped_decode_kernel<NT, WARPS><<<sms, WARPS * 32, smem, s>>>(kmap, vmap, p);
  return check_launch("paged_attention_decode_shared_prefix");
}

// Workspace (sized for either segment shape): pieces (2 per worker),
// whole-segment results (prefix and own keys per (sequence, head)), tile
// prefix over items (at most 9 * batch items: groups * row blocks <= 8 * batch
// when max_group_size * g <= 128 and segments hold 16 rows).
struct Layout {
  size_t ws_o, ws_lse, whole_o, whole_lse, prefix, total;
};

Layout layout(int32_t batch, int32_t num_q_heads) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t sms = (size_t)device_sm_count();
  const size_t piece_rows =  // worker slots x rows per slot, the larger of the two shapes
      std::max(sms * kSmallWarps * kSmallRows, sms * kLargeWarps * kLargeRows);
  const size_t rows = (size_t)batch * num_q_heads;
  Layout l;
  l.ws_o = 0;
  l.ws_lse = l.ws_o + up(2 * piece_rows * kD * 4);
  l.whole_o = l.ws_lse + up(2 * piece_rows * 4);
  l.whole_lse = l.whole_o + up(2 * rows * kD * 4);
  l.prefix = l.whole_lse + up(2 * rows * 4);
  l.total = l.prefix + up(((size_t)9 * batch + 1) * 4);
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
  return layout(batch, num_q_heads).total;
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
  if (cache.block_size < 8)
    return fail(PKV_ERR_UNSUPPORTED, "%s: block_size must be >= 8", fn);
  if (mask.kind == PKV_MASK_SLIDING || mask.kind == PKV_MASK_DOCUMENT)
    return fail(PKV_ERR_UNSUPPORTED, "%s: mask must be none, causal or prefix-LM", fn);
  if (batch < 0 || max_blocks_per_seq <= 0)
    return fail(PKV_ERR_INVALID_ARG, "%s: bad batch or max_blocks_per_seq", fn);
  if (num_q_heads <= 0 || num_q_heads % cache.num_kv_heads)
    return fail(PKV_ERR_INVALID_ARG, "%s: num_q_heads %d not a multiple of num_kv_heads %d", fn,
                num_q_heads, cache.num_kv_heads);
  const int g = num_q_heads / cache.num_kv_heads;
  if (g > kLargeRows)
    return fail(PKV_ERR_UNSUPPORTED, "%s: %d query heads per KV head (at most %d)", fn, g,
                kLargeRows);
  if (!(scale == scale)) return fail(PKV_ERR_INVALID_ARG, "%s: scale is NaN", fn);
  if (batch == 0) return PKV_OK;
  if (num_groups <= 0 || num_groups > batch || max_group_size <= 0)
    return fail(PKV_ERR_INVALID_ARG, "%s: need 1 <= num_groups <= batch and max_group_size >= 1",
                fn);
  if (max_group_size > batch) max_group_size = batch;  // no group is larger than the batch
  if ((int64_t)max_group_size * g > 128)
    return fail(PKV_ERR_UNSUPPORTED,
                "%s: max_group_size * (num_q_heads / num_kv_heads) = %lld exceeds 128", fn,
                (long long)max_group_size * g);
  if (!q || !k_cache || !v_cache || !block_tables || !seq_lens || !group_start || !shared_len ||
      !out || !workspace)
    return fail(PKV_ERR_INVALID_ARG, "%s: null pointer", fn);
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      !aligned16(workspace))
    return fail(PKV_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", fn);
  const Layout l = layout(batch, num_q_heads);
  if (workspace_bytes < l.total)
    return fail(PKV_ERR_WORKSPACE_TOO_SMALL, "%s: workspace needs %zu bytes, got %zu", fn, l.total,
                workspace_bytes);

  const int sms = device_sm_count();
  const int box_rows = cache.block_size >= kTile ? kTile : cache.block_size;
  const int64_t pool_rows = (int64_t)cache.num_blocks * cache.num_kv_heads * cache.block_size;
  alignas(64) CUtensorMap kmap, vmap;
  if (!make_pool_tensor_map(&kmap, k_cache, pool_rows, kD, box_rows) ||
      !make_pool_tensor_map(&vmap, v_cache, pool_rows, kD, box_rows))
    return fail(PKV_ERR_CUDA, "%s: tensor map encoding failed", fn);

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  GroupedParams p = {};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.tables = block_tables;
  p.max_blocks = max_blocks_per_seq;
  p.seq_lens = seq_lens;
  p.group_start = group_start;
  p.shared_len = shared_len;
  p.batch = batch;
  p.num_groups = num_groups;
  p.max_members = max_group_size;
  const bool small = g <= kSmallRows;
  p.seg_rows = small ? kSmallRows : kLargeRows;
  p.row_blocks = (max_group_size * g + p.seg_rows - 1) / p.seg_rows;
  p.items = num_groups * p.row_blocks + batch;
  p.num_kv_heads = cache.num_kv_heads;
  p.group = g;
  p.num_q_heads = num_q_heads;
  p.bs_shift = log2_int(cache.block_size);
  p.num_blocks = cache.num_blocks;
  p.scale_log2 = scale * kLog2e;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.ws_o = reinterpret_cast<float*>(ws + l.ws_o);
  p.ws_lse = reinterpret_cast<float*>(ws + l.ws_lse);
  p.whole_o = reinterpret_cast<float*>(ws + l.whole_o);
  p.whole_lse = reinterpret_cast<float*>(ws + l.whole_lse);
  p.ws_prefix = reinterpret_cast<int32_t*>(ws + l.prefix);
  p.dbg = dbg_err;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int st = small ? launch_grouped<kSmallRows / 8, kSmallWarps>(p, kmap, vmap, sms, s)
                       : launch_grouped<kLargeRows / 8, kLargeWarps>(p, kmap, vmap, sms, s);
  if (st) return st;
  const int64_t rows = (int64_t)batch * num_q_heads;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((rows + 3) / 4));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, grouped_combine_kernel, p);
  return check_launch(fn);
}

}  // extern "C"
