// Paged chunked prefill on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// Method: "Paged Attention Meets FlexAttention" (abstract) — attention of new
// query tokens over the sequence's scattered KV blocks, gathered by the
// fused kernel through the block table, with the mask modifier applied in
// the kernel — computed exactly with the tiled online softmax of
// "FlashAttention" (abstract). Keys are the cached context (positions
// 0 .. ctx-1, read through the block table) followed by the new chunk
// (positions ctx .. ctx+q-1, read from k_new / v_new).
//
// B200 design:
//  * Persistent CTAs, one per SM. A unit of work is (sequence, KV head, pair
//    of query heads of that KV head's group, 128-row query tile); the two
//    heads share every K/V tile the CTA loads (GQA). Units are handed out
//    round-robin, longest (last query tiles) first.
//  * Warp roles: warps 0-7 turn head 0's scores into probabilities, warps
//    8-15 head 1's: two threads per query row, one per half of the 128 key
//    columns (warps 0-3: keys 0-63, warps 4-7: keys 64-127), so each head's
//    softmax runs on two warps per SM sub-partition and its exponentials
//    keep the transcendental unit busy. The halves of a row trade their
//    maxima through shared memory once per tile and their row sums once per
//    unit, ordered by a named barrier of the head's 8 warps. Every tile
//    starts with a vote (bar.red.and) on the head's bounded waits, so the 8
//    warps leave together on a timeout and no barrier is left waiting. Warp
//    16 issues TMA loads; warp 17 allocates tensor memory and issues the MMAs.
//  * Tensor memory (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each.
//    S = Q K^T is written by tcgen05.mma (M=128, N=128 keys, K=16 x 8); the
//    softmax warps read S and write P as bf16 into the same S region (keys
//    0-63 in columns 0-31, keys 64-127 in columns 64-95: each half of a row
//    over its own columns), and O += P V reads P straight from tensor memory
//    (A operand in TMEM) with V as an MN-major shared-memory operand.
//  * MMA issue order S0(j), PV1(j-1), S1(j), PV0(j): while one warpgroup
//    turns its S into P the tensor core runs the other head's work.
//  * K and V tiles (128 keys) have separate 2-stage rings, so the next K can
//    land as soon as both heads' S of the current one are done, while V
//    waits for P*V. Context tiles are 8 TMA boxes of 16 rows, one
//    per 16-token piece of a paged block (block id from the table); chunk
//    tiles are one 3-D box of k_new / v_new. All loads use 128-byte
//    swizzle. Rows past the context end are loaded as out-of-bounds boxes,
//    which TMA fills with zeros, so no stale value reaches P*V.
//  * Online softmax in base 2 with a lazy rescale: O and l are rescaled only
//    when a row maximum grows by more than 8 (a factor 256), otherwise the
//    stale maximum is kept (P stays <= 256, exact in fp32/bf16 range). The
//    final normalisation uses the same maximum, so the result is exact.
#include "prefill_common.cuh"
#include "tc_sm100.cuh"

namespace pkv {

namespace {

using namespace pf;

constexpr int kStages = 2;          // K/V ring depth
constexpr int kThreads = 576;       // softmax head 0 (8 warps), head 1 (8), TMA (1), MMA (1)
constexpr int kTmaWarp = 16;
constexpr int kMmaWarp = 17;

struct SmemLayout {
  // offsets from the 1024-aligned base
  static constexpr int kQ0 = 0;
  static constexpr int kQ1 = kTileBytes;
  static constexpr int kKV = 2 * kTileBytes;  // stage s: K at kKV + s*2*tile, V after it
  static constexpr int kBars = kKV + kStages * 2 * kTileBytes;
  static constexpr int kNumBars = 2 + 4 * kStages + 9;
  static constexpr int kTmemSlot = kBars + kNumBars * 8;
  static constexpr int kMaxQt = kTmemSlot + 4;  // int32, then the abort flag
  // one float per (head, half, parity, row): row maxima / sums traded by the halves
  static constexpr int kXchg = (kTmemSlot + 16 + 15) & ~15;
  static constexpr int kQoff = kXchg + 2 * 2 * 2 * kM * 4;  // int32 [batch + 1]
};

// barrier indices
enum : int {
  BAR_Q_FULL = 0,
  BAR_Q_EMPTY = 1,
  BAR_K_FULL = 2,                  // + stage
  BAR_K_EMPTY = 2 + kStages,       // + stage
  BAR_V_FULL = 2 + 2 * kStages,    // + stage
  BAR_V_EMPTY = 2 + 3 * kStages,   // + stage
  BAR_S_FULL = 2 + 4 * kStages,    // + head
  BAR_P_FULL = BAR_S_FULL + 2,     // + head
  BAR_O_FULL = BAR_P_FULL + 2,     // + head
  BAR_O_FREE = BAR_O_FULL + 2,     // + head
  BAR_V_FIXED = BAR_O_FREE + 2,    // a V tile whose rows past the context end were zeroed
};

// Named barriers (0 is __syncthreads): 1 + head for the 8 softmax warps of a head.
constexpr int kHeadBarrier = 1;

__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ Maps maps, const PrefillParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  using L = SmemLayout;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);
  int32_t* qoff = reinterpret_cast<int32_t*>(smem + L::kQoff);
  int32_t* max_qt_s = reinterpret_cast<int32_t*>(smem + L::kMaxQt);
  int* abort_flag = reinterpret_cast<int*>(smem + L::kMaxQt + 4);

  // ---- set-up: barriers, tensor memory, per-sequence query offsets
  if (warp == kTmaWarp) {
    if (lane == 0) {
      mbar_init(bar(BAR_Q_FULL), 1);
      mbar_init(bar(BAR_Q_EMPTY), 1);
      for (int s = 0; s < kStages; ++s) {
        mbar_init(bar(BAR_K_FULL + s), 1);
        mbar_init(bar(BAR_K_EMPTY + s), 1);
        mbar_init(bar(BAR_V_FULL + s), 1);
        mbar_init(bar(BAR_V_EMPTY + s), 1);
      }
      for (int h = 0; h < 2; ++h) {
        mbar_init(bar(BAR_S_FULL + h), 1);
        mbar_init(bar(BAR_P_FULL + h), 256);
        mbar_init(bar(BAR_O_FULL + h), 1);
        mbar_init(bar(BAR_O_FREE + h), 256);
      }
      mbar_init(bar(BAR_V_FIXED), 1);
      *abort_flag = 0;
      fence_barrier_init();
      prefetch_tmap(&maps.q);
      prefetch_tmap(&maps.knew);
      prefetch_tmap(&maps.vnew);
      prefetch_tmap(&maps.kpool);
      prefetch_tmap(&maps.vpool);
    }
    // exclusive prefix of q_lens and the largest number of query tiles
    query_offsets(p, lane, qoff, max_qt_s);
  } else if (warp == kMmaWarp) {
    tc::tmem_alloc(smem_u32(tmem_slot), 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int max_qt = *max_qt_s;
  const int64_t num_units = (int64_t)max_qt * p.batch * p.num_kv_heads * p.pairs;
  const uint32_t q_bytes = (p.two_heads ? 2u : 1u) * kTileBytes;

  if (warp == kTmaWarp) {
    // ================================================================ TMA producer
    const int nbox = kN / p.box_rows;  // paged boxes per context tile (8 or 16)
    const int bs_mask = (1 << p.bs_shift) - 1;
    // block id of this lane's box of tile j (-2: past the context end, zero fill);
    // issued one tile ahead so the load latency hides behind the copies
    auto fetch_id = [&](const Unit& x, int j) -> int {
      bool ctx;
      int idx, kp0;
      tile_of(x, j, ctx, idx, kp0);
      if (!ctx || lane >= nbox) return -2;
      const int pos = kp0 + lane * p.box_rows;
      if (pos >= x.C) return -2;
      return p.tables[(int64_t)x.b * p.max_blocks + (pos >> p.bs_shift)];
    };
    // row of a paged box, or the first out-of-bounds row (TMA fills zeros)
    auto box_row = [&](const Unit& x, int id, int pos) -> int {
      if (id == -2) return p.pool_rows;
      if (id < 0 || id >= p.num_blocks) {
        flag_error(p.dbg, PKV_DBG_BLOCK_ID);
        return p.pool_rows;
      }
      return ((id * p.num_kv_heads + x.kvh) << p.bs_shift) + (pos & bs_mask);
    };
    int unit_k = 0;
    uint32_t cnt = 0;  // tiles issued (K and V rings advance together)
    for (int64_t u = blockIdx.x; u < num_units; u += gridDim.x) {
      const Unit x = unit_of(p, qoff, max_qt, u);
      if (!x.valid) continue;
      const int h0 = x.kvh * p.group + x.hp * (p.two_heads ? 2 : 1);
      const int n = x.n();
      int id_cur = fetch_id(x, 0);
      // query tiles (slot reusable once the previous unit's MMAs are done)
      if (unit_k > 0 && !wait_or_flag(bar(BAR_Q_EMPTY), (unit_k - 1) & 1, p.dbg, abort_flag)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(BAR_Q_FULL), q_bytes);
        const int row0 = x.qoff + x.qt * kM;
        for (int hh = 0; hh < (p.two_heads ? 2 : 1); ++hh)
          for (int half = 0; half < 2; ++half)
            tma_load_3d(smem_u32(smem + (hh ? L::kQ1 : L::kQ0) + half * kHalfBytes), &maps.q,
                        half * 64, h0 + hh, row0, bar(BAR_Q_FULL));
      }
      bool ok = true;
      for (int j = 0; j < n; ++j, ++cnt) {
        const int s = cnt % kStages;
        const uint32_t ph = ((cnt / kStages) - 1) & 1;
        bool ctx;
        int idx, kp0;
        tile_of(x, j, ctx, idx, kp0);
        const int id_next = (j + 1 < n) ? fetch_id(x, j + 1) : -2;
        const uint32_t kdst = smem_u32(smem + L::kKV + s * 2 * kTileBytes);
        const uint32_t vdst = kdst + kTileBytes;
        for (int kv = 0; kv < 2; ++kv) {
          const uint32_t dst = kv ? vdst : kdst;
          const uint32_t fb = bar((kv ? BAR_V_FULL : BAR_K_FULL) + s);
          if (cnt >= (uint32_t)kStages &&
              !wait_or_flag(bar((kv ? BAR_V_EMPTY : BAR_K_EMPTY) + s), ph, p.dbg, abort_flag)) {
            ok = false;
            break;
          }
          if (lane == 0) mbar_arrive_expect_tx(fb, kTileBytes);
          __syncwarp();
          if (!ctx) {
            if (lane == 0) {
              const int row0 = x.qoff + idx * kN;
              for (int half = 0; half < 2; ++half)
                tma_load_3d(dst + half * kHalfBytes, kv ? &maps.vnew : &maps.knew, half * 64,
                            x.kvh, row0, fb);
            }
          } else if (lane < nbox) {
            const int pos = kp0 + lane * p.box_rows;
            const int row = box_row(x, id_cur, pos);
            const uint32_t off = lane * p.box_rows * 128;
            for (int half = 0; half < 2; ++half)
              tma_load_2d(dst + half * kHalfBytes + off, kv ? &maps.vpool : &maps.kpool,
                          half * 64, row, fb);
          }
        }
        if (!ok) break;
        if (needs_fix(x, ctx, kp0, p.box_rows)) {
          // the box holding the context end also holds pool rows past it:
          // zero them in V once the tile has landed, then release the MMA warp
          if (!wait_or_flag(bar(BAR_V_FULL + s), (cnt / kStages) & 1, p.dbg, abort_flag)) break;
          const int r0 = x.C - kp0;
          const int r1 = (r0 / p.box_rows + 1) * p.box_rows;
          uint8_t* vbase = smem + L::kKV + s * 2 * kTileBytes + kTileBytes;
          for (int i = lane; i < (r1 - r0) * 2 * 8; i += 32) {
            const int rr = r0 + i / 16;
            const int half = (i / 8) & 1;
            const int ch = i & 7;
            *reinterpret_cast<int4*>(vbase + half * kHalfBytes + rr * 128 + ch * 16) =
                make_int4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(BAR_V_FIXED));
        }
        id_cur = id_next;
      }
      if (!ok) break;
      ++unit_k;
    }
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA issuer
    const uint32_t idesc_s = tc::idesc_bf16(kM, kN, false, false);
    const uint32_t idesc_o = tc::idesc_bf16(kM, kD, false, true);
    const uint32_t S0 = tmem, S1 = tmem + 128, O0 = tmem + 256, O1 = tmem + 384;
    const uint32_t q0 = smem_u32(smem + L::kQ0), q1 = smem_u32(smem + L::kQ1);
    int unit_k = 0;
    uint32_t cnt = 0, p_cnt0 = 0, p_cnt1 = 0, fix_count = 0;
    // Descriptors are built once; the k-steps only move the start address
    // (16-byte units in the low bits): +2 per 32-byte step inside a 128-byte
    // swizzle row, +1024 per 64-column half (16 KB), +128 per 16 V rows.
    const uint64_t dq0 = tc::smem_desc(q0, 16, 1024, tc::kSwizzle128B);
    const uint64_t dq1 = tc::smem_desc(q1, 16, 1024, tc::kSwizzle128B);
    const uint64_t dk0 = tc::smem_desc(smem_u32(smem + L::kKV), 16, 1024, tc::kSwizzle128B);
    const uint64_t dv0 =
        tc::smem_desc(smem_u32(smem + L::kKV) + kTileBytes, kHalfBytes, 1024, tc::kSwizzle128B);
    constexpr uint64_t kStageStep = (uint64_t)(2 * kTileBytes) >> 4;
    auto issue_s = [&](uint32_t d, uint64_t dq, uint64_t dk) {
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk) {
        const uint64_t off = (uint64_t)((kk >> 2) * (kHalfBytes >> 4) + (kk & 3) * 2);
        tc::mma_ss(d, dq + off, dk + off, idesc_s, kk > 0);
      }
    };
    // P of keys 0-63 sits in columns 0-31 of the head's S region, P of keys
    // 64-127 in columns 64-95 (each softmax half packs its P over its own
    // first 32 columns); a k-step of 16 keys reads 8 columns
    auto issue_pv = [&](uint32_t d, uint32_t p_tmem, uint64_t dv, bool acc) {
#pragma unroll
      for (int kk = 0; kk < kN / 16; ++kk)
        tc::mma_ts(d, p_tmem + kk * 8 + (kk >= 4 ? 32 : 0), dv + (uint64_t)(kk * (2048 >> 4)),
                   idesc_o, acc || kk > 0);
    };
    for (int64_t u = blockIdx.x; u < num_units; u += gridDim.x) {
      const Unit x = unit_of(p, qoff, max_qt, u);
      if (!x.valid) continue;
      const int n = x.n();
      if (!wait_or_flag(bar(BAR_Q_FULL), unit_k & 1, p.dbg, abort_flag)) break;
      tc::fence_after_sync();
      int prev_s = 0;
      bool ok = true;
      for (int j = 0; j < n; ++j, ++cnt) {
        const int s = cnt % kStages;
        const uint32_t ph = (cnt / kStages) & 1;
        const uint64_t dk = dk0 + (uint64_t)s * kStageStep;
        const uint64_t dv = dv0 + (uint64_t)s * kStageStep;
        if (!(ok = wait_or_flag(bar(BAR_K_FULL + s), ph, p.dbg, abort_flag))) break;
        tc::fence_after_sync();
        if (lane == 0) {
          issue_s(S0, dq0, dk);
          tc::commit(bar(BAR_S_FULL + 0));
        }
        __syncwarp();
        if (p.two_heads) {
          if (j > 0) {
            if (!(ok = wait_or_flag(bar(BAR_P_FULL + 1), p_cnt1 & 1, p.dbg, abort_flag))) break;
            ++p_cnt1;
            if (j == 1 && unit_k > 0 &&
                !(ok = wait_or_flag(bar(BAR_O_FREE + 1), (unit_k - 1) & 1, p.dbg, abort_flag)))
              break;
            tc::fence_after_sync();
            if (lane == 0) {
              issue_pv(O1, S1, dv0 + (uint64_t)prev_s * kStageStep, j - 1 > 0);
              tc::commit(bar(BAR_V_EMPTY + prev_s));
            }
            __syncwarp();
          }
          if (lane == 0) {
            issue_s(S1, dq1, dk);
            tc::commit(bar(BAR_S_FULL + 1));
          }
          __syncwarp();
        }
        if (lane == 0) tc::commit(bar(BAR_K_EMPTY + s));  // K of this tile is no longer read
        __syncwarp();
        if (!(ok = wait_or_flag(bar(BAR_V_FULL + s), ph, p.dbg, abort_flag))) break;
        {
          bool ctx_t;
          int idx_t, kp0_t;
          tile_of(x, j, ctx_t, idx_t, kp0_t);
          if (needs_fix(x, ctx_t, kp0_t, p.box_rows)) {
            if (!(ok = wait_or_flag(bar(BAR_V_FIXED), fix_count & 1, p.dbg, abort_flag))) break;
            ++fix_count;
          }
        }
        if (!(ok = wait_or_flag(bar(BAR_P_FULL + 0), p_cnt0 & 1, p.dbg, abort_flag))) break;
        ++p_cnt0;
        if (j == 0 && unit_k > 0 &&
            !(ok = wait_or_flag(bar(BAR_O_FREE + 0), (unit_k - 1) & 1, p.dbg, abort_flag)))
          break;
        tc::fence_after_sync();
        if (lane == 0) {
          issue_pv(O0, S0, dv, j > 0);
          if (!p.two_heads) tc::commit(bar(BAR_V_EMPTY + s));
        }
        __syncwarp();
        prev_s = s;
      }
      if (!ok) break;
      if (p.two_heads) {
        if (!wait_or_flag(bar(BAR_P_FULL + 1), p_cnt1 & 1, p.dbg, abort_flag)) break;
        ++p_cnt1;
        if (n == 1 && unit_k > 0 &&
            !wait_or_flag(bar(BAR_O_FREE + 1), (unit_k - 1) & 1, p.dbg, abort_flag))
          break;
        tc::fence_after_sync();
        if (lane == 0) {
          issue_pv(O1, S1, dv0 + (uint64_t)prev_s * kStageStep, n - 1 > 0);
          tc::commit(bar(BAR_V_EMPTY + prev_s));
        }
        __syncwarp();
      }
      if (lane == 0) {
        tc::commit(bar(BAR_O_FULL + 0));
        tc::commit(bar(BAR_O_FULL + 1));
        tc::commit(bar(BAR_Q_EMPTY));
      }
      __syncwarp();
      ++unit_k;
    }
  } else if (warp < 16) {
    // ================================================================ softmax warpgroups
    const int hsel = warp >> 3;              // which head of the pair
    const int csel = (warp >> 2) & 1;        // which half of the key columns
    const int row = (warp & 3) * 32 + lane;  // query row of the tile = TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t S = tmem + hsel * 128 + csel * 64 + lane_base;       // this half's 64 scores
    const uint32_t Pw = S;  // its 32 words of bf16 P go over its own first 32 columns
    const uint32_t O = tmem + 256 + hsel * 128 + csel * 64 + lane_base; // its 64 output columns
    float* xch = reinterpret_cast<float*>(smem + L::kXchg);
    const int hbar = kHeadBarrier + hsel;
    uint32_t x_cnt = 0;
    // trade one float of this row with the other half of the head (slots
    // alternate, so a slot is rewritten only after the head's next barrier,
    // which the other half reaches after reading it)
    auto exchange = [&](float mine) -> float {
      const uint32_t par = x_cnt & 1;
      xch[((hsel * 2 + csel) * 2 + par) * kM + row] = mine;
      named_sync(hbar, 256);
      ++x_cnt;
      return xch[((hsel * 2 + (csel ^ 1)) * 2 + par) * kM + row];
    };
    int unit_k = 0;
    uint32_t s_cnt = 0;
    for (int64_t u = blockIdx.x; u < num_units; u += gridDim.x) {
      const Unit x = unit_of(p, qoff, max_qt, u);
      if (!x.valid) continue;
      if (hsel == 1 && !p.two_heads) {
        ++unit_k;
        continue;
      }
      const int n = x.n();
      const int i_row = x.qt * kM + row;      // query index within the chunk
      const int qpos = x.C + i_row;
      const int qmin = x.C + x.qt * kM, qmax = qmin + kM - 1;
      // this row's visible keys [row_lo, row_hi); every row of the tile sees
      // [lo_max, hi_min) (warp-uniform: decides which tiles need no mask)
      const int h_own = x.kvh * p.group + x.hp * (p.two_heads ? 2 : 1) + hsel;
      const int n_keys = x.C + x.Q;
      const int row_lo = mask_lo(p.mask, x.b, h_own, qpos);
      const int row_hi = mask_hi(p.mask, x.b, qpos, n_keys);
      const int lo_max = mask_lo(p.mask, x.b, h_own, qmax);
      const int hi_min = mask_hi(p.mask, x.b, qmin, n_keys);
      float m = -INFINITY, l = 0.f;  // l: this half's share of the row sum
      bool ok = true;
      for (int j = 0; j < n; ++j, ++s_cnt) {
        ok = wait_or_flag(bar(BAR_S_FULL + hsel), s_cnt & 1, p.dbg, abort_flag, true);
        if (!named_and(hbar, 256, ok)) { ok = false; break; }  // all 8 warps go on, or none
        tc::fence_after_sync();
        bool ctx;
        int idx, kp0;
        tile_of(x, j, ctx, idx, kp0);
        const int key_end = ctx ? x.C : n_keys;
        const bool full = kp0 + kN <= min(key_end, hi_min) && kp0 >= lo_max;
        // pass 1: this half's 64 scores, masked in tensor memory (masked keys
        // become -inf, so pass 2 needs no mask), and their maximum
        float mx;
        {
          uint32_t r[2][32];
          tc::ld32(S, r[0]);
          tc::ld32(S + 32, r[1]);
          tc::wait_ld();
          if (!full) {
            // the visible keys of a row form one interval of columns [vlo, vhi)
            const int c0 = kp0 + csel * 64;  // key of this half's first column
            const int vhi = min(64, min(key_end, row_hi) - c0);
            const int vlo = max(0, row_lo - c0);
            const uint32_t span = (uint32_t)max(vhi - vlo, 0);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if ((uint32_t)(c * 32 + i - vlo) >= span) r[c][i] = __float_as_uint(-INFINITY);
              tc::st32(S + c * 32, r[c]);
            }
            tc::wait_st();
          }
          float a0 = -INFINITY, a1 = -INFINITY;
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            a0 = fmax3(a0, __uint_as_float(r[0][i]), __uint_as_float(r[0][i + 1]));
            a1 = fmax3(a1, __uint_as_float(r[1][i]), __uint_as_float(r[1][i + 1]));
          }
          mx = fmaxf(a0, a1);
        }
        mx = fmaxf(mx, exchange(mx));         // the row maximum, the same in both halves
        const float mxs = mx * p.scale_log2;  // scale > 0 keeps the order
        // lazy rescale: move the reference maximum only when it grows by > 2^8
        float alpha = 1.f;
        if (mxs > m + kRescaleThreshold || (m == -INFINITY && mxs != -INFINITY)) {
          if (m != -INFINITY) alpha = fast_exp2(m - mxs);
          m = mxs;
        }
        const float mb = (m == -INFINITY) ? 0.f : m;
        // pass 2, 32 columns at a time: P = exp2(s*c - m) (masked keys hold
        // -inf and give 0) with the argument and the row sum on packed float
        // pairs, packed to bf16 pairs (P[2k], P[2k+1] -> word k) and stored
        // over the first 32 of this half's own columns, so neither half
        // writes where the other still reads
        float ls[8];
        {
          const uint64_t c2 = f2(p.scale_log2, p.scale_log2), nm2 = f2(-mb, -mb);
          uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
          uint32_t pw[32];
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t r[32];
            tc::ld32(S + c * 32, r);
            tc::wait_ld();
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const uint64_t xv =
                  ffma2(f2(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1])), c2, nm2);
              float x0, x1;
              f2_split(xv, x0, x1);
              const float e0 = fast_exp2(x0), e1 = fast_exp2(x1);
              acc[k & 3] = fadd2(acc[k & 3], f2(e0, e1));
              pw[c * 16 + k] = pack_bf16x2(e0, e1);
            }
          }
          tc::st32(Pw, pw);
#pragma unroll
          for (int k = 0; k < 4; ++k) f2_split(acc[k], ls[2 * k], ls[2 * k + 1]);
        }
        l = l * alpha + ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
        // tcgen05.ld/st are warp-collective: the whole warp takes this branch
        // when any of its rows moved its maximum (the others scale by 1)
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
          // rescale this half of the row of O; the previous P*V has completed
          // (it was issued before this S) and the next one waits for this
          // thread's arrival
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t o[32];
            tc::ld32(O + c * 32, o);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tc::st32(O + c * 32, o);
          }
        }
        tc::wait_st();
        tc::fence_before_sync();
        mbar_arrive(bar(BAR_P_FULL + hsel));
      }
      if (!ok) break;
      // ---- epilogue: O / l -> bf16 (each half its 64 columns), lse
      ok = wait_or_flag(bar(BAR_O_FULL + hsel), unit_k & 1, p.dbg, abort_flag, true);
      if (!named_and(hbar, 256, ok)) break;
      tc::fence_after_sync();
      const float l_other = exchange(l);
      const float lt = csel == 0 ? l + l_other : l_other + l;  // same order in both halves
      const int h = x.kvh * p.group + x.hp * (p.two_heads ? 2 : 1) + hsel;
      const bool valid_row = i_row < x.Q && x.qoff + i_row < p.total_q;
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      __nv_bfloat16* dst = p.out + ((int64_t)(x.qoff + i_row) * p.num_q_heads + h) * kD + csel * 64;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t o[32];
        tc::ld32(O + c * 32, o);
        tc::wait_ld();
        if (valid_row) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[i + 0]) * inv, __uint_as_float(o[i + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv);
            __stcs(reinterpret_cast<uint4*>(dst + c * 32 + i), v);  // streaming: leave L2 early
          }
        }
      }
      if (csel == 0 && valid_row && p.lse)
        p.lse[(int64_t)(x.qoff + i_row) * p.num_q_heads + h] =
            lt > 0.f ? (m + log2f(lt)) * kLn2 : -INFINITY;
      tc::fence_before_sync();
      mbar_arrive(bar(BAR_O_FREE + hsel));
      ++unit_k;
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box) {
  return make_tensor_map_bf16(m, base, rank, dims, strides_bytes, box);
}

}  // namespace

int launch_prefill(const PrefillArgs& a) {
  const char* fn = "paged_attention_prefill";
  if (a.cache.dtype != PKV_BF16)
    return fail(PKV_ERR_UNSUPPORTED, "%s: only bf16 pools are supported", fn);
  if (a.cache.head_dim != kD)
    return fail(PKV_ERR_UNSUPPORTED, "%s: head_dim %d (128 supported)", fn, a.cache.head_dim);
  if (a.cache.block_size < 8)
    return fail(PKV_ERR_UNSUPPORTED, "%s: block_size must be >= 8", fn);
  if (a.batch > kMaxBatch)
    return fail(PKV_ERR_UNSUPPORTED, "%s: batch %d > %d", fn, a.batch, kMaxBatch);
  const int Hkv = a.cache.num_kv_heads;
  const int g = a.num_q_heads / Hkv;
  PrefillParams p;
  p.tables = a.tables;
  p.max_blocks = a.max_blocks;
  p.ctx_lens = a.ctx_lens;
  p.q_lens = a.q_lens;
  p.batch = a.batch;
  p.total_q = a.total_q;
  p.num_q_heads = a.num_q_heads;
  p.num_kv_heads = Hkv;
  p.group = g;
  p.two_heads = (g % 2 == 0) ? 1 : 0;
  p.pairs = p.two_heads ? g / 2 : g;
  p.bs_shift = log2_int(a.cache.block_size);
  p.box_rows = a.cache.block_size < 16 ? a.cache.block_size : 16;
  p.num_blocks = a.cache.num_blocks;
  const int64_t pool_rows = (int64_t)a.cache.num_blocks * Hkv * a.cache.block_size;
  p.pool_rows = (int32_t)pool_rows;
  const float scale = a.scale > 0.f ? a.scale : 1.f / sqrtf((float)kD);
  p.scale_log2 = scale * kLog2e;
  p.mask = a.mask;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.dbg = a.dbg;

  alignas(64) Maps maps;
  {
    const uint64_t dq[3] = {(uint64_t)kD, (uint64_t)a.num_q_heads, (uint64_t)a.total_q};
    const uint64_t sq[2] = {(uint64_t)kD * 2, (uint64_t)a.num_q_heads * kD * 2};
    const uint64_t dk[3] = {(uint64_t)kD, (uint64_t)Hkv, (uint64_t)a.total_q};
    const uint64_t sk[2] = {(uint64_t)kD * 2, (uint64_t)Hkv * kD * 2};
    const uint32_t box3[3] = {64, 1, (uint32_t)kM};
    const uint64_t dp[2] = {(uint64_t)kD, (uint64_t)pool_rows};
    const uint64_t sp[1] = {(uint64_t)kD * 2};
    const uint32_t boxp[2] = {64, (uint32_t)p.box_rows};
    if (!make_map(&maps.q, a.q, 3, dq, sq, box3) || !make_map(&maps.knew, a.k_new, 3, dk, sk, box3) ||
        !make_map(&maps.vnew, a.v_new, 3, dk, sk, box3) ||
        !make_map(&maps.kpool, a.k_cache, 2, dp, sp, boxp) ||
        !make_map(&maps.vpool, a.v_cache, 2, dp, sp, boxp))
      return fail(PKV_ERR_CUDA, "%s: tensor map encoding failed", fn);
  }
  const size_t smem = SmemLayout::kQoff + (size_t)(a.batch + 1) * 4 + 1024;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    const size_t max_smem = SmemLayout::kQoff + (size_t)(kMaxBatch + 1) * 4 + 1024;
    if (cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)max_smem) != cudaSuccess)
      return check_launch("paged_attention_prefill: smem attribute");
    attr_set[dev] = true;
  }
  const int grid = device_sm_count();
  prefill_kernel<<<grid, kThreads, smem, a.stream>>>(maps, p);
  return check_launch(fn);
}

}  // namespace pkv
