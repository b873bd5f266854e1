// Device-side block allocation for appends, with copy-on-write of shared
// partly filled blocks: a decode step's bookkeeping stays on the GPU (and can
// be captured in a CUDA graph with the append and the attention).
//
// Source: "Ultimate Guide to PagedAttention": a growing request takes a new
// block from the free list when its last block is full and appends it to its
// block table, moving no data (dynamic growth); requests that share a prefix
// point at the same physical blocks with a reference count, and a shared block
// is copied when one of its holders writes to it (memory sharing,
// copy-on-write).
//
// Semantics are those of handling the sequences one after another in batch
// order, popping blocks from the top of a free stack:
//  * sequence b appends num_new[b] tokens at positions seq_lens[b] ..;
//  * if it writes into its partly filled last block and that block is
//    shared (refcount > 1), it first takes a private copy (one pop; the old
//    block's refcount drops by one) -- except the last of the block's holders
//    in batch order when all of them append now, which finds the refcount at 1
//    and writes in place;
//  * every further block it grows into is one pop.
// Pops are handed out in that order, so sequence b's k-th pop is
// free_stack[top - 1 - (pops of sequences before b) - k].
//
// Three launches: (1) every appending sequence that writes into an existing
// block counts itself on that block (atomics on a zeroed scratch: holders and
// the last holder in batch order); (2) one CTA decides the copies, scans the
// pops, checks the pool, updates tables, refcounts, the free-stack top and the
// lengths, writes the new tokens' slots and zeroes the scratch again; (3) the
// block copies.
#include "pkv_common.cuh"
#include "pkv_internal.h"

namespace pkv {

namespace {

constexpr int kMaxReserveBatch = 8192;
constexpr int kThreads = 1024;

struct ReserveParams {
  int32_t* tables;
  int32_t max_blocks;
  int32_t* seq_lens;
  const int32_t* num_new;
  int32_t batch;
  int32_t* free_stack;
  int32_t* free_top;
  int32_t* refcount;
  int32_t* holders;    // scratch [num_blocks]: appending holders of a block this call
  int32_t* last;       // scratch [num_blocks]: last such holder + 1
  int64_t* slots;
  int32_t num_tokens;
  int32_t* pairs;      // [batch, 2] or null
  int32_t num_blocks;
  int32_t bs_shift;
  int32_t* dbg;
};

// Block sequence b writes into (its partly filled last block), or -1.
__device__ __forceinline__ int written_block(const ReserveParams& p, int b, int L, int n) {
  const int bs_mask = (1 << p.bs_shift) - 1;
  if (n <= 0 || (L & bs_mask) == 0) return -1;
  const int j = L >> p.bs_shift;
  if (j >= p.max_blocks) return -2;
  const int blk = p.tables[(int64_t)b * p.max_blocks + j];
  return (blk < 0 || blk >= p.num_blocks) ? -2 : blk;
}

__global__ void __launch_bounds__(256) reserve_count_kernel(const ReserveParams p) {
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < p.batch; b += gridDim.x * blockDim.x) {
    const int blk = written_block(p, b, max(0, p.seq_lens[b]), p.num_new[b]);
    if (blk >= 0) {
      atomicAdd(p.holders + blk, 1);
      atomicMax(p.last + blk, b + 1);
    }
  }
}

// Inclusive block-wide scan of one value per thread (1024 threads).
__device__ __forceinline__ int block_scan(int v, int* warp_sums) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  if (lane == 31) warp_sums[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int s = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_sums[lane] = s;
  }
  __syncthreads();
  const int r = v + (warp > 0 ? warp_sums[warp - 1] : 0);
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kThreads, 1) reserve_apply_kernel(const ReserveParams p) {
  extern __shared__ int sm[];
  int* pop_off = sm;                     // [batch + 1] pops before sequence b
  int* tok_off = pop_off + p.batch + 1;  // [batch + 1] new tokens before sequence b
  int* old_len = tok_off + p.batch + 1;  // [batch] length before the append
  int* cow_src = old_len + p.batch;      // [batch] block copied from, or -1
  __shared__ int warp_sums[32];
  __shared__ int s_tot[2];
  __shared__ int s_bad;
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();
  const int bs = 1 << p.bs_shift;

  // pass 1: copy decisions, pops and new tokens per sequence, exclusive scans
  int run_pop = 0, run_tok = 0;
  for (int base = 0; base < p.batch; base += kThreads) {
    const int b = base + threadIdx.x;
    int need = 0, n = 0;
    if (b < p.batch) {
      const int L = max(0, p.seq_lens[b]);
      n = max(0, p.num_new[b]);
      old_len[b] = L;
      cow_src[b] = -1;
      const int nb0 = (L + bs - 1) >> p.bs_shift, nb1 = (L + n + bs - 1) >> p.bs_shift;
      if (nb1 > p.max_blocks) atomicOr(&s_bad, PKV_DBG_LENGTH);
      need = nb1 - nb0;
      const int blk = written_block(p, b, L, n);
      if (blk == -2) atomicOr(&s_bad, PKV_DBG_BLOCK_ID);
      if (blk >= 0) {
        const int rc = p.refcount[blk], k = p.holders[blk];
        if (k > rc || rc < 1) atomicOr(&s_bad, PKV_DBG_REFCOUNT);
        // all holders appending: the last one in batch order keeps the block
        if (rc > 1 && !(k >= rc && p.last[blk] == b + 1)) {
          cow_src[b] = blk;
          need += 1;
        }
      }
    }
    const int ip = block_scan(need, warp_sums);
    const int it = block_scan(n, warp_sums);
    if (b < p.batch) {
      pop_off[b] = run_pop + ip - need;
      tok_off[b] = run_tok + it - n;
    }
    if (threadIdx.x == kThreads - 1) {
      s_tot[0] = ip;
      s_tot[1] = it;
    }
    __syncthreads();
    run_pop += s_tot[0];
    run_tok += s_tot[1];
    __syncthreads();
  }
  const int top = *p.free_top;
  if (threadIdx.x == 0) {
    pop_off[p.batch] = run_pop;
    tok_off[p.batch] = run_tok;
    if (run_tok != p.num_tokens) atomicOr(&s_bad, PKV_DBG_LENGTH);
    if (top < 0 || top > p.num_blocks || run_pop > top) atomicOr(&s_bad, PKV_DBG_OUT_OF_BLOCKS);
  }
  __syncthreads();
  // the blocks about to be popped must be real block ids; the scratch goes
  // back to zero now (every decision has been taken, no table changed yet)
  if (s_bad == 0)
    for (int i = top - run_pop + (int)threadIdx.x; i < top; i += kThreads) {
      const int blk = p.free_stack[i];
      if (blk < 0 || blk >= p.num_blocks) atomicOr(&s_bad, PKV_DBG_OUT_OF_BLOCKS);
    }
  for (int b = threadIdx.x; b < p.batch; b += kThreads) {
    const int blk = written_block(p, b, old_len[b], max(0, p.num_new[b]));
    if (blk >= 0) {
      p.holders[blk] = 0;
      p.last[blk] = 0;
    }
  }
  __syncthreads();
  const int bad = s_bad;

  // pass 2: tables and refcounts of the popped blocks (nothing changes when
  // anything is wrong)
  for (int b = threadIdx.x; b < p.batch; b += kThreads) {
    int dst = -1;
    if (!bad) {
      const int L = old_len[b];
      const int n = max(0, p.num_new[b]);
      int k = top - 1 - pop_off[b];
      int* row = p.tables + (int64_t)b * p.max_blocks;
      if (cow_src[b] >= 0) {
        dst = p.free_stack[k--];
        row[L >> p.bs_shift] = dst;
        p.refcount[dst] = 1;
      }
      const int nb0 = (L + bs - 1) >> p.bs_shift, nb1 = (L + n + bs - 1) >> p.bs_shift;
      for (int j = nb0; j < nb1; ++j) {
        const int nb = p.free_stack[k--];
        row[j] = nb;
        p.refcount[nb] = 1;
      }
    }
    if (p.pairs) {
      p.pairs[2 * b] = bad ? -1 : cow_src[b];
      p.pairs[2 * b + 1] = dst;
    }
  }
  __syncthreads();
  // copied-from blocks lose a holder (after every decision read its count)
  if (!bad)
    for (int b = threadIdx.x; b < p.batch; b += kThreads)
      if (cow_src[b] >= 0) atomicSub(p.refcount + cow_src[b], 1);
  __syncthreads();
  // slots of the new tokens from the final tables, then the lengths
  for (int t = threadIdx.x; t < p.num_tokens; t += kThreads) {
    int64_t slot = -1;
    if (!bad) {
      int lo = 0, hi = p.batch;  // last b with tok_off[b] <= t
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tok_off[mid] <= t) lo = mid; else hi = mid;
      }
      const int pos = old_len[lo] + (t - tok_off[lo]);
      const int blk = p.tables[(int64_t)lo * p.max_blocks + (pos >> p.bs_shift)];
      slot = ((int64_t)blk << p.bs_shift) + (pos & (bs - 1));
    }
    p.slots[t] = slot;
  }
  __syncthreads();
  if (!bad) {
    for (int b = threadIdx.x; b < p.batch; b += kThreads)
      p.seq_lens[b] = old_len[b] + max(0, p.num_new[b]);
    if (threadIdx.x == 0) *p.free_top = top - run_pop;
  } else if (threadIdx.x == 0) {
    flag_error(p.dbg, bad);
  }
}

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" {

PKV_API size_t paged_kv_reserve_scratch_size(pkv_cache_desc cache) {
  if (cache.num_blocks <= 0) return 0;
  return (size_t)2 * cache.num_blocks * sizeof(int32_t);
}

// The reserve step; k_scale / v_scale are the row scales of E4M3 pools (copied
// with the codes), null for other pools.
static int reserve(const char* fn, void* k_cache, void* v_cache, float* k_scale, float* v_scale,
                   pkv_cache_desc cache, int32_t* block_tables, int32_t max_blocks_per_seq,
                   int32_t* seq_lens, const int32_t* num_new, int32_t batch, int32_t* free_stack,
                   int32_t* free_top, int32_t* refcount, int32_t* scratch,
                   int64_t* slot_mapping, int32_t num_tokens, int32_t* cow_pairs,
                   int32_t* dbg_err, void* stream) {
  clear_last_error();
  if (int st = check_cache(cache, fn)) return st;
  const bool fp8 = cache.dtype == PKV_FP8_E4M3;
  if (fp8 != (k_scale != nullptr))
    return fail(PKV_ERR_UNSUPPORTED, "%s: %s", fn,
                fp8 ? "E4M3 pools take paged_kv_reserve_slots_fp8 (row scales move with blocks)"
                    : "row scales belong to E4M3 pools");
  const int64_t scale_bytes = (int64_t)cache.num_kv_heads * cache.block_size * 4;
  if (fp8 && scale_bytes % 16)
    return fail(PKV_ERR_UNSUPPORTED, "%s: num_kv_heads * block_size must be a multiple of 4", fn);
  if (batch < 0 || num_tokens < 0 || max_blocks_per_seq <= 0)
    return fail(PKV_ERR_INVALID_ARG, "%s: bad batch, num_tokens or max_blocks_per_seq", fn);
  if (batch > kMaxReserveBatch)
    return fail(PKV_ERR_UNSUPPORTED, "%s: batch %d > %d", fn, batch, kMaxReserveBatch);
  if (batch == 0) return PKV_OK;
  if (!k_cache || !v_cache || !block_tables || !seq_lens || !num_new || !free_stack ||
      !free_top || !refcount || !scratch || (num_tokens > 0 && !slot_mapping) || !cow_pairs ||
      (fp8 && !v_scale))
    return fail(PKV_ERR_INVALID_ARG, "%s: null pointer", fn);
  if (!aligned16(k_cache) || !aligned16(v_cache) ||
      (fp8 && (!aligned16(k_scale) || !aligned16(v_scale))))
    return fail(PKV_ERR_INVALID_ARG, "%s: pools must be 16-byte aligned", fn);
  ReserveParams p = {};
  p.tables = block_tables;
  p.max_blocks = max_blocks_per_seq;
  p.seq_lens = seq_lens;
  p.num_new = num_new;
  p.batch = batch;
  p.free_stack = free_stack;
  p.free_top = free_top;
  p.refcount = refcount;
  p.holders = scratch;
  p.last = scratch + cache.num_blocks;
  p.slots = slot_mapping;
  p.num_tokens = num_tokens;
  p.pairs = cow_pairs;
  p.num_blocks = cache.num_blocks;
  p.bs_shift = log2_int(cache.block_size);
  p.dbg = dbg_err;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int grid1 = (batch + 255) / 256;
  reserve_count_kernel<<<grid1, 256, 0, s>>>(p);
  if (int st = check_launch(fn)) return st;
  const size_t smem = ((size_t)4 * batch + 2) * sizeof(int);
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(reserve_apply_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(((size_t)4 * kMaxReserveBatch + 2) * sizeof(int))) !=
        cudaSuccess)
      return check_launch("paged_kv_reserve_slots: smem attribute");
    attr_set[dev] = true;
  }
  reserve_apply_kernel<<<1, kThreads, smem, s>>>(p);
  if (int st = check_launch(fn)) return st;
  if (int st = launch_copy_blocks(k_cache, v_cache, cache, cow_pairs, batch, dbg_err, s, true))
    return st;
  if (!fp8) return PKV_OK;
  return launch_copy_spans(k_scale, v_scale, scale_bytes, cache.num_blocks, cow_pairs, batch,
                           dbg_err, s, true);
}

PKV_API int paged_kv_reserve_slots(void* k_cache, void* v_cache, pkv_cache_desc cache,
                                   int32_t* block_tables, int32_t max_blocks_per_seq,
                                   int32_t* seq_lens, const int32_t* num_new, int32_t batch,
                                   int32_t* free_stack, int32_t* free_top, int32_t* refcount,
                                   int32_t* scratch, int64_t* slot_mapping, int32_t num_tokens,
                                   int32_t* cow_pairs, int32_t* dbg_err, void* stream) {
  return reserve("paged_kv_reserve_slots", k_cache, v_cache, nullptr, nullptr, cache,
                 block_tables, max_blocks_per_seq, seq_lens, num_new, batch, free_stack,
                 free_top, refcount, scratch, slot_mapping, num_tokens, cow_pairs, dbg_err,
                 stream);
}

PKV_API int paged_kv_reserve_slots_fp8(void* k_cache, void* v_cache, float* k_scale,
                                       float* v_scale, pkv_cache_desc cache,
                                       int32_t* block_tables, int32_t max_blocks_per_seq,
                                       int32_t* seq_lens, const int32_t* num_new, int32_t batch,
                                       int32_t* free_stack, int32_t* free_top, int32_t* refcount,
                                       int32_t* scratch, int64_t* slot_mapping,
                                       int32_t num_tokens, int32_t* cow_pairs, int32_t* dbg_err,
                                       void* stream) {
  const char* fn = "paged_kv_reserve_slots_fp8";
  if (cache.dtype != PKV_FP8_E4M3 || !k_scale) {
    clear_last_error();
    return fail(cache.dtype != PKV_FP8_E4M3 ? PKV_ERR_UNSUPPORTED : PKV_ERR_INVALID_ARG,
                "%s: E4M3 pools with their row scales only", fn);
  }
  return reserve(fn, k_cache, v_cache, k_scale, v_scale, cache, block_tables,
                 max_blocks_per_seq, seq_lens, num_new, batch, free_stack, free_top, refcount,
                 scratch, slot_mapping, num_tokens, cow_pairs, dbg_err, stream);
}

}  // extern "C"
