/*
 * pagedkv.h — C ABI of a B200 (sm_100a) paged KV-cache attention library.
 *
 * What it computes. Attention over a key/value cache that is cut into
 * fixed-size blocks of `block_size` tokens (a power of two, 16 by default)
 * scattered over a physical pool, each sequence reaching its blocks through a
 * per-sequence block table ("Ultimate Guide to PagedAttention", sections on
 * KV blocks and on the block table, which maps a sequence's logical positions
 * to physical memory). The attention kernels gather the scattered blocks
 * themselves and apply FlexAttention-style mask modifiers inside the fused
 * kernel ("Paged Attention Meets FlexAttention: Unlocking Long-Context
 * Efficiency in Deployed Inference", abstract). The result is exact softmax
 * attention ("FlashAttention: Fast and Memory-Efficient Exact Attention with
 * IO-Awareness", abstract): tiling changes memory traffic, not the result.
 *
 * Layouts (all row-major, all device pointers unless stated):
 *   k_cache, v_cache  [num_blocks, num_kv_heads, block_size, head_dim]
 *   block_tables      int32 [batch, max_blocks_per_seq]; entry j of row b is
 *                     the physical block holding positions j*bs .. j*bs+bs-1
 *                     of sequence b. Entries past ceil(len/bs) are ignored.
 *   slot              block * block_size + row; a token at position p of
 *                     sequence b has slot table[b][p/bs]*bs + p%bs.
 *   Query head h reads KV head h / (num_q_heads / num_kv_heads).
 *   lse               float32, natural-log log-sum-exp of the scaled, masked
 *                     scores, one per (query token, query head).
 *
 * Ownership. The caller owns every buffer; the library allocates and frees
 * nothing. Every call is asynchronous and ordered on `stream` (a
 * cudaStream_t; NULL means the legacy default stream); none synchronises.
 *
 * Errors. Calls return PKV_OK or a negative status. Arguments are checked on
 * the host before any launch; a rejected call launches nothing.
 * pkv_last_error() gives a message for the last failure on the calling thread.
 * Index errors that can only be seen on the device (a block id outside
 * [0, num_blocks), a slot outside the pool, a length beyond the table) never
 * trap: the kernel skips the access and ORs a PKV_DBG_* bit into *dbg_err when
 * dbg_err is not NULL. Read it after the stream completes.
 */
#ifndef PAGEDKV_H_
#define PAGEDKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PKV_VERSION 1

#if defined(__GNUC__)
#define PKV_API __attribute__((visibility("default")))
#else
#define PKV_API
#endif

/* Status codes. */
#define PKV_OK 0
#define PKV_ERR_INVALID_ARG -1         /* null pointer, bad size, misaligned, ... */
#define PKV_ERR_UNSUPPORTED -2         /* dtype / head_dim / block_size not built */
#define PKV_ERR_CUDA -3                /* a CUDA runtime call or launch failed */
#define PKV_ERR_WORKSPACE_TOO_SMALL -4 /* workspace_bytes below the required size */
#define PKV_ERR_BAD_INDEX -5           /* for wrappers that read dbg_err */

/* Bits ORed into *dbg_err by the kernels. */
#define PKV_DBG_BLOCK_ID 1    /* block table entry outside [0, num_blocks) */
#define PKV_DBG_SLOT 2        /* slot_mapping entry outside the pool */
#define PKV_DBG_LENGTH 4      /* a length needs more table entries than given */
#define PKV_DBG_TIMEOUT 8     /* a bounded wait on a copy gave up */
#define PKV_DBG_QLEN_SUM 16   /* prefill: sum of q_lens differs from total_q */
#define PKV_DBG_OUT_OF_BLOCKS 32  /* reserve: too few free blocks, or a bad free stack */
#define PKV_DBG_REFCOUNT 64   /* reserve: a block held by more sequences than its refcount */

/* PKV_FP8_E4M3: one-byte E4M3 codes (1 sign, 4 exponent bits with bias 7, 3
 * mantissa bits; largest finite value 448) with one float32 scale per stored
 * row -- see paged_kv_append_fp8. */
typedef enum { PKV_F32 = 0, PKV_BF16 = 1, PKV_FP8_E4M3 = 2 } pkv_dtype;

typedef enum {
  PKV_MASK_NONE = 0,      /* every key of the sequence is visible */
  PKV_MASK_CAUSAL = 1,    /* key position <= query position */
  PKV_MASK_SLIDING = 2,   /* causal and query - key < window (window keys incl. self) */
  PKV_MASK_PREFIX_LM = 3, /* causal, plus every key below the sequence's prefix_len */
  PKV_MASK_DOCUMENT = 4   /* causal within documents packed into one sequence */
} pkv_mask_kind;

/* FlexAttention-style mask modifier, as data (a C ABI cannot take a callable).
 * "Paged Attention Meets FlexAttention" (abstract) applies FlexAttention mask
 * modifiers inside the paged kernel; the kinds here are the ones whose
 * visible keys, for a query at position q, form one interval [lo(q), hi(q))
 * with both ends non-decreasing in q, so whole tiles outside it are skipped
 * and only boundary tiles are masked element by element.
 *   window           PKV_MASK_SLIDING: keys q-window+1 .. q are visible;
 *                    window <= 0 means causal only.
 *   window_per_seq   device int32 [batch] or NULL: overrides `window` per
 *                    sequence (same <= 0 rule).
 *   window_per_head  device int32 [num_q_heads] or NULL: overrides both per
 *                    query head (same rule). The decode kernels read the union
 *                    of the heads' ranges and mask each head's own.
 *   prefix_len       PKV_MASK_PREFIX_LM: device int32 [batch]; keys below
 *                    prefix_len[b] are visible to every query of sequence b
 *                    (a bidirectional prefix), the rest causally.
 *   doc_offsets      PKV_MASK_DOCUMENT: device int32 [batch + 1]; sequence b's
 *   doc_starts       document start positions are doc_starts[doc_offsets[b]
 *                    .. doc_offsets[b+1]-1], ascending. A document runs from
 *                    its start to the next start; positions before the first
 *                    start form a document of their own. A query sees the keys
 *                    of its own document up to itself.
 * Pointers a kind does not use are ignored. */
typedef struct {
  int32_t kind;
  int32_t window;
  const int32_t* window_per_seq;
  const int32_t* window_per_head;
  const int32_t* prefix_len;
  const int32_t* doc_offsets;
  const int32_t* doc_starts;
} pkv_mask_mod;

/* Shape of one K (or V) pool. */
typedef struct {
  int32_t num_blocks;
  int32_t block_size;   /* power of two */
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t dtype;        /* pkv_dtype */
} pkv_cache_desc;

/*
 * paged_kv_append — write new tokens' K and V into their slots.
 * Source: "Ultimate Guide to PagedAttention", dynamic growth: a growing
 * request takes new blocks and updates its table; no existing data moves.
 *   k, v          [num_tokens, num_kv_heads, head_dim], cache dtype
 *   slot_mapping  int64 [num_tokens]; slot < 0 skips the token (padding);
 *                 slots must be distinct (otherwise which write lands is
 *                 unspecified). A slot >= num_blocks*block_size is skipped
 *                 and flagged PKV_DBG_SLOT.
 * Every other row of the pools is left bit-identical. The copy is exact.
 * Supported: dtype F32 or BF16, head_dim*elem_size a multiple of 16 bytes,
 * all pointers 16-byte aligned.
 */
PKV_API int paged_kv_append(const void* k, const void* v, const int64_t* slot_mapping, int32_t num_tokens,
                    void* k_cache, void* v_cache, pkv_cache_desc cache, int32_t* dbg_err,
                    void* stream);

/*
 * paged_kv_append_fp8 — write new tokens into E4M3 pools (quantised KV).
 * The pages only gesture at compressing the KV cache, so the format is this
 * library's reading: every stored row (one token's K or V for one KV head) has
 * its own float32 scale s = amax / 448 (IEEE float32 division; 1 for an
 * all-zero row), fixed when the row is written, and a value x is stored as the
 * E4M3 code of x / s (IEEE division, round to nearest even, saturating at
 * +-448); it reads back as code * s. Relative error <= 2^-4 for all but the
 * smallest values of a row; no clipping, since every row sets its own scale.
 *   k, v          [num_tokens, num_kv_heads, 128] BF16
 *   k_cache, v_cache  E4M3 pools [num_blocks, num_kv_heads, block_size, 128] (1 byte each)
 *   k_scale, v_scale  float32 [num_blocks, num_kv_heads, block_size]: row scales
 *   slot_mapping  as for paged_kv_append.
 * Supported: cache.dtype PKV_FP8_E4M3, head_dim 128.
 */
PKV_API int paged_kv_append_fp8(const void* k, const void* v, const int64_t* slot_mapping,
                                int32_t num_tokens, void* k_cache, void* v_cache, float* k_scale,
                                float* v_scale, pkv_cache_desc cache, int32_t* dbg_err,
                                void* stream);

/*
 * paged_kv_gather — resolve block tables into contiguous K and V.
 * Source: "Ultimate Guide to PagedAttention", block table section (logical
 * positions to physical blocks). Used to check indexing bit for bit.
 *   k_out, v_out  [batch, num_kv_heads, out_max_len, head_dim], cache dtype;
 *                 position p < seq_lens[b] holds the stored row exactly,
 *                 positions >= seq_lens[b] are written as zeros. Lengths
 *                 beyond out_max_len are cut at out_max_len.
 */
PKV_API int paged_kv_gather(const void* k_cache, const void* v_cache, pkv_cache_desc cache,
                    const int32_t* block_tables, int32_t max_blocks_per_seq,
                    const int32_t* seq_lens, int32_t batch, int32_t out_max_len, void* k_out,
                    void* v_out, int32_t* dbg_err, void* stream);

/*
 * paged_kv_copy_blocks — copy-on-write of shared blocks.
 * Source: "Ultimate Guide to PagedAttention", memory-sharing section: shared
 * blocks are stored once and copied when one of their holders writes to them.
 *   block_pairs  int32 [num_pairs, 2] device: (src, dst) physical block ids.
 * Every KV head's rows of block src are copied to block dst, in K and in V,
 * exactly. A dst must not appear twice nor be a src of another pair in the
 * same call (the copies run concurrently). Ids outside [0, num_blocks) skip
 * the pair and set PKV_DBG_BLOCK_ID.
 */
PKV_API int paged_kv_copy_blocks(void* k_cache, void* v_cache, pkv_cache_desc cache,
                                 const int32_t* block_pairs, int32_t num_pairs,
                                 int32_t* dbg_err, void* stream);

/*
 * paged_kv_copy_blocks_fp8 — paged_kv_copy_blocks for E4M3 pools: each pair
 * copies block src's codes (K and V) and its row scales (k_scale, v_scale:
 * float32 [num_blocks, num_kv_heads, block_size], 16-byte aligned) to block
 * dst, so a copied row decodes to the same values. Requires
 * num_kv_heads * block_size to be a multiple of 4; same pair rules and error
 * reporting as paged_kv_copy_blocks. Two kernel launches on `stream`.
 */
PKV_API int paged_kv_copy_blocks_fp8(void* k_cache, void* v_cache, float* k_scale,
                                     float* v_scale, pkv_cache_desc cache,
                                     const int32_t* block_pairs, int32_t num_pairs,
                                     int32_t* dbg_err, void* stream);

/*
 * paged_kv_reserve_slots — device-side block allocation for an append step:
 * slots for the new tokens, new blocks from a free stack, copy-on-write of
 * shared partly filled blocks; no host round trip (CUDA-graph capturable).
 * Source: "Ultimate Guide to PagedAttention": dynamic growth (a request whose
 * last block is full takes a free block and appends it to its table) and
 * memory sharing (blocks of a common prefix are held with a reference count
 * and copied when one of their holders writes to them).
 * The result is that of serving the sequences one by one in batch order:
 * sequence b reserves positions seq_lens[b] .. seq_lens[b]+num_new[b]-1; if
 * the first of them falls in its partly filled last block and that block is
 * shared (refcount > 1), the sequence first takes a private copy of it (the
 * old block's refcount drops by one; when every holder of the block appends
 * in the same call, the last holder in batch order keeps the block); each
 * further block it grows into is taken from the free stack. Blocks are taken
 * from the top of the stack in that order.
 *   block_tables   int32 [batch, max_blocks_per_seq], updated in place.
 *   seq_lens       int32 [batch]: lengths before; on success += num_new.
 *   num_new        int32 [batch] >= 0.
 *   free_stack     int32 [num_blocks]: free block ids; the top is
 *   free_top       free_stack[*free_top - 1]; *free_top (int32) is updated.
 *   refcount       int32 [num_blocks]: holders of each block, updated (taken
 *                  blocks get 1).
 *   scratch        int32 [2 * num_blocks] (paged_kv_reserve_scratch_size()
 *                  bytes), zero before the first call; every call leaves it zero.
 *   slot_mapping   out int64 [num_tokens], num_tokens = sum of num_new: the
 *                  new tokens' slots, sequence by sequence (the slot_mapping of
 *                  paged_kv_append).
 *   cow_pairs      out int32 [batch, 2]: (src, dst) of the copy sequence b made,
 *                  (-1, -1) if none. The copies of K and V happen in this call.
 * All arrays are device memory. If the free stack holds too few blocks, a
 * table is too narrow, a block id is outside the pool, a refcount is below
 * the number of holders, or num_tokens differs from the sum, nothing changes,
 * every slot is -1 and a PKV_DBG_* bit is set in dbg_err. batch <= 8192.
 * Three kernel launches on `stream`.
 */
PKV_API size_t paged_kv_reserve_scratch_size(pkv_cache_desc cache);
/*
 * paged_kv_reserve_slots_fp8 — paged_kv_reserve_slots for E4M3 pools: the
 * same bookkeeping, and each copy-on-write also copies the block's row scales
 * (k_scale, v_scale as in paged_kv_copy_blocks_fp8). paged_kv_reserve_slots
 * rejects E4M3 pools. Four kernel launches on `stream`.
 */
PKV_API int paged_kv_reserve_slots_fp8(void* k_cache, void* v_cache, float* k_scale,
                                       float* v_scale, pkv_cache_desc cache,
                                       int32_t* block_tables, int32_t max_blocks_per_seq,
                                       int32_t* seq_lens, const int32_t* num_new, int32_t batch,
                                       int32_t* free_stack, int32_t* free_top, int32_t* refcount,
                                       int32_t* scratch, int64_t* slot_mapping,
                                       int32_t num_tokens, int32_t* cow_pairs, int32_t* dbg_err,
                                       void* stream);
PKV_API int paged_kv_reserve_slots(void* k_cache, void* v_cache, pkv_cache_desc cache,
                                   int32_t* block_tables, int32_t max_blocks_per_seq,
                                   int32_t* seq_lens, const int32_t* num_new, int32_t batch,
                                   int32_t* free_stack, int32_t* free_top, int32_t* refcount,
                                   int32_t* scratch, int64_t* slot_mapping, int32_t num_tokens,
                                   int32_t* cow_pairs, int32_t* dbg_err, void* stream);

/*
 * paged_attention_decode_workspace_size — bytes of scratch the decode call
 * needs on the current device (depends on the device's SM count, the group
 * size num_q_heads/num_kv_heads, head_dim and batch). 0 for float32 pools.
 */
PKV_API size_t paged_attention_decode_workspace_size(int32_t batch, int32_t num_q_heads,
                                             pkv_cache_desc cache);

/*
 * paged_attention_decode — one query token per sequence over its paged
 * context. Source: "Paged Attention Meets FlexAttention" (fused kernel that
 * gathers scattered KV blocks, FlexAttention masks) with the exact softmax
 * of "FlashAttention" (online softmax, tiling). Long contexts are split
 * across workers and merged by log-sum-exp; each KV block is read once per
 * KV head for the whole query-head group.
 *   q          [batch, num_q_heads, head_dim], cache dtype
 *   seq_lens   int32 [batch]: keys 0 .. seq_lens[b]-1 (including the token
 *              just appended); the query sits at position seq_lens[b]-1.
 *   scale      multiplies q.k (e.g. 1/sqrt(head_dim)).
 *   out        [batch, num_q_heads, head_dim], cache dtype (bf16 outputs are
 *              rounded to nearest even from float32).
 *   lse        float32 [batch, num_q_heads] (may be NULL).
 *   workspace  device scratch of at least
 *              paged_attention_decode_workspace_size(...) bytes, 16-byte
 *              aligned; may be NULL when that size is 0. Contents need no
 *              initialisation. Calls that share a workspace must not overlap.
 * A sequence of length 0 gets out = 0 and lse = -inf.
 * Supported: BF16 with head_dim 64 or 128, block_size >= 8, group size
 * num_q_heads/num_kv_heads in 1..8; F32 with head_dim <= 256 (any group).
 */
PKV_API int paged_attention_decode(const void* q, const void* k_cache, const void* v_cache,
                           pkv_cache_desc cache, const int32_t* block_tables,
                           int32_t max_blocks_per_seq, const int32_t* seq_lens, int32_t batch,
                           int32_t num_q_heads, float scale, pkv_mask_mod mask, void* out,
                           float* lse, void* workspace, size_t workspace_bytes,
                           int32_t* dbg_err, void* stream);

/*
 * paged_attention_decode_append — one decode step in one launch: each
 * sequence's new token is appended to the cache and the step's queries attend
 * to the cache including it. Source: "Ultimate Guide to PagedAttention",
 * dynamic growth (a generated token's K/V go into the next position of the
 * sequence's blocks, no existing data moves) followed by the decode of
 * "Paged Attention Meets FlexAttention".
 *   k_new, v_new  [batch, num_kv_heads, head_dim] BF16: the token at position
 *                 seq_lens[b]-1 of sequence b (seq_lens include it, as for
 *                 paged_attention_decode); it is written, for every KV head,
 *                 to block block_tables[b][(seq_lens[b]-1) / block_size], row
 *                 (seq_lens[b]-1) % block_size of both pools (the block must
 *                 already be in the table). Sequences with seq_lens[b] = 0
 *                 append nothing.
 * The pools and every result are bit-identical to paged_kv_append with those
 * slots followed by paged_attention_decode with the same arguments. Other
 * arguments, limits and errors as paged_attention_decode; BF16 pools only.
 */
PKV_API int paged_attention_decode_append(const void* q, const void* k_new, const void* v_new,
                                          void* k_cache, void* v_cache, pkv_cache_desc cache,
                                          const int32_t* block_tables, int32_t max_blocks_per_seq,
                                          const int32_t* seq_lens, int32_t batch,
                                          int32_t num_q_heads, float scale, pkv_mask_mod mask,
                                          void* out, float* lse, void* workspace,
                                          size_t workspace_bytes, int32_t* dbg_err, void* stream);

/*
 * paged_attention_decode_fp8 — paged_attention_decode over E4M3 pools written
 * by paged_kv_append_fp8 (half the bytes of bf16 per token). Same arguments,
 * layouts, results and errors as paged_attention_decode, plus the row scales
 * k_scale, v_scale (float32 [num_blocks, num_kv_heads, block_size], 16-byte
 * aligned). q and out stay BF16; the result is attention over the decoded
 * values code * scale. Codes are decoded exactly to f16 and the products run
 * in f16 with float32 accumulation. Supported: head_dim 128, block_size >= 8,
 * query groups of 1..8 heads, every mask kind; |q| < 65504.
 */
PKV_API int paged_attention_decode_fp8(const void* q, const void* k_cache, const void* v_cache,
                                       const float* k_scale, const float* v_scale,
                                       pkv_cache_desc cache, const int32_t* block_tables,
                                       int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                       int32_t batch, int32_t num_q_heads, float scale,
                                       pkv_mask_mod mask, void* out, float* lse, void* workspace,
                                       size_t workspace_bytes, int32_t* dbg_err, void* stream);

/*
 * paged_attention_prefill — a chunk of new query tokens per sequence over the
 * sequence's paged context followed by the chunk itself.
 * Source: "Paged Attention Meets FlexAttention" (paged, masked attention in
 * one fused kernel), exact softmax as in "FlashAttention".
 *   q            [total_q, num_q_heads, head_dim] BF16, packed by sequence
 *                in batch order (sequence b owns q_lens[b] rows)
 *   k_new, v_new [total_q, num_kv_heads, head_dim] BF16, packed the same way
 *   ctx_lens     int32 [batch]: tokens already in the paged cache, read
 *                through block_tables (positions 0 .. ctx-1)
 *   q_lens       int32 [batch]: new tokens; new token i of sequence b is at
 *                position ctx_lens[b] + i, and its K/V come from k_new/v_new.
 *   scale        multiplies q.k; <= 0 selects 1/sqrt(head_dim).
 *   out          [total_q, num_q_heads, head_dim] BF16; lse float32
 *                [total_q, num_q_heads] (may be NULL).
 * The call does not write the cache: append the chunk with paged_kv_append
 * (before or after) so later steps see it; the result equals attention over
 * the appended cache. Supported: BF16, head_dim 128, block_size >= 8.
 */
PKV_API int paged_attention_prefill(const void* q, const void* k_new, const void* v_new,
                            const void* k_cache, const void* v_cache, pkv_cache_desc cache,
                            const int32_t* block_tables, int32_t max_blocks_per_seq,
                            const int32_t* ctx_lens, const int32_t* q_lens, int32_t batch,
                            int32_t total_q, int32_t num_q_heads, float scale, pkv_mask_mod mask,
                            void* out, float* lse, int32_t* dbg_err, void* stream);

/*
 * paged_attention_decode_shared_prefix_workspace_size — bytes of scratch the
 * shared-prefix decode call needs on the current device (float32 pieces of
 * split segments for every worker, per-(sequence, head) results of the prefix
 * and of the own keys, a tile prefix over the work items). 0 on invalid
 * arguments.
 */
PKV_API size_t paged_attention_decode_shared_prefix_workspace_size(int32_t batch,
                                                                   int32_t num_q_heads,
                                                                   pkv_cache_desc cache);

/*
 * paged_attention_decode_shared_prefix — paged_attention_decode for batches
 * whose sequences come in groups (beams, parallel samples) that share a
 * prompt stored once. Source: "Ultimate Guide to PagedAttention", memory
 * sharing and beam search (sequences of one request map their common
 * prefix to the same physical blocks). Each sequence's attention is split
 * into its group's shared prefix and its own keys and the two parts are
 * merged by log-sum-exp, which is exact ("FlashAttention", exact tiled
 * attention). The prefix is attended once per group and KV head with every
 * member's query heads together, so each shared block is read once per group
 * instead of once per sequence. Two kernel launches on `stream`.
 * Same arguments, layouts, results and errors as paged_attention_decode, plus:
 *   group_start     int32 [num_groups + 1] on the device: group i holds batch
 *                   entries group_start[i] .. group_start[i+1]-1; groups tile
 *                   0 .. batch-1 in order (group_start[0] = 0, last = batch).
 *   num_groups      host int, 1 .. batch.
 *   max_group_size  host int, >= every group's size; max_group_size *
 *                   (num_q_heads / num_kv_heads) must be <= 128.
 *   shared_len      int32 [batch] on the device: keys 0 .. shared_len[b]-1
 *                   of sequence b are its group's shared prefix. All members
 *                   of a group give the same value, 0 <= shared_len[b] <=
 *                   seq_lens[b], and those keys hold the same K/V in every
 *                   member (normally the same physical blocks; the call reads
 *                   them through the first member's block table).
 *   workspace       >= paged_attention_decode_shared_prefix_workspace_size()
 *                   bytes, 16-byte aligned; calls sharing it must not overlap.
 * A group whose shared length is 0 reduces to plain decode for its members.
 * Group descriptions that break these rules are flagged in dbg_err
 * (PKV_DBG_LENGTH); the affected rows then skip the prefix.
 * Supported: BF16, head_dim 128, block_size >= 8, at most 32 query heads per
 * KV head, masks none and causal (a decode query sees its whole context
 * under both).
 */
PKV_API int paged_attention_decode_shared_prefix(
    const void* q, const void* k_cache, const void* v_cache, pkv_cache_desc cache,
    const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
    int32_t batch, int32_t num_q_heads, float scale, pkv_mask_mod mask,
    const int32_t* group_start, int32_t num_groups, int32_t max_group_size,
    const int32_t* shared_len, void* out, float* lse, void* workspace, size_t workspace_bytes,
    int32_t* dbg_err, void* stream);

/*
 * paged_attention_block_mask — the block-sparse table of a mask modifier.
 * Source: "Paged Attention Meets FlexAttention" (abstract): FlexAttention mask
 * modifiers applied inside the paged kernel, which skips blocks no query of
 * a tile can see. The attention calls derive these classes themselves; this
 * call writes them out (for inspection, for planning work, for tests).
 * Sequence b has ctx_lens[b] keys before q_lens[b] queries at positions
 * ctx_lens[b] + i, and ctx_lens[b] + q_lens[b] keys in all (a decode step is
 * ctx = seq_len - 1, q = 1). For query head h, query tile qt (queries
 * qt*q_tile .. qt*q_tile+q_tile-1 of the sequence's q_lens[b]) and key tile kt
 * (keys kt*k_tile .. kt*k_tile+k_tile-1), out[((b*num_q_heads + h)*n_q_tiles
 * + qt)*n_k_tiles + kt] is PKV_BLOCK_SKIP (no pair visible, or the tile lies
 * past the sequence), PKV_BLOCK_PARTIAL or PKV_BLOCK_FULL (every pair visible).
 *   ctx_lens, q_lens  device int32 [batch]; out  device uint8, written in full.
 */
#define PKV_BLOCK_SKIP 0
#define PKV_BLOCK_PARTIAL 1
#define PKV_BLOCK_FULL 2
PKV_API int paged_attention_block_mask(const int32_t* ctx_lens, const int32_t* q_lens,
                                       int32_t batch, int32_t num_q_heads, pkv_mask_mod mask,
                                       int32_t q_tile, int32_t k_tile, int32_t n_q_tiles,
                                       int32_t n_k_tiles, uint8_t* out, void* stream);

/*
 * paged_attention_decode_noalloc — paged_attention_decode without a
 * caller-provided workspace. The pages have no counterpart to this call: it
 * exists for callers that cannot allocate device memory (a runtime whose
 * device memory all belongs to its own pool, a C or embedded host without a
 * device allocator, a loop that cannot afford cudaMalloc's synchronisation).
 * Same arguments, layouts, results and errors as paged_attention_decode,
 * minus workspace/workspace_bytes. The split-KV scratch is a fixed array of
 * PKV_NOALLOC_SCRATCH_BYTES inside the library's device image, held on every
 * GPU that loads the library until the process exits. The first call on a
 * device looks up that array's address (once per device, with the device
 * current); make that first call before any stream capture begins. Every
 * call shares the array: calls that overlap on the GPU race and give wrong
 * results, so order them on one stream. Nothing in the array needs to start
 * at zero. A problem that needs more scratch than the array holds (more than
 * paged_attention_decode_workspace_size reports for the same sizes) returns
 * PKV_ERR_WORKSPACE_TOO_SMALL and launches nothing; batch < 0 returns
 * PKV_ERR_INVALID_ARG, as the regular call does. The call allocates and
 * frees nothing.
 */
#define PKV_NOALLOC_SCRATCH_BYTES (8u << 20)
PKV_API int paged_attention_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                           pkv_cache_desc cache, const int32_t* block_tables,
                                           int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                           int32_t batch, int32_t num_q_heads, float scale,
                                           pkv_mask_mod mask, void* out, float* lse,
                                           int32_t* dbg_err, void* stream);

/*
 * pkv_debug_wait_timeout — diagnostic, not part of the attention API: one warp
 * waits on a shared-memory mbarrier that nothing arrives on, through the
 * library's bounded wait (the one every TMA/MMA wait in the kernels uses). When
 * the wait gives up (after about 4 s) the kernel sets PKV_DBG_TIMEOUT in
 * *dbg_err and returns; the context stays usable. elapsed_ns (device, nullable)
 * receives the globaltimer nanoseconds the wait took. It exists so that the
 * timeout path can be tested without a stuck copy or any GPU fault.
 */
PKV_API int pkv_debug_wait_timeout(int32_t* dbg_err, uint64_t* elapsed_ns, void* stream);

/* Name of a status code (static string). */
PKV_API const char* pkv_status_string(int status);

/* Message of the last failed call on this thread ("" if none). */
PKV_API const char* pkv_last_error(void);

/* Library version (PKV_VERSION). */
PKV_API int pkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H_ */
