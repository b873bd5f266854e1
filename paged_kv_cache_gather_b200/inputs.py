"""Seeded synthetic inputs for paged-attention workloads.

Shared by the tests, the benchmark and the smoke check. This module holds no
attention arithmetic: only shapes, seeds, random values and block-table
layouts. Values are N(0, 1) drawn in float32 from a seeded CPU
``torch.Generator`` and then rounded (round-to-nearest-even) to the storage
dtype; block tables come from a seeded NumPy permutation of the pool.

The workloads follow the ones named for this method (a Llama-style 32/8-head,
head_dim 128 model stands in for the unnamed model of "Paged Attention Meets
FlexAttention"; the block size of 16 tokens is the typical value of "Ultimate
Guide to PagedAttention", KV-block section):

1. tiny fp32 decode: 1 sequence, 4/4 heads, d 64, 128 tokens in 8 blocks
   mapped into a 32-block pool, no mask, plus the append of the last token;
2. batch-1 bf16 decode sweep over 128..4096 tokens, 32/8 heads, d 128,
   4096-block pool, causal;
3. batched ragged bf16 decode: 64 sequences, lengths U[1, 8192], first-fit
   blocks from a shuffled free list of a 40000-block pool, sliding window 4096
   on even sequences, causal on odd ones; each step appends one token per
   sequence;
4. shared-prefix beams: 8 groups x 8 beams, a 4096-token prefix shared by
   block id inside each group, 256 own tokens per beam;
5. chunked prefill: 4 sequences with 30720 cached tokens plus a 2048-token
   chunk, causal across context and chunk, 16384-block pool.
"""

from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

MASK_NONE = 0
MASK_CAUSAL = 1
MASK_SLIDING = 2
MASK_PREFIX_LM = 3
MASK_DOCUMENT = 4

SEED_BASE = 1234


def seed_for(config_id: int) -> int:
    return SEED_BASE + config_id


def randn(shape, gen: torch.Generator, dtype=torch.bfloat16, chunk=1 << 26):
    """N(0,1) float32 draws rounded to ``dtype``; large tensors are drawn in chunks."""
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=dtype)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        out[s:e] = torch.randn(e - s, generator=gen, dtype=torch.float32).to(dtype)
    return out.view(*shape)


@dataclass
class PagedCase:
    """One workload instance; every tensor lives on the CPU."""

    name: str
    dtype: torch.dtype
    num_blocks: int
    block_size: int
    num_kv_heads: int
    num_q_heads: int
    head_dim: int
    k_cache: torch.Tensor            # [NB, Hkv, bs, d]
    v_cache: torch.Tensor
    block_tables: torch.Tensor       # int32 [B, max_blocks]; unused entries are -1
    seq_lens: torch.Tensor           # int32 [B]; decode: includes the appended token
    scale: float
    mask_kind: int = MASK_NONE
    window: int = 0
    window_per_seq: Optional[torch.Tensor] = None   # int32 [B] or None
    q: Optional[torch.Tensor] = None                # decode [B, Hq, d]; prefill [sum Q, Hq, d]
    k_new: Optional[torch.Tensor] = None            # [T, Hkv, d]
    v_new: Optional[torch.Tensor] = None
    slot_mapping: Optional[torch.Tensor] = None     # int64 [T]
    ctx_lens: Optional[torch.Tensor] = None         # prefill only
    q_lens: Optional[torch.Tensor] = None
    extra: dict = field(default_factory=dict)

    @property
    def batch(self):
        return int(self.seq_lens.shape[0])


def _table_tensor(rows, width):
    t = np.full((len(rows), width), -1, dtype=np.int32)
    for b, r in enumerate(rows):
        t[b, :len(r)] = r
    return torch.from_numpy(t)


def decode_slots(block_tables, seq_lens, block_size):
    """Slot of the token at position ``seq_len - 1`` of each sequence (the one appended)."""
    tabs = block_tables.numpy().astype(np.int64)
    lens = seq_lens.numpy().astype(np.int64)
    slots = np.full(len(lens), -1, dtype=np.int64)
    for b, L in enumerate(lens):
        if L > 0:
            p = L - 1
            slots[b] = tabs[b, p // block_size] * block_size + p % block_size
    return torch.from_numpy(slots)


def make_decode_case(name, *, lens, num_q_heads, num_kv_heads, head_dim, block_size,
                     num_blocks, dtype, seed, mask_kind=MASK_CAUSAL, window=0,
                     window_per_seq=None, scale=None, table_width=None, first_fit=True,
                     peaky=False):
    """General decode case: pool filled with N(0,1), tables drawn from a shuffled pool.

    ``first_fit``: sequences take blocks in batch order from the front of one
    seeded permutation of the pool (a shuffled free list). The new token of
    each sequence sits at position ``lens[b] - 1``; k_new/v_new/slot_mapping
    describe its append.
    """
    gen = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    lens = [int(x) for x in lens]
    B = len(lens)
    nblk = [(L + block_size - 1) // block_size for L in lens]
    if sum(nblk) > num_blocks:
        raise ValueError("pool too small for the requested lengths")
    free = rng.permutation(num_blocks)
    rows, pos = [], 0
    for n in nblk:
        rows.append(free[pos:pos + n].tolist())
        pos += n
    width = table_width or max(1, max(nblk))
    tables = _table_tensor(rows, width)
    seq_lens = torch.tensor(lens, dtype=torch.int32)
    k_cache = randn((num_blocks, num_kv_heads, block_size, head_dim), gen, dtype)
    v_cache = randn((num_blocks, num_kv_heads, block_size, head_dim), gen, dtype)
    q = randn((B, num_q_heads, head_dim), gen, dtype)
    k_new = randn((B, num_kv_heads, head_dim), gen, dtype)
    v_new = randn((B, num_kv_heads, head_dim), gen, dtype)
    if scale is None:
        scale = 1.0 / float(np.sqrt(head_dim))
    case = PagedCase(name, dtype, num_blocks, block_size, num_kv_heads, num_q_heads, head_dim,
                     k_cache, v_cache, tables, seq_lens, scale, mask_kind, window,
                     window_per_seq, q, k_new, v_new, decode_slots(tables, seq_lens, block_size))
    case.extra["free_list"] = free
    case.extra["blocks_used"] = pos
    if peaky:
        make_peaky(case, seed + 7)
    return case


def make_peaky(case, seed):
    """Sharpen the softmax so outputs are O(1): q x 8, and per (b, kv head) one
    planted key at a seeded visible position, pointing along the first query
    head of the group with length 6 (stored rounded to the cache dtype)."""
    rng = np.random.default_rng(seed)
    g = case.num_q_heads // case.num_kv_heads
    case.q = (case.q.float() * 8.0).to(case.dtype)
    tabs = case.block_tables.numpy()
    bs = case.block_size
    for b in range(case.batch):
        L = int(case.seq_lens[b])
        if L <= 1:
            continue
        w = 0
        if case.window_per_seq is not None:
            w = int(case.window_per_seq[b])
        elif case.mask_kind == MASK_SLIDING:
            w = case.window
        lo = max(0, L - w) if (case.mask_kind == MASK_SLIDING and w > 0) else 0
        if lo >= L - 1:
            continue
        for kvh in range(case.num_kv_heads):
            p = int(rng.integers(lo, L - 1))  # not the appended token
            qh = case.q[b, kvh * g].float()
            key = 6.0 * qh / qh.norm()
            case.k_cache[int(tabs[b, p // bs]), kvh, p % bs] = key.to(case.dtype)
    case.extra["peaky"] = True


# --------------------------------------------------------------------------- configs


def config1(L=128, num_blocks=32, seed=None):
    """Tiny fp32 decode: 1 seq, 4/4 heads, d 64, bs 16, table = permutation(32)[:ceil(L/16)]."""
    return make_decode_case(f"cfg1_tiny_fp32_L{L}", lens=[L], num_q_heads=4, num_kv_heads=4,
                            head_dim=64, block_size=16, num_blocks=num_blocks,
                            dtype=torch.float32, seed=seed if seed is not None else seed_for(1),
                            mask_kind=MASK_NONE, scale=1.0 / 8.0)


CONFIG2_LENGTHS = (128, 256, 512, 1024, 2048, 4096)


def config2(L, seed=None, peaky=False):
    """Batch-1 bf16 decode, 32/8 heads, d 128, bs 16, 4096-block shuffled pool, causal."""
    return make_decode_case(f"cfg2_single_L{L}", lens=[L], num_q_heads=32, num_kv_heads=8,
                            head_dim=128, block_size=16, num_blocks=4096, dtype=torch.bfloat16,
                            seed=seed if seed is not None else seed_for(2),
                            mask_kind=MASK_CAUSAL, peaky=peaky)


def config3_lengths(batch=64, max_len=8192, seed=None):
    rng = np.random.default_rng(seed if seed is not None else seed_for(3))
    return rng.integers(1, max_len + 1, size=batch).tolist()


def config3(batch=64, max_len=8192, num_blocks=40000, window=4096, growth_steps=16,
            seed=None, peaky=False):
    """Ragged batched bf16 decode; even sequences use a sliding window, odd ones causal.

    Tables have room for ``growth_steps`` more tokens per sequence (the step
    loop appends one token per sequence and allocates a block when a new one
    starts).
    """
    s = seed if seed is not None else seed_for(3)
    lens = config3_lengths(batch, max_len, s)
    wps = torch.tensor([window if b % 2 == 0 else 0 for b in range(batch)], dtype=torch.int32)
    width = (max_len + growth_steps + 15) // 16 + 1
    case = make_decode_case(f"cfg3_ragged_B{batch}", lens=lens, num_q_heads=32, num_kv_heads=8,
                            head_dim=128, block_size=16, num_blocks=num_blocks,
                            dtype=torch.bfloat16, seed=s, mask_kind=MASK_SLIDING,
                            window=window, window_per_seq=wps, table_width=width, peaky=peaky)
    case.extra["free_list_next"] = sum((L + 15) // 16 for L in lens)
    return case


def config4(groups=8, beams=8, prefix=4096, suffix=256, num_blocks=4096, shared=True,
            seed=None, peaky=False):
    """Shared-prefix beams. ``shared=False`` gives every beam its own copy of the
    prefix blocks (same values, distinct block ids, in a pool large enough to
    hold them)."""
    s = seed if seed is not None else seed_for(4)
    gen = torch.Generator().manual_seed(s)
    rng = np.random.default_rng(s)
    bs, Hkv, Hq, d = 16, 8, 32, 128
    npre, nsuf = prefix // bs, suffix // bs
    B = groups * beams
    need_unshared = B * (npre + nsuf)
    pool = num_blocks if shared else max(num_blocks, need_unshared)
    perm = rng.permutation(pool)
    k_cache = randn((pool, Hkv, bs, d), gen)
    v_cache = randn((pool, Hkv, bs, d), gen)
    rows = []
    if shared:
        pos = 0
        for g_ in range(groups):
            pre = perm[pos:pos + npre].tolist()
            pos += npre
            for _ in range(beams):
                rows.append(pre + perm[pos:pos + nsuf].tolist())
                pos += nsuf
    else:
        # same logical content as the shared layout: build the shared one first
        shared_case = config4(groups, beams, prefix, suffix, num_blocks, True, s, peaky=False)
        k_src, v_src = shared_case.k_cache, shared_case.v_cache
        tab_src = shared_case.block_tables.numpy()
        pos = 0
        for b in range(B):
            r = perm[pos:pos + npre + nsuf].tolist()
            pos += npre + nsuf
            for j, dst in enumerate(r):
                k_cache[dst] = k_src[tab_src[b, j]]
                v_cache[dst] = v_src[tab_src[b, j]]
            rows.append(r)
        q = shared_case.q
    L = prefix + suffix
    tables = _table_tensor(rows, npre + nsuf)
    seq_lens = torch.full((B,), L, dtype=torch.int32)
    if shared:
        q = randn((B, Hq, d), gen)
    case = PagedCase(f"cfg4_beams_{'shared' if shared else 'copied'}", torch.bfloat16, pool, bs,
                     Hkv, Hq, d, k_cache, v_cache, tables, seq_lens, 1.0 / float(np.sqrt(d)),
                     MASK_CAUSAL, 0, None, q)
    case.extra["unique_blocks"] = len(set(int(x) for r in rows for x in r))
    case.extra["group_start"] = torch.arange(0, B + 1, beams, dtype=torch.int32)
    case.extra["shared_len"] = torch.full((B,), prefix if shared else 0, dtype=torch.int32)
    case.extra["max_group_size"] = beams
    if peaky:
        make_peaky(case, s + 7)
    return case


def make_shared_prefix_case(name, *, group_sizes, prefix_lens, suffix_lens, num_q_heads=32,
                            num_kv_heads=8, head_dim=128, block_size=16, spare_blocks=64,
                            seed, mask_kind=MASK_CAUSAL, peaky=False):
    """Groups of decode sequences that share a prefix, laid out as a fork leaves them.

    Group ``i`` has ``group_sizes[i]`` members and a prefix of
    ``prefix_lens[i]`` tokens; member ``b`` then has ``suffix_lens[b]`` tokens
    of its own. The prefix's full blocks are one set of block ids in every
    member's table. When the prefix ends inside a block, every member holds its
    own copy of that block (as after a copy-on-write): the prefix rows are the
    first member's values, the rows after them the member's own. Tables come
    from one seeded permutation of the pool; the query of each sequence sits at
    its last position. ``extra`` gets ``group_start`` (int32 [G+1]),
    ``shared_len`` (int32 [B]), ``max_group_size`` and ``unique_blocks``.
    """
    gen = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    bs = block_size
    group_sizes = [int(n) for n in group_sizes]
    B = sum(group_sizes)
    if len(prefix_lens) != len(group_sizes) or len(suffix_lens) != B:
        raise ValueError("prefix_lens needs one entry per group, suffix_lens one per sequence")
    need, b = 0, 0
    for gi, n in enumerate(group_sizes):
        need += prefix_lens[gi] // bs
        for _ in range(n):
            L = prefix_lens[gi] + suffix_lens[b]
            need += (L + bs - 1) // bs - prefix_lens[gi] // bs
            b += 1
    pool = need + spare_blocks
    free = rng.permutation(pool)
    k_cache = randn((pool, num_kv_heads, bs, head_dim), gen)
    v_cache = randn((pool, num_kv_heads, bs, head_dim), gen)
    rows, lens, shared, starts, partial = [], [], [], [0], []
    pos, b = 0, 0
    for gi, n in enumerate(group_sizes):
        P = int(prefix_lens[gi])
        full = P // bs
        pre = free[pos:pos + full].tolist()
        pos += full
        leader_row = None
        for _ in range(n):
            L = P + int(suffix_lens[b])
            own = (L + bs - 1) // bs - full
            r = pre + free[pos:pos + own].tolist()
            pos += own
            rows.append(r)
            lens.append(L)
            shared.append(P)
            if leader_row is None:
                leader_row = r
            elif P % bs and own > 0:
                partial.append((leader_row[full], r[full], P % bs))
            b += 1
        starts.append(starts[-1] + n)
    width = max(1, max(len(r) for r in rows))
    tables = _table_tensor(rows, width)
    seq_lens = torch.tensor(lens, dtype=torch.int32)
    q = randn((B, num_q_heads, head_dim), gen)
    case = PagedCase(name, torch.bfloat16, pool, bs, num_kv_heads, num_q_heads, head_dim, k_cache,
                     v_cache, tables, seq_lens, 1.0 / float(np.sqrt(head_dim)), mask_kind, 0,
                     None, q)
    if peaky:
        make_peaky(case, seed + 7)

    def copy_prefix_rows():
        for src, dst, r in partial:
            case.k_cache[dst, :, :r] = case.k_cache[src, :, :r]
            case.v_cache[dst, :, :r] = case.v_cache[src, :, :r]

    copy_prefix_rows()
    case.extra["group_start"] = torch.tensor(starts, dtype=torch.int32)
    case.extra["shared_len"] = torch.tensor(shared, dtype=torch.int32)
    case.extra["max_group_size"] = max(group_sizes)
    case.extra["unique_blocks"] = len(set(int(x) for r in rows for x in r))
    return case


def make_prefill_case(name, *, ctx_lens, q_lens, num_q_heads, num_kv_heads, head_dim,
                      block_size, num_blocks, dtype=torch.bfloat16, seed, mask_kind=MASK_CAUSAL,
                      window=0, window_per_seq=None, scale=None, peaky=False):
    """Chunked prefill: sequence b holds ctx_lens[b] cached tokens and gets
    q_lens[b] new ones. Each sequence's table covers ctx + q tokens (blocks
    from one seeded permutation, in batch order) so the chunk can be appended
    through ``slot_mapping``."""
    gen = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    ctx_lens = [int(x) for x in ctx_lens]
    q_lens = [int(x) for x in q_lens]
    B = len(ctx_lens)
    nblk = [(c + q + block_size - 1) // block_size for c, q in zip(ctx_lens, q_lens)]
    if sum(nblk) > num_blocks:
        raise ValueError("pool too small")
    perm = rng.permutation(num_blocks)
    rows, pos = [], 0
    for n in nblk:
        rows.append(perm[pos:pos + n].tolist())
        pos += n
    tables = _table_tensor(rows, max(1, max(nblk)))
    T = sum(q_lens)
    k_cache = randn((num_blocks, num_kv_heads, block_size, head_dim), gen, dtype)
    v_cache = randn((num_blocks, num_kv_heads, block_size, head_dim), gen, dtype)
    q = randn((T, num_q_heads, head_dim), gen, dtype)
    k_new = randn((T, num_kv_heads, head_dim), gen, dtype)
    v_new = randn((T, num_kv_heads, head_dim), gen, dtype)
    slots = np.empty(T, dtype=np.int64)
    t = 0
    for b in range(B):
        for i in range(q_lens[b]):
            p = ctx_lens[b] + i
            slots[t] = rows[b][p // block_size] * block_size + p % block_size
            t += 1
    if scale is None:
        scale = 1.0 / float(np.sqrt(head_dim))
    case = PagedCase(name, dtype, num_blocks, block_size, num_kv_heads, num_q_heads, head_dim,
                     k_cache, v_cache, tables,
                     torch.tensor([c + q for c, q in zip(ctx_lens, q_lens)], dtype=torch.int32),
                     scale, mask_kind, window, window_per_seq, q, k_new, v_new,
                     torch.from_numpy(slots), torch.tensor(ctx_lens, dtype=torch.int32),
                     torch.tensor(q_lens, dtype=torch.int32))
    if peaky:
        g = num_q_heads // num_kv_heads
        case.q = (case.q.float() * 8.0).to(dtype)
        # plant one strong key per (b, kv head) in the context, along query head 0 of
        # the group at the chunk's first token
        start = 0
        for b in range(B):
            if ctx_lens[b] > 0 and q_lens[b] > 0:
                for kvh in range(num_kv_heads):
                    p = int(rng.integers(0, ctx_lens[b]))
                    qh = case.q[start, kvh * g].float()
                    case.k_cache[rows[b][p // block_size], kvh, p % block_size] = \
                        (6.0 * qh / qh.norm()).to(dtype)
            start += q_lens[b]
        case.extra["peaky"] = True
    return case


def config5(batch=4, ctx=30720, chunk=2048, num_blocks=16384, seed=None, peaky=False):
    """Long-context chunked prefill: 30720 cached + 2048 new tokens per sequence."""
    return make_prefill_case(f"cfg5_prefill_B{batch}", ctx_lens=[ctx] * batch,
                             q_lens=[chunk] * batch, num_q_heads=32, num_kv_heads=8,
                             head_dim=128, block_size=16, num_blocks=num_blocks,
                             seed=seed if seed is not None else seed_for(5),
                             mask_kind=MASK_CAUSAL, peaky=peaky)


# --------------------------------------------------------------------------- mask data

def document_starts(lens, seed, mean_doc=200, first_at_zero=True):
    """Seeded document boundaries for packed sequences: for sequence b, start
    positions in [0, lens[b]) with gaps drawn from an exponential of mean
    ``mean_doc`` (at least 1). Returns (doc_offsets int32 [B+1], doc_starts
    int32), the CSR form the mask takes."""
    rng = np.random.default_rng(seed)
    per = []
    for L in lens:
        st = [0] if first_at_zero else []
        p = 0 if first_at_zero else int(rng.integers(1, max(2, mean_doc)))
        if not first_at_zero and p < L:
            st.append(p)
        while True:
            p += max(1, int(rng.exponential(mean_doc)))
            if p >= L:
                break
            st.append(p)
        per.append(st)
    off = np.concatenate([[0], np.cumsum([len(x) for x in per])]).astype(np.int32)
    flat = np.array([x for st in per for x in st], dtype=np.int32)
    return torch.from_numpy(off), torch.from_numpy(flat)


def with_mask(case, kind, **tensors):
    """Set a case's mask kind and its further mask tensors (window_per_head,
    prefix_len, doc_offsets, doc_starts; CPU int32)."""
    case.mask_kind = kind
    case.extra["mask"] = {k: v for k, v in tensors.items() if v is not None}
    case.name += f"_mask{kind}"
    return case
