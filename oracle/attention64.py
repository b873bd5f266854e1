"""Plain float64 definition of paged attention, KV append and block-table gather.

TEST INFRASTRUCTURE ONLY. Imported by the tests, the smoke check and the CPU
baseline of ``bench.py``; never by the library. Slow and obvious on purpose:
every step is the definition, with NumPy's matmul/exp/log as the only library
primitives and no blocking, fusion or reordering.

Conventions (readings of the pages, listed with reasons in the design notes):

* Cache pools are ``[num_blocks, num_kv_heads, block_size, head_dim]``. The
  token at logical position ``p`` of sequence ``b`` lives in physical block
  ``block_tables[b][p // block_size]`` at row ``p % block_size`` ("Ultimate
  Guide to PagedAttention", the block-table section: the table maps logical
  positions of a sequence to physical memory).
* A slot is ``block * block_size + row``; appending a token writes its K/V to
  that slot and moves nothing else (same page, the section on dynamic growth).
* Masks follow FlexAttention's ``mask_mod(b, h, q_idx, kv_idx)`` idea ("Paged
  Attention Meets FlexAttention", abstract): none, causal (``kv <= q``),
  sliding window W (causal and ``q - kv < W``, i.e. exactly W keys including
  the query's own position; a window ``<= 0`` means causal only; the window
  may be per sequence or per query head, the per-head one taking precedence),
  prefix-LM (causal, plus every key of the sequence's first ``prefix_len``
  positions), and documents (sequences packed from several documents: causal
  and both positions in the same document, documents being the runs between
  consecutive start positions).
* Query head ``h`` reads KV head ``h // (Hq / Hkv)`` (contiguous grouping).
* ``lse`` is the natural-log log-sum-exp of the scaled, masked scores. A row
  that sees no key returns ``out = 0`` and ``lse = -inf``.
"""

import numpy as np

MASK_NONE = 0
MASK_CAUSAL = 1
MASK_SLIDING = 2
MASK_PREFIX_LM = 3
MASK_DOCUMENT = 4


def _f64(x):
    """Upcast a NumPy array or a CPU torch tensor (any float dtype) to float64."""
    if hasattr(x, "detach"):  # torch tensor: bf16 has no NumPy dtype, go via float64
        import torch

        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _i64(x):
    if hasattr(x, "detach"):
        return x.detach().cpu().numpy().astype(np.int64)
    return np.asarray(x, dtype=np.int64)


def document_of(doc_starts, pos):
    """Index of the document holding each position: the number of document
    start positions at or before it."""
    starts = np.sort(np.asarray(doc_starts, dtype=np.int64))
    return np.searchsorted(starts, np.asarray(pos), side="right")


def visible(kind, q_pos, k_pos, window, prefix_len=0, doc_starts=None):
    """Mask modifier: may query position ``q_pos`` see key position ``k_pos``?

    Works elementwise on broadcastable integer arrays. Keys beyond the
    sequence are never passed in, so ``none`` is always true here.
    ``window`` is the sliding window of this (sequence, head); ``prefix_len``
    the sequence's bidirectional prefix (prefix-LM); ``doc_starts`` the
    sequence's document start positions (documents).
    """
    q_pos = np.asarray(q_pos)
    k_pos = np.asarray(k_pos)
    if kind == MASK_NONE:
        return np.ones(np.broadcast(q_pos, k_pos).shape, dtype=bool)
    causal = k_pos <= q_pos
    if kind == MASK_CAUSAL:
        return causal
    if kind == MASK_SLIDING:
        if window is None or window <= 0:
            return causal
        return causal & (q_pos - k_pos < window)
    if kind == MASK_PREFIX_LM:
        return causal | (k_pos < prefix_len)
    if kind == MASK_DOCUMENT:
        return causal & (document_of(doc_starts, q_pos) == document_of(doc_starts, k_pos))
    raise ValueError(f"unknown mask kind {kind}")


def resolve_block_table(cache, table_row, length, block_size):
    """Contiguous ``[length, Hkv, d]`` view of one sequence's paged K or V.

    Position p is read from block ``table_row[p // block_size]``, row
    ``p % block_size``; table entries past the last needed block are unused.
    """
    table_row = _i64(table_row)
    pos = np.arange(length)
    blocks = table_row[pos // block_size]
    rows = pos % block_size
    if hasattr(cache, "detach"):
        import torch

        blocks = torch.from_numpy(blocks)
        rows = torch.from_numpy(rows)
    # advanced indices on axes 0 and 2 around a slice: result is [length, Hkv, d]
    return _f64(cache[blocks, :, rows, :])


def masked_attention(q, k, v, q_pos, k_pos, scale, kind, window, prefix_len=0, doc_starts=None):
    """Softmax attention of one head.

    q: [nq, d]; k, v: [n, d]; q_pos: [nq]; k_pos: [n]; the mask arguments are
    those of ``visible``.
    Returns out [nq, d] and lse [nq] (natural log of the sum of exp of the
    scaled visible scores).
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    nq = q.shape[0]
    d = v.shape[1]
    out = np.zeros((nq, d))
    lse = np.full(nq, -np.inf)
    if k.shape[0] == 0 or nq == 0:
        return out, lse
    s = scale * (q @ k.T)  # [nq, n]
    vis = visible(kind, np.asarray(q_pos)[:, None], np.asarray(k_pos)[None, :], window,
                  prefix_len, doc_starts)
    s = np.where(vis, s, -np.inf)
    any_vis = vis.any(axis=1)
    m = np.where(any_vis, s.max(axis=1), 0.0)
    e = np.exp(s - m[:, None])  # exp(-inf) = 0 for masked keys
    total = e.sum(axis=1)
    lse = np.where(any_vis, m + np.log(np.where(any_vis, total, 1.0)), -np.inf)
    p = np.where(any_vis[:, None], e / np.where(any_vis, total, 1.0)[:, None], 0.0)
    out = p @ v
    return out, lse


def _mask_of(b, h, window, window_per_seq, window_per_head, prefix_len, doc_offsets,
             doc_starts):
    """(window, prefix_len, doc_starts) of sequence b, query head h."""
    if window_per_head is not None:
        w = int(_i64(window_per_head)[h])
    elif window_per_seq is not None:
        w = int(_i64(window_per_seq)[b])
    else:
        w = int(window) if window is not None else 0
    P = int(_i64(prefix_len)[b]) if prefix_len is not None else 0
    starts = None
    if doc_offsets is not None:
        off = _i64(doc_offsets)
        starts = _i64(doc_starts)[off[b]:off[b + 1]]
    return w, P, starts


def paged_decode_rows(q, k_cache, v_cache, block_tables, seq_lens, scale, kind,
                      window=0, window_per_seq=None, rows=None, window_per_head=None,
                      prefix_len=None, doc_offsets=None, doc_starts=None):
    """Decode attention for selected (b, h) pairs (all pairs when rows is None).

    One query token per sequence at position ``seq_lens[b] - 1`` (the token
    just appended) attends to the sequence's first ``seq_lens[b]`` keys.
    Mask arguments: ``window_per_head`` [Hq], ``prefix_len`` [B], and the
    documents of sequence b at ``doc_starts[doc_offsets[b]:doc_offsets[b+1]]``.
    Returns dict (b, h) -> (out [d], lse).
    """
    q = _f64(q)
    seq_lens = _i64(seq_lens)
    tables = _i64(block_tables)
    B, Hq, _ = q.shape
    Hkv = k_cache.shape[1]
    bs = k_cache.shape[2]
    g = Hq // Hkv
    if rows is None:
        rows = [(b, h) for b in range(B) for h in range(Hq)]
    res = {}
    cache_kv = {}
    for b, h in rows:
        L = int(seq_lens[b])
        if b not in cache_kv:
            cache_kv[b] = (resolve_block_table(k_cache, tables[b], L, bs),
                           resolve_block_table(v_cache, tables[b], L, bs))
        K, V = cache_kv[b]
        kvh = h // g
        w, P, starts = _mask_of(b, h, window, window_per_seq, window_per_head, prefix_len,
                                doc_offsets, doc_starts)
        o, l = masked_attention(q[b, h][None, :], K[:, kvh, :], V[:, kvh, :],
                                np.array([L - 1]), np.arange(L), scale, kind, w, P, starts)
        res[(b, h)] = (o[0], l[0])
    return res


def paged_decode(q, k_cache, v_cache, block_tables, seq_lens, scale, kind,
                 window=0, window_per_seq=None, **mask):
    """Full decode: out [B, Hq, d] float64, lse [B, Hq] float64. ``mask`` takes
    the further mask arguments of ``paged_decode_rows``."""
    B, Hq, d = q.shape
    res = paged_decode_rows(q, k_cache, v_cache, block_tables, seq_lens, scale, kind,
                            window, window_per_seq, **mask)
    out = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    for (b, h), (o, l) in res.items():
        out[b, h] = o
        lse[b, h] = l
    return out, lse


def paged_prefill_rows(q, k_new, v_new, k_cache, v_cache, block_tables, ctx_lens, q_lens,
                       scale, kind, window=0, window_per_seq=None, rows=None,
                       window_per_head=None, prefix_len=None, doc_offsets=None,
                       doc_starts=None):
    """Chunked prefill for selected (b, h, i) rows (all rows when rows is None).

    Sequence b has ``ctx_lens[b]`` tokens already in the paged cache, followed
    by ``q_lens[b]`` new tokens packed (in batch order) in q / k_new / v_new.
    New query i of sequence b sits at absolute position ``ctx_lens[b] + i``;
    its keys are the context (positions ``0 .. ctx-1`` from the cache) and the
    new chunk (positions ``ctx + j`` from k_new/v_new), masked by the mask
    modifier. Returns dict (b, h, i) -> (out [d], lse).
    """
    q = _f64(q)
    ctx = _i64(ctx_lens)
    ql = _i64(q_lens)
    tables = _i64(block_tables)
    B = ctx.shape[0]
    Hq = q.shape[1]
    Hkv = k_cache.shape[1]
    bs = k_cache.shape[2]
    g = Hq // Hkv
    starts = np.concatenate([[0], np.cumsum(ql)])
    if rows is None:
        rows = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(int(ql[b]))]
    kv_of = {}
    res = {}
    for b, h, i in rows:
        C = int(ctx[b])
        Q = int(ql[b])
        if b not in kv_of:
            kctx = resolve_block_table(k_cache, tables[b], C, bs)
            vctx = resolve_block_table(v_cache, tables[b], C, bs)
            kn = _f64(k_new[starts[b]:starts[b] + Q])
            vn = _f64(v_new[starts[b]:starts[b] + Q])
            kv_of[b] = (np.concatenate([kctx, kn], axis=0), np.concatenate([vctx, vn], axis=0))
        K, V = kv_of[b]
        kvh = h // g
        n = C + Q
        w, P, dst = _mask_of(b, h, window, window_per_seq, window_per_head, prefix_len,
                             doc_offsets, doc_starts)
        o, l = masked_attention(q[starts[b] + i, h][None, :], K[:, kvh, :], V[:, kvh, :],
                                np.array([C + i]), np.arange(n), scale, kind, w, P, dst)
        res[(b, h, i)] = (o[0], l[0])
    return res


def paged_prefill_tile(q, k_new, v_new, k_cache, v_cache, block_tables, ctx_lens, q_lens,
                      scale, kind, b, i0, i1, heads=None, window=0, window_per_seq=None,
                      window_per_head=None, prefix_len=None, doc_offsets=None,
                      doc_starts=None):
    """Chunked prefill of new queries i0 .. i1-1 of sequence b, for the given
    query heads (all when None): out [i1-i0, len(heads), d], lse [i1-i0,
    len(heads)] (float64). The same definition as ``paged_prefill``, evaluated
    on one block of query rows at a time (a whole query tile of a long
    sequence costs one matrix product per head)."""
    q = _f64(q)
    ctx = _i64(ctx_lens)
    ql = _i64(q_lens)
    tables = _i64(block_tables)
    Hq = q.shape[1]
    Hkv = k_cache.shape[1]
    bs = k_cache.shape[2]
    g = Hq // Hkv
    heads = list(range(Hq)) if heads is None else list(heads)
    starts = np.concatenate([[0], np.cumsum(ql)])
    C, Q = int(ctx[b]), int(ql[b])
    i1 = min(int(i1), Q)
    s0 = int(starts[b])
    kn = _f64(k_new[s0:s0 + Q])
    vn = _f64(v_new[s0:s0 + Q])
    d = q.shape[2]
    out = np.zeros((max(i1 - i0, 0), len(heads), d))
    lse = np.zeros((max(i1 - i0, 0), len(heads)))
    by_kv = {}
    for j, h in enumerate(heads):
        kvh = h // g
        if kvh not in by_kv:
            kctx = resolve_block_table(k_cache[:, kvh:kvh + 1], tables[b], C, bs)[:, 0]
            vctx = resolve_block_table(v_cache[:, kvh:kvh + 1], tables[b], C, bs)[:, 0]
            by_kv[kvh] = (np.concatenate([kctx, kn[:, kvh]], axis=0),
                          np.concatenate([vctx, vn[:, kvh]], axis=0))
        K, V = by_kv[kvh]
        w, P, dst = _mask_of(b, h, window, window_per_seq, window_per_head, prefix_len,
                             doc_offsets, doc_starts)
        o, l = masked_attention(q[s0 + i0:s0 + i1, h], K, V, C + np.arange(i0, i1),
                                np.arange(C + Q), scale, kind, w, P, dst)
        out[:, j] = o
        lse[:, j] = l
    return out, lse


def paged_prefill(q, k_new, v_new, k_cache, v_cache, block_tables, ctx_lens, q_lens,
                  scale, kind, window=0, window_per_seq=None, window_per_head=None,
                  prefix_len=None, doc_offsets=None, doc_starts=None):
    """Full chunked prefill: out [sum Q, Hq, d], lse [sum Q, Hq] (float64).

    Computed head by head as one matrix of queries per sequence; mask
    arguments as in ``paged_prefill_rows``.
    """
    q = _f64(q)
    ctx = _i64(ctx_lens)
    ql = _i64(q_lens)
    tables = _i64(block_tables)
    T, Hq, d = q.shape
    Hkv = k_cache.shape[1]
    bs = k_cache.shape[2]
    g = Hq // Hkv
    out = np.zeros((T, Hq, d))
    lse = np.zeros((T, Hq))
    start = 0
    for b in range(ctx.shape[0]):
        C, Q = int(ctx[b]), int(ql[b])
        kctx = resolve_block_table(k_cache, tables[b], C, bs)
        vctx = resolve_block_table(v_cache, tables[b], C, bs)
        K = np.concatenate([kctx, _f64(k_new[start:start + Q])], axis=0)
        V = np.concatenate([vctx, _f64(v_new[start:start + Q])], axis=0)
        for h in range(Hq):
            w, P, dst = _mask_of(b, h, window, window_per_seq, window_per_head, prefix_len,
                                 doc_offsets, doc_starts)
            o, l = masked_attention(q[start:start + Q, h], K[:, h // g], V[:, h // g],
                                    C + np.arange(Q), np.arange(C + Q), scale, kind, w, P, dst)
            out[start:start + Q, h] = o
            lse[start:start + Q, h] = l
        start += Q
    return out, lse


def kv_append(k, v, slot_mapping, k_cache, v_cache):
    """Expected pools after appending tokens: copies, inputs are not modified.

    Token t (slot >= 0) overwrites row ``slot % block_size`` of block
    ``slot // block_size`` for every KV head; negative slots are padding and
    write nothing. Works on the stored bit patterns (any dtype); slots are
    assumed distinct.
    """
    kc = k_cache.clone() if hasattr(k_cache, "clone") else np.array(k_cache, copy=True)
    vc = v_cache.clone() if hasattr(v_cache, "clone") else np.array(v_cache, copy=True)
    bs = kc.shape[2]
    slots = _i64(slot_mapping)
    for t, slot in enumerate(slots):
        if slot < 0:
            continue
        kc[slot // bs, :, slot % bs, :] = k[t]
        vc[slot // bs, :, slot % bs, :] = v[t]
    return kc, vc


def kv_gather(k_cache, v_cache, block_tables, seq_lens, out_max_len):
    """Contiguous copies ``[B, Hkv, out_max_len, d]`` of each sequence's K and V.

    Positions ``>= seq_lens[b]`` are zero; a longer sequence is cut at
    ``out_max_len``. Copies stored values exactly (any
    dtype, torch or NumPy), so it can be compared bit for bit.
    """
    lens = _i64(seq_lens)
    tables = _i64(block_tables)
    B = lens.shape[0]
    NB, Hkv, bs, d = k_cache.shape
    if hasattr(k_cache, "new_zeros"):
        ko = k_cache.new_zeros((B, Hkv, out_max_len, d))
        vo = v_cache.new_zeros((B, Hkv, out_max_len, d))
    else:
        ko = np.zeros((B, Hkv, out_max_len, d), dtype=k_cache.dtype)
        vo = np.zeros((B, Hkv, out_max_len, d), dtype=v_cache.dtype)
    for b in range(B):
        L = min(int(lens[b]), out_max_len)
        pos = np.arange(L)
        blocks, rows = tables[b][pos // bs], pos % bs
        if hasattr(k_cache, "detach"):
            import torch

            blocks, rows = torch.from_numpy(blocks), torch.from_numpy(rows)
        # k_cache[blocks, :, rows, :] is [L, Hkv, d]; the output wants [Hkv, L, d]
        ko[b, :, :L, :] = k_cache[blocks, :, rows, :].transpose(1, 0, 2) \
            if not hasattr(k_cache, "detach") else k_cache[blocks, :, rows, :].transpose(0, 1)
        vo[b, :, :L, :] = v_cache[blocks, :, rows, :].transpose(1, 0, 2) \
            if not hasattr(v_cache, "detach") else v_cache[blocks, :, rows, :].transpose(0, 1)
    return ko, vo


def kv_copy_blocks(k_cache, v_cache, block_pairs):
    """Expected pools after copy-on-write: for each (src, dst) pair, block dst
    becomes a copy of block src (all KV heads, K and V). Copies, inputs are not
    modified; destinations are assumed distinct and not sources."""
    kc = k_cache.clone() if hasattr(k_cache, "clone") else np.array(k_cache, copy=True)
    vc = v_cache.clone() if hasattr(v_cache, "clone") else np.array(v_cache, copy=True)
    for src, dst in _i64(block_pairs).reshape(-1, 2):
        kc[dst] = k_cache[src]
        vc[dst] = v_cache[src]
    return kc, vc
