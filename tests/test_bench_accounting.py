"""The bench's unit counts against independent definitions (CPU): the decode
bytes per step come from the number of visible tokens, which must equal a
count of the keys the oracle's mask admits; the growth plan must hand every
sequence distinct physical blocks and put each new token at the slot the
block-table rule gives; the prefill FLOP count must equal 4 d Hq times the
number of (query, key) pairs the causal mask admits."""

import numpy as np
import torch

import bench
import oracle
from paged_kv_cache_gather_b200 import inputs as I


def test_visible_tokens_match_the_mask():
    rng = np.random.default_rng(0)
    lens = rng.integers(0, 300, size=40)
    wps = rng.choice([0, 1, 7, 64, 500], size=40)
    got = bench.visible_tokens(lens, wps)
    for L, w, n in zip(lens, wps, got):
        q = L - 1
        want = sum(oracle.visible(oracle.MASK_SLIDING, q, k, int(w)) for k in range(L))
        assert n == want, (L, w, n, want)


def test_growth_plan_blocks_and_slots():
    steps = 40
    case = I.config3(batch=8, max_len=200, num_blocks=400, window=64, growth_steps=steps + 1,
                     seed=5)
    tab, lens, slots = bench.decode_plan(case, steps)
    tab, lens, slots = tab.numpy(), lens.numpy(), slots.numpy()
    bs = case.block_size
    lens0 = case.seq_lens.numpy()
    for s in range(steps):
        assert np.array_equal(lens[s], lens0 + s)
        assert len(set(slots[s].tolist())) == case.batch
        for b in range(case.batch):
            p = int(lens[s, b]) - 1
            assert slots[s, b] == tab[b, p // bs] * bs + p % bs
    # every block a sequence uses (up to its final length) is its own
    owner = {}
    for b in range(case.batch):
        for j in range((int(lens[-1, b]) + bs - 1) // bs):
            blk = int(tab[b, j])
            assert 0 <= blk < case.num_blocks and owner.setdefault(blk, b) == b


def test_prefill_flops_match_the_causal_pair_count():
    C = np.array([5, 0, 37])
    Q = np.array([3, 9, 4])
    pairs = 0
    for c, q in zip(C, Q):
        for i in range(q):
            pairs += sum(oracle.visible(oracle.MASK_CAUSAL, c + i, k, 0) for k in range(c + q))
    assert bench.causal_pairs(C, Q) == pairs


def brute_pairs(C, Q, kind, **kw):
    n = 0
    for b, (c, q) in enumerate(zip(C, Q)):
        extra = {}
        if kind == oracle.MASK_PREFIX_LM:
            extra["prefix_len"] = int(kw["prefix_len"][b])
        if kind == oracle.MASK_DOCUMENT:
            off, st = kw["doc_offsets"], kw["doc_starts"]
            extra["doc_starts"] = np.asarray(st[off[b]:off[b + 1]])
        for i in range(q):
            n += sum(oracle.visible(kind, c + i, k, 0, **extra) for k in range(c + q))
    return n


def test_document_and_prefix_lm_pair_counts_match_the_mask():
    C = [40, 0, 17]
    Q = [30, 25, 9]
    off, st = I.document_starts([c + q for c, q in zip(C, Q)], 3, mean_doc=12)
    off, st = off.numpy(), st.numpy()
    assert bench.document_pairs(C, Q, off, st) == brute_pairs(
        C, Q, oracle.MASK_DOCUMENT, doc_offsets=off, doc_starts=st)
    plen = [c + q // 2 for c, q in zip(C, Q)]
    assert bench.prefix_lm_pairs(C, Q, plen) == brute_pairs(C, Q, oracle.MASK_PREFIX_LM,
                                                            prefix_len=plen)

