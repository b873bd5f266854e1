"""Pins of the float64 oracle against things other than itself (CPU only).

* dense attention from a different library routine (torch SDPA, float64) on a
  contiguous layout, and ``torch.logsumexp`` of explicit scores;
* invariance under any permutation of the physical blocks ("Ultimate Guide to
  PagedAttention": blocks may sit anywhere without changing results);
* closed forms: identical keys give the mean of V and ``lse = s + ln n``; one
  dominant key returns its V row; a window at least as long as the sequence
  equals causal; decode equals the last row of a one-token prefill;
  splitting the keys and merging by log-sum-exp gives the whole;
* a pure-Python brute force (scalar loops, ``math.exp``) on tiny inputs;
* shared-prefix block ids versus copied prefixes (same page, sharing section);
* planted mistakes in the oracle are caught by the brute force.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from oracle import attention64 as A
from paged_kv_cache_gather_b200 import inputs as I

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ----------------------------------------------------------------- brute force

def brute_doc(starts, p):
    n = 0
    for st in starts:
        if st <= p:
            n += 1
    return n


def brute_visible(kind, qp, kp, w, P=0, starts=()):
    if kind == 0:
        return True
    if kind == 3 and kp < P:
        return True
    if kp > qp:
        return False
    if kind == 2 and w > 0 and qp - kp >= w:
        return False
    if kind == 4 and brute_doc(starts, qp) != brute_doc(starts, kp):
        return False
    return True


def brute_paged_attention(qrow, k_cache, v_cache, table, n_keys, q_pos, kvh, scale, kind, w,
                          extra_k=(), extra_v=(), P=0, starts=()):
    """Scalar loops over Python lists; keys 0..n_keys-1 come from the paged
    cache, further keys (positions n_keys, n_keys+1, ...) from extra_k/extra_v."""
    bs = len(k_cache[0][0])
    keys, vals = [], []
    for p in range(n_keys):
        blk = table[p // bs]
        keys.append(k_cache[blk][kvh][p % bs])
        vals.append(v_cache[blk][kvh][p % bs])
    keys += list(extra_k)
    vals += list(extra_v)
    scores = []
    for p, k in enumerate(keys):
        if brute_visible(kind, q_pos, p, w, P, starts):
            s = 0.0
            for a, b in zip(qrow, k):
                s += a * b
            scores.append((p, scale * s))
    d = len(vals[0]) if vals else len(qrow)
    if not scores:
        return [0.0] * d, -math.inf
    m = max(s for _, s in scores)
    z = 0.0
    for _, s in scores:
        z += math.exp(s - m)
    out = [0.0] * d
    for p, s in scores:
        wgt = math.exp(s - m) / z
        for i in range(d):
            out[i] += wgt * vals[p][i]
    return out, m + math.log(z)


def tiny_case(seed, B, Hq, Hkv, d, bs, NB, lens, kind, window, dtype=torch.float64):
    gen = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    kc = torch.randn(NB, Hkv, bs, d, generator=gen, dtype=torch.float64).to(dtype)
    vc = torch.randn(NB, Hkv, bs, d, generator=gen, dtype=torch.float64).to(dtype)
    q = torch.randn(B, Hq, d, generator=gen, dtype=torch.float64).to(dtype)
    perm = rng.permutation(NB)
    nblk = [-(-L // bs) for L in lens]
    width = max(1, max(nblk))
    tab = np.full((B, width), -1, dtype=np.int64)
    pos = 0
    for b, n in enumerate(nblk):
        tab[b, :n] = perm[pos:pos + n]
        pos += n
    return q, kc, vc, tab, np.array(lens), 1.0 / math.sqrt(d)


BRUTE_CASES = [
    # (B, Hq, Hkv, d, bs, NB, lens, kind, window)
    (2, 2, 1, 4, 1, 80, [17, 40], A.MASK_NONE, 0),
    (3, 4, 2, 8, 2, 64, [1, 13, 33], A.MASK_CAUSAL, 0),
    (2, 4, 4, 8, 4, 32, [29, 40], A.MASK_SLIDING, 5),
    (2, 6, 3, 8, 16, 8, [16, 39], A.MASK_SLIDING, 16),
    (1, 8, 2, 5, 4, 16, [38], A.MASK_SLIDING, 1),
]


@pytest.mark.parametrize("case", BRUTE_CASES)
def test_decode_matches_brute_force(case):
    B, Hq, Hkv, d, bs, NB, lens, kind, w = case
    q, kc, vc, tab, lens, scale = tiny_case(11, B, Hq, Hkv, d, bs, NB, lens, kind, w)
    out, lse = oracle.paged_decode(q, kc, vc, tab, lens, scale, kind, w)
    kl, vl, ql = kc.tolist(), vc.tolist(), q.tolist()
    g = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            o_ref, l_ref = brute_paged_attention(ql[b][h], kl, vl, tab[b].tolist(), int(lens[b]),
                                                 int(lens[b]) - 1, h // g, scale, kind, w)
            np.testing.assert_allclose(out[b, h], o_ref, rtol=0, atol=1e-13)
            assert abs(lse[b, h] - l_ref) < 1e-13


@pytest.mark.parametrize("kind,w", [(A.MASK_NONE, 0), (A.MASK_CAUSAL, 0), (A.MASK_SLIDING, 7)])
def test_prefill_matches_brute_force(kind, w):
    B, Hq, Hkv, d, bs = 3, 4, 2, 8, 4
    ctx, ql = [0, 9, 22], [5, 7, 3]
    gen = torch.Generator().manual_seed(5)
    q, kc, vc, tab, _, scale = tiny_case(5, B, Hq, Hkv, d, bs, 40,
                                         [c + n for c, n in zip(ctx, ql)], kind, w)
    T = sum(ql)
    qp = torch.randn(T, Hq, d, generator=gen, dtype=torch.float64)
    kn = torch.randn(T, Hkv, d, generator=gen, dtype=torch.float64)
    vn = torch.randn(T, Hkv, d, generator=gen, dtype=torch.float64)
    out, lse = oracle.paged_prefill(qp, kn, vn, kc, vc, tab, ctx, ql, scale, kind, w)
    kl, vl = kc.tolist(), vc.tolist()
    g = Hq // Hkv
    start = 0
    for b in range(B):
        for i in range(ql[b]):
            for h in range(Hq):
                ek = [kn[start + j, h // g].tolist() for j in range(ql[b])]
                ev = [vn[start + j, h // g].tolist() for j in range(ql[b])]
                o_ref, l_ref = brute_paged_attention(qp[start + i, h].tolist(), kl, vl,
                                                     tab[b].tolist(), ctx[b], ctx[b] + i, h // g,
                                                     scale, kind, w, ek, ev)
                np.testing.assert_allclose(out[start + i, h], o_ref, rtol=0, atol=1e-13)
                assert abs(lse[start + i, h] - l_ref) < 1e-13
        start += ql[b]


def test_rows_api_matches_full():
    q, kc, vc, tab, lens, scale = tiny_case(3, 3, 4, 2, 8, 4, 64, [5, 30, 17], A.MASK_SLIDING, 6)
    out, lse = oracle.paged_decode(q, kc, vc, tab, lens, scale, A.MASK_SLIDING, 6)
    rows = oracle.paged_decode_rows(q, kc, vc, tab, lens, scale, A.MASK_SLIDING, 6,
                                    rows=[(2, 3), (0, 0)])
    for (b, h), (o, l) in rows.items():
        assert np.array_equal(o, out[b, h]) and l == lse[b, h]


# ----------------------------------------------------------------- planted mistakes

def _mut_causal_strict(kind, q_pos, k_pos, window, prefix_len=0, doc_starts=None):
    q_pos, k_pos = np.asarray(q_pos), np.asarray(k_pos)
    if kind == A.MASK_NONE:
        return np.ones(np.broadcast(q_pos, k_pos).shape, dtype=bool)
    c = k_pos < q_pos  # planted: drops the query's own key
    if kind == A.MASK_SLIDING and window > 0:
        return c & (q_pos - k_pos < window)
    return c


def _mut_window_inclusive(kind, q_pos, k_pos, window, prefix_len=0, doc_starts=None):
    q_pos, k_pos = np.asarray(q_pos), np.asarray(k_pos)
    if kind == A.MASK_NONE:
        return np.ones(np.broadcast(q_pos, k_pos).shape, dtype=bool)
    c = k_pos <= q_pos
    if kind == A.MASK_SLIDING and window > 0:
        return c & (q_pos - k_pos <= window)  # planted: W + 1 keys
    return c


@pytest.mark.parametrize("mutation", ["causal_strict", "window_inclusive", "kv_head_swap",
                                      "no_scale", "row_index"])
def test_planted_mistakes_are_caught(monkeypatch, mutation):
    """Each plausible slip in the oracle must make the brute-force pin fail."""
    B, Hq, Hkv, d, bs, NB, lens, kind, w = (2, 4, 2, 8, 4, 32, [13, 22], A.MASK_SLIDING, 5)
    q, kc, vc, tab, lens, scale = tiny_case(21, B, Hq, Hkv, d, bs, NB, lens, kind, w)
    if mutation == "causal_strict":
        monkeypatch.setattr(A, "visible", _mut_causal_strict)
    elif mutation == "window_inclusive":
        monkeypatch.setattr(A, "visible", _mut_window_inclusive)
    elif mutation == "kv_head_swap":
        # planted: query heads read the wrong KV head (the pool's heads swapped)
        kc = kc[:, [1, 0]]
        vc = vc[:, [1, 0]]
    elif mutation == "row_index":
        orig_res = A.resolve_block_table

        def wrong_rows(cache, table_row, length, block_size):
            r = orig_res(cache, table_row, length + 1, block_size)
            return r[1:]  # planted: off by one position
        monkeypatch.setattr(A, "resolve_block_table", wrong_rows)
    s = 1.0 if mutation == "no_scale" else scale
    out, lse = A.paged_decode(q, kc, vc, tab, lens, s, kind, w)
    monkeypatch.undo()
    q2, kc2, vc2, _, _, _ = tiny_case(21, B, Hq, Hkv, d, bs, NB, [13, 22], kind, w)
    kl, vl = kc2.tolist(), vc2.tolist()
    g = Hq // Hkv
    worst = 0.0
    for b in range(B):
        for h in range(Hq):
            o_ref, l_ref = brute_paged_attention(q2[b, h].tolist(), kl, vl, tab[b].tolist(),
                                                 int(lens[b]), int(lens[b]) - 1, h // g, scale,
                                                 kind, w)
            worst = max(worst, float(np.max(np.abs(out[b, h] - o_ref))), abs(lse[b, h] - l_ref))
    assert worst > 1e-6, f"mutation {mutation} went unnoticed"


# ----------------------------------------------------------------- library special case

@pytest.mark.parametrize("kind,w", [(A.MASK_NONE, 0), (A.MASK_CAUSAL, 0), (A.MASK_SLIDING, 9)])
def test_contiguous_layout_matches_sdpa(kind, w):
    """Identity block table over a contiguous pool == dense SDPA (float64, bool mask)."""
    gen = torch.Generator().manual_seed(7)
    B, Hq, Hkv, d, bs, C, Q = 2, 8, 2, 16, 4, 24, 12
    n = C + Q
    nb = -(-C // bs)
    K = torch.randn(B, n, Hkv, d, generator=gen, dtype=torch.float64)
    V = torch.randn(B, n, Hkv, d, generator=gen, dtype=torch.float64)
    q = torch.randn(B * Q, Hq, d, generator=gen, dtype=torch.float64)
    # contiguous pool: sequence b owns blocks b*nb .. b*nb+nb-1, in order
    kc = torch.zeros(B * nb, Hkv, bs, d, dtype=torch.float64)
    vc = torch.zeros_like(kc)
    for b in range(B):
        kc[b * nb:(b + 1) * nb] = torch.nn.functional.pad(
            K[b, :C], (0, 0, 0, 0, 0, nb * bs - C)).view(nb, bs, Hkv, d).transpose(1, 2)
        vc[b * nb:(b + 1) * nb] = torch.nn.functional.pad(
            V[b, :C], (0, 0, 0, 0, 0, nb * bs - C)).view(nb, bs, Hkv, d).transpose(1, 2)
    tab = np.arange(B * nb).reshape(B, nb)
    scale = 0.3
    kn = K[:, C:].reshape(B * Q, Hkv, d)
    vn = V[:, C:].reshape(B * Q, Hkv, d)
    out, lse = oracle.paged_prefill(q, kn, vn, kc, vc, tab, [C] * B, [Q] * B, scale, kind, w)
    g = Hq // Hkv
    qpos = torch.arange(C, C + Q)[:, None]
    kpos = torch.arange(n)[None, :]
    if kind == A.MASK_NONE:
        mask = torch.ones(Q, n, dtype=torch.bool)
    else:
        mask = kpos <= qpos
        if kind == A.MASK_SLIDING:
            mask &= (qpos - kpos) < w
    for b in range(B):
        qb = q[b * Q:(b + 1) * Q].transpose(0, 1)  # [Hq, Q, d]
        kb = K[b].transpose(0, 1).repeat_interleave(g, 0)  # [Hq, n, d]
        vb = V[b].transpose(0, 1).repeat_interleave(g, 0)
        ref = torch.nn.functional.scaled_dot_product_attention(qb, kb, vb, attn_mask=mask,
                                                               scale=scale)
        np.testing.assert_allclose(out[b * Q:(b + 1) * Q], ref.transpose(0, 1).numpy(),
                                   rtol=0, atol=1e-12)
        scores = (qb @ kb.transpose(1, 2)) * scale
        scores = scores.masked_fill(~mask, float("-inf"))
        lref = torch.logsumexp(scores, dim=-1).transpose(0, 1)
        np.testing.assert_allclose(lse[b * Q:(b + 1) * Q], lref.numpy(), rtol=0, atol=1e-12)


# ----------------------------------------------------------------- invariants

def test_physical_permutation_invariance():
    q, kc, vc, tab, lens, scale = tiny_case(9, 4, 8, 2, 16, 4, 96, [7, 50, 64, 33],
                                            A.MASK_SLIDING, 20)
    out, lse = oracle.paged_decode(q, kc, vc, tab, lens, scale, A.MASK_SLIDING, 20)
    perm = np.random.default_rng(3).permutation(kc.shape[0])  # new id of old block i
    kc2 = torch.empty_like(kc)
    vc2 = torch.empty_like(vc)
    kc2[torch.from_numpy(perm)] = kc
    vc2[torch.from_numpy(perm)] = vc
    tab2 = np.where(tab >= 0, perm[np.maximum(tab, 0)], -1)
    out2, lse2 = oracle.paged_decode(q, kc2, vc2, tab2, lens, scale, A.MASK_SLIDING, 20)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_identical_keys_give_mean_of_values():
    q, kc, vc, tab, lens, scale = tiny_case(4, 2, 4, 2, 8, 4, 32, [21, 30], A.MASK_SLIDING, 11)
    key = torch.randn(8, dtype=torch.float64, generator=torch.Generator().manual_seed(1))
    kc[:] = key
    out, lse = oracle.paged_decode(q, kc, vc, tab, lens, scale, A.MASK_SLIDING, 11)
    for b in range(2):
        L = int(lens[b])
        lo = max(0, L - 11)
        n_vis = L - lo
        vis_v = torch.stack([vc[tab[b, p // 4], :, p % 4] for p in range(lo, L)])  # [n, Hkv, d]
        for h in range(4):
            np.testing.assert_allclose(out[b, h], vis_v[:, h // 2].mean(0).numpy(), atol=1e-13)
            expect = scale * float(q[b, h] @ key) + math.log(n_vis)
            assert abs(lse[b, h] - expect) < 1e-12


def test_dominant_key_returns_its_value():
    q, kc, vc, tab, lens, scale = tiny_case(6, 2, 2, 1, 16, 16, 8, [40, 57], A.MASK_CAUSAL, 0)
    for b in range(2):
        j = 13 + b
        # one KV head shared by both q heads: point the key along q[b, 0] + q[b, 1]
        direction = q[b, 0] + q[b, 1]
        kc[tab[b, j // 16], 0, j % 16] = 40.0 * direction / direction.norm() * math.sqrt(16)
    out, _ = oracle.paged_decode(q, kc, vc, tab, lens, scale, A.MASK_CAUSAL, 0)
    for b in range(2):
        j = 13 + b
        for h in range(2):
            # margin: the planted score beats every other by far more than 30 nats
            np.testing.assert_allclose(out[b, h], vc[tab[b, j // 16], 0, j % 16].numpy(),
                                       atol=1e-10)


def test_wide_window_equals_causal():
    q, kc, vc, tab, lens, scale = tiny_case(8, 3, 4, 2, 8, 4, 64, [3, 31, 45], A.MASK_SLIDING, 0)
    o1, l1 = oracle.paged_decode(q, kc, vc, tab, lens, scale, A.MASK_CAUSAL, 0)
    o2, l2 = oracle.paged_decode(q, kc, vc, tab, lens, scale, A.MASK_SLIDING, 45)
    o3, l3 = oracle.paged_decode(q, kc, vc, tab, lens, scale, A.MASK_SLIDING, 1000)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    assert np.array_equal(o1, o3) and np.array_equal(l1, l3)
    # causal in decode sees every key: equal to no mask as well
    o4, l4 = oracle.paged_decode(q, kc, vc, tab, lens, scale, A.MASK_NONE, 0)
    np.testing.assert_allclose(o1, o4, atol=1e-15)


def test_decode_equals_last_row_of_one_token_prefill():
    q, kc, vc, tab, lens, scale = tiny_case(12, 3, 4, 2, 8, 4, 64, [9, 26, 40], A.MASK_SLIDING, 7)
    od, ld = oracle.paged_decode(q, kc, vc, tab, lens, scale, A.MASK_SLIDING, 7)
    # the last token of each sequence becomes the "new" chunk of a 1-token prefill
    kn = torch.stack([kc[tab[b, (int(lens[b]) - 1) // 4], :, (int(lens[b]) - 1) % 4]
                      for b in range(3)])
    vn = torch.stack([vc[tab[b, (int(lens[b]) - 1) // 4], :, (int(lens[b]) - 1) % 4]
                      for b in range(3)])
    op, lp = oracle.paged_prefill(q, kn, vn, kc, vc, tab, lens - 1, [1, 1, 1], scale,
                                  A.MASK_SLIDING, 7)
    np.testing.assert_allclose(op, od, atol=1e-14)
    np.testing.assert_allclose(lp, ld, atol=1e-14)


def test_split_and_merge_equals_whole():
    """Attention over disjoint key chunks, merged by log-sum-exp weights, equals
    attention over all keys (the merge written out here, separately)."""
    gen = torch.Generator().manual_seed(2)
    n, d = 100, 16
    q = torch.randn(1, d, generator=gen, dtype=torch.float64)
    k = torch.randn(n, d, generator=gen, dtype=torch.float64)
    v = torch.randn(n, d, generator=gen, dtype=torch.float64)
    qp = np.array([n - 1])
    o, l = A.masked_attention(q, k, v, qp, np.arange(n), 0.25, A.MASK_SLIDING, 70)
    parts = []
    for lo, hi in [(0, 10), (10, 37), (37, 64), (64, 100)]:
        parts.append(A.masked_attention(q, k[lo:hi], v[lo:hi], qp, np.arange(lo, hi), 0.25,
                                        A.MASK_SLIDING, 70))
    lses = np.array([p[1][0] for p in parts])
    m = np.max(lses)
    lse = m + math.log(sum(math.exp(x - m) for x in lses if x != -math.inf))
    out = sum(math.exp(p[1][0] - lse) * p[0][0] for p in parts if p[1][0] != -math.inf)
    np.testing.assert_allclose(out, o[0], atol=1e-14)
    assert abs(lse - l[0]) < 1e-13
    assert parts[0][1][0] == -math.inf  # chunk 0..9 lies entirely outside the window


def test_empty_sequence_gives_zero_and_minus_inf():
    q, kc, vc, tab, lens, scale = tiny_case(1, 2, 2, 2, 8, 4, 8, [0, 5], A.MASK_CAUSAL, 0)
    out, lse = oracle.paged_decode(q, kc, vc, tab, lens, scale, A.MASK_CAUSAL, 0)
    assert np.all(out[0] == 0) and np.all(lse[0] == -np.inf)
    assert np.all(np.isfinite(lse[1]))


def test_shared_prefix_equals_copied_prefix():
    sh = I.config4(groups=2, beams=3, prefix=64, suffix=32, num_blocks=64, shared=True)
    cp = I.config4(groups=2, beams=3, prefix=64, suffix=32, num_blocks=64, shared=False)
    assert sh.extra["unique_blocks"] < cp.extra["unique_blocks"]
    o1, l1 = oracle.paged_decode(sh.q, sh.k_cache, sh.v_cache, sh.block_tables, sh.seq_lens,
                                 sh.scale, sh.mask_kind)
    o2, l2 = oracle.paged_decode(cp.q, cp.k_cache, cp.v_cache, cp.block_tables, cp.seq_lens,
                                 cp.scale, cp.mask_kind)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


# ----------------------------------------------------------------- append / gather

def test_append_brute_force_and_untouched_slots():
    NB, Hkv, bs, d = 6, 2, 4, 8
    kc = torch.full((NB, Hkv, bs, d), -7.0)
    vc = torch.full((NB, Hkv, bs, d), -9.0)
    k = torch.arange(5 * Hkv * d, dtype=torch.float32).view(5, Hkv, d)
    v = -k
    slots = torch.tensor([3, -1, 22, 8, 0])
    ek, ev = oracle.kv_append(k, v, slots, kc, vc)
    for blk in range(NB):
        for h in range(Hkv):
            for r in range(bs):
                slot = blk * bs + r
                t = [i for i, s in enumerate(slots.tolist()) if s == slot]
                want_k = k[t[0], h] if t else torch.full((d,), -7.0)
                want_v = v[t[0], h] if t else torch.full((d,), -9.0)
                assert torch.equal(ek[blk, h, r], want_k) and torch.equal(ev[blk, h, r], want_v)
    assert torch.all(kc == -7.0)  # inputs untouched


def test_gather_brute_force():
    q, kc, vc, tab, lens, _ = tiny_case(2, 3, 2, 2, 4, 4, 32, [5, 0, 14], A.MASK_NONE, 0,
                                        dtype=torch.bfloat16)
    ko, vo = oracle.kv_gather(kc, vc, tab, lens, 16)
    assert ko.dtype == torch.bfloat16 and ko.shape == (3, 2, 16, 4)
    cut, _ = oracle.kv_gather(kc, vc, tab, lens, 9)  # the 14-token sequence is cut at 9
    assert torch.equal(cut, ko[:, :, :9])
    for b in range(3):
        for h in range(2):
            for p in range(16):
                if p < lens[b]:
                    assert torch.equal(ko[b, h, p], kc[tab[b, p // 4], h, p % 4])
                    assert torch.equal(vo[b, h, p], vc[tab[b, p // 4], h, p % 4])
                else:
                    assert torch.all(ko[b, h, p] == 0) and torch.all(vo[b, h, p] == 0)


def test_copy_blocks_brute_force():
    kc = torch.arange(6 * 2 * 4 * 3, dtype=torch.float32).view(6, 2, 4, 3)
    vc = -kc
    ek, ev = oracle.kv_copy_blocks(kc, vc, [[1, 4], [5, 0]])
    for blk in range(6):
        src = {4: 1, 0: 5}.get(blk, blk)
        assert torch.equal(ek[blk], kc[src]) and torch.equal(ev[blk], vc[src])
    assert torch.equal(kc, torch.arange(6 * 2 * 4 * 3, dtype=torch.float32).view(6, 2, 4, 3))


# ----------------------------------------------------------------- further mask_mods

def _docs_csr(per_seq):
    off = np.concatenate([[0], np.cumsum([len(x) for x in per_seq])]).astype(np.int64)
    flat = np.concatenate([np.asarray(x, dtype=np.int64) for x in per_seq]) if per_seq else \
        np.zeros(0, dtype=np.int64)
    return off, flat


MASK_CASES = [
    # (kind, per-head windows, prefix lens, document starts per sequence)
    (A.MASK_PREFIX_LM, None, [6, 30], None),
    (A.MASK_PREFIX_LM, None, [0, 41], None),
    (A.MASK_DOCUMENT, None, None, [[0, 5, 9], [0, 17, 18, 30]]),
    (A.MASK_DOCUMENT, None, None, [[3], [0]]),
    (A.MASK_SLIDING, [3, 0, 7, 1], None, None),
]


@pytest.mark.parametrize("case", MASK_CASES)
def test_further_masks_decode_match_brute_force(case):
    kind, wph, plen, docs = case
    B, Hq, Hkv, d, bs, NB = 2, 4, 2, 8, 4, 40
    lens = [13, 38]
    q, kc, vc, tab, lens, scale = tiny_case(31, B, Hq, Hkv, d, bs, NB, lens, kind, 0)
    off, flat = _docs_csr(docs) if docs else (None, None)
    out, lse = oracle.paged_decode(q, kc, vc, tab, lens, scale, kind, 0, None,
                                   window_per_head=wph, prefix_len=plen, doc_offsets=off,
                                   doc_starts=flat)
    kl, vl, ql = kc.tolist(), vc.tolist(), q.tolist()
    g = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            o_ref, l_ref = brute_paged_attention(
                ql[b][h], kl, vl, tab[b].tolist(), int(lens[b]), int(lens[b]) - 1, h // g, scale,
                kind, wph[h] if wph else 0, P=plen[b] if plen else 0,
                starts=docs[b] if docs else ())
            np.testing.assert_allclose(out[b, h], o_ref, rtol=0, atol=1e-13)
            assert abs(lse[b, h] - l_ref) < 1e-13


@pytest.mark.parametrize("case", MASK_CASES)
def test_further_masks_prefill_match_brute_force(case):
    kind, wph, plen, docs = case
    B, Hq, Hkv, d, bs = 2, 4, 2, 8, 4
    ctx, ql = [9, 22], [6, 19]
    gen = torch.Generator().manual_seed(8)
    q, kc, vc, tab, _, scale = tiny_case(8, B, Hq, Hkv, d, bs, 40,
                                         [c + n for c, n in zip(ctx, ql)], kind, 0)
    T = sum(ql)
    qp = torch.randn(T, Hq, d, generator=gen, dtype=torch.float64)
    kn = torch.randn(T, Hkv, d, generator=gen, dtype=torch.float64)
    vn = torch.randn(T, Hkv, d, generator=gen, dtype=torch.float64)
    off, flat = _docs_csr(docs) if docs else (None, None)
    out, lse = oracle.paged_prefill(qp, kn, vn, kc, vc, tab, ctx, ql, scale, kind, 0, None,
                                    window_per_head=wph, prefix_len=plen, doc_offsets=off,
                                    doc_starts=flat)
    kl, vl = kc.tolist(), vc.tolist()
    g = Hq // Hkv
    start = 0
    for b in range(B):
        for i in range(ql[b]):
            for h in range(Hq):
                ek = [kn[start + j, h // g].tolist() for j in range(ql[b])]
                ev = [vn[start + j, h // g].tolist() for j in range(ql[b])]
                o_ref, l_ref = brute_paged_attention(
                    qp[start + i, h].tolist(), kl, vl, tab[b].tolist(), ctx[b], ctx[b] + i,
                    h // g, scale, kind, wph[h] if wph else 0, ek, ev,
                    P=plen[b] if plen else 0, starts=docs[b] if docs else ())
                np.testing.assert_allclose(out[start + i, h], o_ref, rtol=0, atol=1e-13)
                assert abs(lse[start + i, h] - l_ref) < 1e-13
        start += ql[b]


def test_packed_documents_equal_separate_sequences():
    """A sequence packed from documents, under the document mask, gives for each
    query exactly causal attention over its own document alone (positions
    rebased), computed as a separate contiguous sequence."""
    gen = torch.Generator().manual_seed(4)
    Hq, Hkv, d = 4, 2, 16
    starts = [0, 7, 20, 21, 40]
    n = 52
    K = torch.randn(n, Hkv, d, generator=gen, dtype=torch.float64)
    V = torch.randn(n, Hkv, d, generator=gen, dtype=torch.float64)
    Qm = torch.randn(n, Hq, d, generator=gen, dtype=torch.float64)
    scale = 0.3
    # packed: the whole sequence as one chunk with no context (identity layout, bs 4)
    bs = 4
    kc = K.view(n // bs, bs, Hkv, d).permute(0, 2, 1, 3).contiguous()
    vc = V.view(n // bs, bs, Hkv, d).permute(0, 2, 1, 3).contiguous()
    tab = np.arange(n // bs)[None, :]
    out, lse = oracle.paged_prefill(Qm, K, V, kc, vc, tab, [0], [n], scale, A.MASK_DOCUMENT,
                                    doc_offsets=[0, len(starts)], doc_starts=starts)
    bounds = starts + [n]
    for s0, s1 in zip(bounds[:-1], bounds[1:]):
        for h in range(Hq):
            o_ref, l_ref = A.masked_attention(Qm[s0:s1, h], K[s0:s1, h // 2], V[s0:s1, h // 2],
                                              np.arange(s1 - s0), np.arange(s1 - s0), scale,
                                              A.MASK_CAUSAL, 0)
            np.testing.assert_allclose(out[s0:s1, h], o_ref, rtol=0, atol=1e-13)
            np.testing.assert_allclose(lse[s0:s1, h], l_ref, rtol=0, atol=1e-13)


def test_prefix_lm_limits():
    """prefix_len 0 is causal; a prefix covering every key is no mask."""
    q, kc, vc, tab, lens, scale = tiny_case(9, 2, 4, 2, 8, 4, 40, [20, 33], A.MASK_CAUSAL, 0)
    ctx, ql = [8, 12], [12, 21]
    gen = torch.Generator().manual_seed(9)
    qp = torch.randn(33, 4, 8, generator=gen, dtype=torch.float64)
    kn = torch.randn(33, 2, 8, generator=gen, dtype=torch.float64)
    vn = torch.randn(33, 2, 8, generator=gen, dtype=torch.float64)
    causal = oracle.paged_prefill(qp, kn, vn, kc, vc, tab, ctx, ql, scale, A.MASK_CAUSAL)
    p0 = oracle.paged_prefill(qp, kn, vn, kc, vc, tab, ctx, ql, scale, A.MASK_PREFIX_LM,
                              prefix_len=[0, 0])
    none = oracle.paged_prefill(qp, kn, vn, kc, vc, tab, ctx, ql, scale, A.MASK_NONE)
    full = oracle.paged_prefill(qp, kn, vn, kc, vc, tab, ctx, ql, scale, A.MASK_PREFIX_LM,
                                prefix_len=[20, 33])
    for a, b in ((causal, p0), (none, full)):
        np.testing.assert_array_equal(a[0], b[0])
        np.testing.assert_array_equal(a[1], b[1])


def test_per_head_windows_equal_one_window_per_call():
    q, kc, vc, tab, lens, scale = tiny_case(12, 3, 4, 2, 8, 4, 60, [5, 30, 47],
                                            A.MASK_SLIDING, 0)
    wph = [1, 9, 0, 30]
    out, lse = oracle.paged_decode(q, kc, vc, tab, lens, scale, A.MASK_SLIDING, 0,
                                   window_per_head=wph)
    for h, w in enumerate(wph):
        o1, l1 = oracle.paged_decode(q, kc, vc, tab, lens, scale, A.MASK_SLIDING, w)
        np.testing.assert_array_equal(out[:, h], o1[:, h])
        np.testing.assert_array_equal(lse[:, h], l1[:, h])


def _mut_prefix_inclusive(kind, q_pos, k_pos, window, prefix_len=0, doc_starts=None):
    q_pos, k_pos = np.asarray(q_pos), np.asarray(k_pos)
    return (k_pos <= q_pos) | (k_pos <= prefix_len)  # planted: prefix one key too long


def _mut_doc_start_in_previous(kind, q_pos, k_pos, window, prefix_len=0, doc_starts=None):
    q_pos, k_pos = np.asarray(q_pos), np.asarray(k_pos)
    st = np.sort(np.asarray(doc_starts))
    d = lambda p: np.searchsorted(st, p, side="left")  # planted: a start joins the previous doc
    return (k_pos <= q_pos) & (d(q_pos) == d(k_pos))


@pytest.mark.parametrize("mutation", ["prefix_inclusive", "doc_start_in_previous"])
def test_planted_mask_mistakes_are_caught(monkeypatch, mutation):
    kind = A.MASK_PREFIX_LM if mutation == "prefix_inclusive" else A.MASK_DOCUMENT
    plen, docs = [6, 30], [[0, 5, 9], [0, 17, 18, 30]]
    q, kc, vc, tab, lens, scale = tiny_case(31, 2, 4, 2, 8, 4, 40, [13, 38], kind, 0)
    off, flat = _docs_csr(docs)
    monkeypatch.setattr(A, "visible", _mut_prefix_inclusive if mutation == "prefix_inclusive"
                        else _mut_doc_start_in_previous)
    # decode queries see the whole prefix anyway: plant in a prefill
    ctx, ql = [9, 22], [4, 16]
    gen = torch.Generator().manual_seed(8)
    qp = torch.randn(20, 4, 8, generator=gen, dtype=torch.float64)
    kn = torch.randn(20, 2, 8, generator=gen, dtype=torch.float64)
    vn = torch.randn(20, 2, 8, generator=gen, dtype=torch.float64)
    out, lse = A.paged_prefill(qp, kn, vn, kc, vc, tab, ctx, ql, scale, kind, prefix_len=plen,
                               doc_offsets=off, doc_starts=flat)
    monkeypatch.undo()
    kl, vl = kc.tolist(), vc.tolist()
    worst, start = 0.0, 0
    for b in range(2):
        for i in range(ql[b]):
            for h in range(4):
                ek = [kn[start + j, h // 2].tolist() for j in range(ql[b])]
                ev = [vn[start + j, h // 2].tolist() for j in range(ql[b])]
                o_ref, l_ref = brute_paged_attention(
                    qp[start + i, h].tolist(), kl, vl, tab[b].tolist(), ctx[b], ctx[b] + i,
                    h // 2, scale, kind, 0, ek, ev, P=plen[b], starts=docs[b])
                worst = max(worst, float(np.max(np.abs(out[start + i, h] - o_ref))))
        start += ql[b]
    assert worst > 1e-6, f"mutation {mutation} went unnoticed"


@pytest.mark.parametrize("kind,w,wph", [(A.MASK_NONE, 0, None), (A.MASK_CAUSAL, 0, None),
                                        (A.MASK_SLIDING, 7, None),
                                        (A.MASK_SLIDING, 0, [3, 0, 9, 1])])
def test_prefill_tile_matches_brute_force(kind, w, wph):
    """The tile entry (a block of query rows of one sequence, some heads) is the
    same definition evaluated on a block: checked against the scalar brute
    force over tiles that start mid-sequence and one cut by the chunk end."""
    B, Hq, Hkv, d, bs = 2, 4, 2, 8, 4
    ctx, ql = [9, 22], [7, 13]
    gen = torch.Generator().manual_seed(17)
    q, kc, vc, tab, _, scale = tiny_case(17, B, Hq, Hkv, d, bs, 40,
                                         [c + n for c, n in zip(ctx, ql)], kind, w)
    T = sum(ql)
    qp = torch.randn(T, Hq, d, generator=gen, dtype=torch.float64)
    kn = torch.randn(T, Hkv, d, generator=gen, dtype=torch.float64)
    vn = torch.randn(T, Hkv, d, generator=gen, dtype=torch.float64)
    kl, vl = kc.tolist(), vc.tolist()
    g = Hq // Hkv
    starts = [0, ql[0]]
    for b, i0, i1, heads in [(0, 0, 7, None), (1, 4, 11, [3, 0]), (1, 10, 20, [1])]:
        out, lse = oracle.paged_prefill_tile(qp, kn, vn, kc, vc, tab, ctx, ql, scale, kind, b,
                                             i0, i1, heads=heads, window=w,
                                             window_per_head=wph)
        hs = list(range(Hq)) if heads is None else heads
        rows = range(i0, min(i1, ql[b]))
        assert out.shape == (len(rows), len(hs), d)
        for r, i in enumerate(rows):
            for j, h in enumerate(hs):
                s0 = starts[b]
                ek = [kn[s0 + t, h // g].tolist() for t in range(ql[b])]
                ev = [vn[s0 + t, h // g].tolist() for t in range(ql[b])]
                o_ref, l_ref = brute_paged_attention(
                    qp[s0 + i, h].tolist(), kl, vl, tab[b].tolist(), ctx[b], ctx[b] + i, h // g,
                    scale, kind, wph[h] if wph else w, ek, ev)
                np.testing.assert_allclose(out[r, j], o_ref, rtol=0, atol=1e-13)
                assert abs(lse[r, j] - l_ref) < 1e-13
