"""CPU: the rule the kernels use to skip and to leave unmasked whole tiles.

Each mask kind gives the query at position q one visible key interval
[lo(q), hi(q)) with both ends non-decreasing in q, so a tile of queries
[q0, q1] sees the union [lo(q0), hi(q1)) and, for every row, the
intersection [lo(q1), hi(q0)). This restates that rule in plain Python and
checks it against the oracle's pairwise visibility on ragged sequences,
documents, prefixes and per-head windows, for several tile shapes.
"""

import numpy as np
import pytest

import oracle
from paged_kv_cache_gather_b200 import inputs as I

CTX, QL = [0, 37, 300, 5], [200, 1, 129, 64]
WPS = np.array([0, 5, 40, 17])
WPH = np.array([1, 0, 33, 300])
PLEN = np.array([10, 50, 1000, 0])


def _starts():
    off, st = I.document_starts([c + q for c, q in zip(CTX, QL)], 3, mean_doc=40)
    return off.numpy(), st.numpy()


def interval(kind, b, h, q, n, per_head, off, st):
    if kind == I.MASK_NONE:
        return 0, n
    lo, hi = 0, q + 1
    if kind == I.MASK_SLIDING:
        w = WPH[h] if per_head else WPS[b]
        lo = max(0, q - w + 1) if w > 0 else 0
    elif kind == I.MASK_DOCUMENT:
        s = st[off[b]:off[b + 1]]
        s = s[s <= q]
        lo = int(s.max()) if len(s) else 0
    elif kind == I.MASK_PREFIX_LM:
        hi = max(hi, int(PLEN[b]))
    return lo, min(hi, n)


@pytest.mark.parametrize("kind,q_tile,k_tile", [(I.MASK_NONE, 128, 128), (I.MASK_CAUSAL, 7, 16),
                                                (I.MASK_SLIDING, 16, 16),
                                                (I.MASK_PREFIX_LM, 32, 16),
                                                (I.MASK_DOCUMENT, 64, 16),
                                                (I.MASK_DOCUMENT, 1, 1)])
@pytest.mark.parametrize("per_head", [False, True])
def test_interval_rule_classifies_tiles(kind, q_tile, k_tile, per_head):
    off, st = _starts()
    per_head = per_head and kind == I.MASK_SLIDING
    for b in range(len(CTX)):
        C, Q = CTX[b], QL[b]
        n = C + Q
        qpos = C + np.arange(Q)
        for h in range(4):
            w = WPH[h] if per_head else WPS[b]
            vis = oracle.visible(kind, qpos[:, None], np.arange(n)[None, :], w, PLEN[b],
                                 st[off[b]:off[b + 1]])
            for qt in range(-(-Q // q_tile)):
                q0 = C + qt * q_tile
                q1 = min(q0 + q_tile, n) - 1
                for kt in range(-(-n // k_tile)):
                    k0 = kt * k_tile
                    k1 = min(k0 + k_tile, n) - 1
                    t = vis[q0 - C:q1 - C + 1, k0:k1 + 1]
                    lo0, hi0 = interval(kind, b, h, q0, n, per_head, off, st)
                    lo1, hi1 = interval(kind, b, h, q1, n, per_head, off, st)
                    assert (k0 < hi1 and k1 >= lo0) == bool(t.any())
                    assert (k0 >= lo1 and k1 < hi0) == bool(t.all())
