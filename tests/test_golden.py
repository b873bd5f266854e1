"""The oracle against a worked example whose answers are derived by hand
(tests/golden/paged_attention_worked_example.json, with its citation and
derivation): decode under no mask, causal and two sliding windows, a chunked
prefill with one context token, an append and a gather, all through a block
table that scatters the sequence over the pool, with a sentinel in every row
that must not be read."""

import numpy as np
import pytest

import oracle
from golden_case import array, load, value

MASKS = {"none": oracle.MASK_NONE, "causal": oracle.MASK_CAUSAL, "sliding": oracle.MASK_SLIDING}


@pytest.fixture(scope="module")
def golden():
    return load()


def test_decode_cases(golden):
    g, k, v = golden
    d = g["decode"]
    q = array(d["q"]).reshape(1, 1, -1)
    tables = np.array([g["block_table"]], dtype=np.int32)
    lens = np.array([d["seq_len"]], dtype=np.int32)
    for c in d["cases"]:
        out, lse = oracle.paged_decode(q, k, v, tables, lens, d["scale"], MASKS[c["mask"]],
                                       window=c["window"])
        assert np.allclose(out[0, 0], array(c["out"]), rtol=0, atol=1e-12), c
        assert abs(lse[0, 0] - value(c["lse"])) < 1e-12, c


def test_prefill(golden):
    g, k, v = golden
    p = g["prefill"]
    q = array(p["q"])[:, None, :]
    kn = array(p["k_new"])[:, None, :]
    vn = array(p["v_new"])[:, None, :]
    tables = np.array([g["block_table"]], dtype=np.int32)
    out, lse = oracle.paged_prefill(q, kn, vn, k, v, tables, np.array([p["ctx_len"]]),
                                    np.array([q.shape[0]]), p["scale"], MASKS[p["mask"]])
    assert np.allclose(out[:, 0], array(p["out"]), rtol=0, atol=1e-12)
    assert np.allclose(lse[:, 0], array(p["lse"]), rtol=0, atol=1e-12)


def test_append_slot_and_untouched_rows(golden):
    g, k, v = golden
    a = g["append"]
    bs = g["block_size"]
    pos = a["seq_len_after"] - 1
    slot = g["block_table"][pos // bs] * bs + pos % bs
    assert slot == a["slot"]
    kn = array(a["k"]).reshape(1, 1, -1)
    vn = array(a["v"]).reshape(1, 1, -1)
    k2, v2 = oracle.kv_append(kn, vn, np.array([slot]), k, v)
    ek, ev = k.copy(), v.copy()
    ek[a["block"], :, a["row"], :] = kn[0]
    ev[a["block"], :, a["row"], :] = vn[0]
    assert np.array_equal(k2, ek) and np.array_equal(v2, ev)


def test_gather(golden):
    g, k, v = golden
    tables = np.array([g["block_table"]], dtype=np.int32)
    lens = np.array([g["decode"]["seq_len"]], dtype=np.int32)
    ko, vo = oracle.kv_gather(k, v, tables, lens, g["gather"]["out_max_len"])
    assert np.array_equal(ko[0, 0], array(g["gather"]["k"]))
    assert np.array_equal(vo[0, 0], array(g["gather"]["v"]))


def test_a_wrong_table_index_is_caught(golden):
    # reading the table transposed (block 0 first) must break the example
    g, k, v = golden
    d = g["decode"]
    q = array(d["q"]).reshape(1, 1, -1)
    lens = np.array([d["seq_len"]], dtype=np.int32)
    out, _ = oracle.paged_decode(q, k, v, np.array([g["block_table"][::-1]], dtype=np.int32),
                                 lens, d["scale"], oracle.MASK_NONE)
    assert not np.allclose(out[0, 0], array(d["cases"][0]["out"]), atol=1e-3)
