"""Pins of the E4M3 pool oracle's placement and read-back (CPU).

``oracle.fp8.kv_append_fp8`` and ``oracle.fp8.dequantize_pool`` are the
checkers of the library's E4M3 append and E4M3 decode. They are pinned here by
things other than themselves:

* a worked example with hand-derived codes, scales and read-back values
  (``tests/golden/e4m3_append_example.json``: rounding up, ties to even in the
  normal and the subnormal range, saturation at 448, skipped padding slots,
  untouched sentinel rows);
* a scalar brute force that places each (token, KV head) row by the
  block-table rule of "Ultimate Guide to PagedAttention" (block-table and
  dynamic-growth sections: slot s lands in block s // block_size, row
  s % block_size) and quantises it with torch's float8_e4m3fn cast, a separate
  implementation of the format;
* planted mistakes (head swapped, block and row swapped, one pool's scales
  used for both, a scale per block instead of per row, the scale broadcast over
  the wrong axis) that the same checks must reject.
"""

import json
import os
from fractions import Fraction

import numpy as np
import torch

from oracle import fp8 as F

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden", "e4m3_append_example.json")


def frac(x):
    return float(Fraction(x))


def load_golden():
    with open(GOLDEN) as f:
        g = json.load(f)
    rows = {k: np.array([frac(x) for x in v]) for k, v in g["rows"].items()}
    T, H, d = len(g["tokens"]), g["num_kv_heads"], g["head_dim"]
    k = np.zeros((T, H, d), dtype=np.float32)
    v = np.zeros((T, H, d), dtype=np.float32)
    for t, tok in enumerate(g["tokens"]):
        for h in range(H):
            name, times = tok["k"][h]
            k[t, h] = rows[name] * frac(times)
            name, times = tok["v"][h]
            v[t, h] = rows[name] * frac(times)
    # every input value is exact in bf16, as the library's inputs are
    for x in (k, v):
        xt = torch.from_numpy(x)
        assert torch.equal(xt.to(torch.bfloat16).float(), xt)
    slots = np.array([tok["slot"] for tok in g["tokens"]], dtype=np.int64)
    return g, k, v, slots


def sentinel_pools(g):
    shape = (g["num_blocks"], g["num_kv_heads"], g["block_size"], g["head_dim"])
    codes = np.full(shape, g["sentinel_code"], dtype=np.uint8)
    scales = np.full(shape[:3], g["sentinel_scale"], dtype=np.float32)
    return codes, codes.copy(), scales, scales.copy()


def test_worked_example_codes_scales_and_untouched_rows():
    g, k, v, slots = load_golden()
    kc0, vc0, ks0, vs0 = sentinel_pools(g)
    kc, vc, ks, vs = F.kv_append_fp8(k, v, slots, kc0, vc0, ks0, vs0)
    pools = {"k": (kc, ks), "v": (vc, vs)}
    written = {"k": np.zeros(ks.shape, bool), "v": np.zeros(vs.shape, bool)}
    for e in g["expected"]:
        codes, scales = pools[e["pool"]]
        at = (e["block"], e["head"], e["row"])
        want = np.array([int(c, 16) for c in g["codes"][e["row_of"]]], dtype=np.uint8)
        assert np.array_equal(codes[at], want), e
        assert scales[at] == np.float32(frac(g["scale"][e["row_of"]]) * frac(e["times"])), e
        back = F.dequantize_pool(codes, scales)[at]
        deq = np.array([frac(x) for x in g["dequantized"][e["row_of"]]]) * frac(e["times"])
        assert np.array_equal(back, deq), e
        written[e["pool"]][at] = True
    for name, (codes, scales) in pools.items():
        keep = ~written[name]
        assert np.all(codes[keep] == g["sentinel_code"]), name
        assert np.all(scales[keep] == g["sentinel_scale"]), name
    # the inputs were not modified
    assert np.all(kc0 == g["sentinel_code"]) and np.all(ks0 == g["sentinel_scale"])


# ---------------------------------------------------------------- brute force

NB, H, BS, D = 7, 3, 4, 16


def random_case(seed):
    rng = np.random.default_rng(seed)
    T = 12
    slots = rng.permutation(NB * BS)[:T].astype(np.int64)
    slots[[2, 7]] = -1                                   # padding tokens
    mag = rng.uniform(0.01, 50.0, (2, T, H, 1))
    x = (rng.normal(0, 1, (2, T, H, D)) * mag).astype(np.float32)
    x = torch.from_numpy(x).to(torch.bfloat16).float().numpy()  # bf16 inputs
    k, v = x[0], x[1]
    kc0 = rng.integers(0, 256, (NB, H, BS, D)).astype(np.uint8)
    vc0 = rng.integers(0, 256, (NB, H, BS, D)).astype(np.uint8)
    ks0 = rng.uniform(-3, -1, (NB, H, BS)).astype(np.float32)
    vs0 = rng.uniform(-3, -1, (NB, H, BS)).astype(np.float32)
    return k, v, slots, kc0, vc0, ks0, vs0


def torch_row(row):
    """(codes, scale) of one row by torch's float8_e4m3fn cast."""
    r = torch.from_numpy(np.ascontiguousarray(row, dtype=np.float32))
    s = r.abs().max() / torch.tensor(448.0)
    if float(s) == 0.0:
        s = torch.tensor(1.0)
    codes = (r / s).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return codes, np.float32(s)


def brute_force_append(k, v, slots, kc0, vc0, ks0, vs0):
    kc, vc, ks, vs = kc0.copy(), vc0.copy(), ks0.copy(), vs0.copy()
    for t in range(len(slots)):
        s = int(slots[t])
        if s < 0:
            continue
        blk, row = s // BS, s % BS
        for h in range(H):
            kc[blk, h, row], ks[blk, h, row] = torch_row(k[t, h])
            vc[blk, h, row], vs[blk, h, row] = torch_row(v[t, h])
    return kc, vc, ks, vs


def append_ok(fn, seeds=(0, 1, 2)):
    for seed in seeds:
        case = random_case(seed)
        got = fn(*case)
        want = brute_force_append(*case)
        if not all(np.array_equal(a, b) for a, b in zip(got, want)):
            return False
    return True


def brute_force_dequantize(codes, scales):
    vals = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double().numpy()
    out = np.empty(codes.shape, dtype=np.float64)
    for b in range(codes.shape[0]):
        for h in range(codes.shape[1]):
            for r in range(codes.shape[2]):
                for c in range(codes.shape[3]):
                    out[b, h, r, c] = vals[b, h, r, c] * float(scales[b, h, r])
    return out


def dequantize_ok(fn):
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 256, (NB, H, BS, D)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x11                  # no NaN codes
    scales = rng.uniform(0.001, 2.0, (NB, H, BS)).astype(np.float32)
    return np.array_equal(fn(codes, scales), brute_force_dequantize(codes, scales))


def test_append_matches_scalar_brute_force():
    assert append_ok(F.kv_append_fp8)


def test_dequantize_matches_scalar_brute_force():
    assert dequantize_ok(F.dequantize_pool)


# planted mistakes: each copy of the placement gets one plausible error


def _append_with(place):
    def fn(k, v, slots, kc0, vc0, ks0, vs0):
        kc, vc, ks, vs = kc0.copy(), vc0.copy(), ks0.copy(), vs0.copy()
        for t, s in enumerate(slots):
            if s < 0:
                continue
            for h in range(H):
                place(kc, vc, ks, vs, k, v, t, int(s), h)
        return kc, vc, ks, vs
    return fn


def _head_swapped(kc, vc, ks, vs, k, v, t, s, h):
    hh = H - 1 - h
    kc[s // BS, hh, s % BS], ks[s // BS, hh, s % BS] = F.quantize_row(k[t, h])
    vc[s // BS, hh, s % BS], vs[s // BS, hh, s % BS] = F.quantize_row(v[t, h])


def _block_row_swapped(kc, vc, ks, vs, k, v, t, s, h):
    blk, row = s % NB, (s // NB) % BS
    kc[blk, h, row], ks[blk, h, row] = F.quantize_row(k[t, h])
    vc[blk, h, row], vs[blk, h, row] = F.quantize_row(v[t, h])


def _k_scale_for_both(kc, vc, ks, vs, k, v, t, s, h):
    kc[s // BS, h, s % BS], ks[s // BS, h, s % BS] = F.quantize_row(k[t, h])
    vc[s // BS, h, s % BS], _ = F.quantize_row(v[t, h])
    vs[s // BS, h, s % BS] = ks[s // BS, h, s % BS]


def _scale_per_block(kc, vc, ks, vs, k, v, t, s, h):
    kc[s // BS, h, s % BS], ks[s // BS, h, :] = F.quantize_row(k[t, h])
    vc[s // BS, h, s % BS], vs[s // BS, h, :] = F.quantize_row(v[t, h])


def test_planted_placement_mistakes_are_caught():
    for place in (_head_swapped, _block_row_swapped, _k_scale_for_both, _scale_per_block):
        assert not append_ok(_append_with(place)), place.__name__


def test_planted_read_back_mistakes_are_caught():
    def heads_transposed(codes, scales):
        return F.decode_e4m3(codes) * np.asarray(scales, np.float64)[:, ::-1, :, None]

    def block_scale(codes, scales):
        return F.decode_e4m3(codes) * np.asarray(scales, np.float64)[:, :, :1, None]

    def wrong_axis(codes, scales):
        s = np.asarray(scales, np.float64)               # scale of row c used for column c
        return F.decode_e4m3(codes) * np.resize(s, codes.shape[:2] + (1, codes.shape[3]))

    for fn in (heads_transposed, block_scale, wrong_axis):
        assert not dequantize_ok(fn), fn.__name__
