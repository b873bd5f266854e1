"""Pins of the E4M3 oracle (CPU): rounding against torch's float8_e4m3fn cast
(a separate implementation of the format), decoding of all 256 codes against
torch's reinterpretation, encode/decode round trips, saturation and the
relative error bound of the per-row quantisation."""

import numpy as np
import pytest
import torch

from oracle import fp8 as F


def test_round_matches_torch_cast():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.normal(0, 1, 20000), rng.normal(0, 100, 20000), rng.uniform(-448, 448, 20000),
        rng.uniform(-2 ** -6, 2 ** -6, 20000),            # subnormal range
        F.decode_e4m3(np.arange(256))[np.isfinite(F.decode_e4m3(np.arange(256)))],
    ]).astype(np.float32)
    # exact ties between neighbouring codes, both ways
    vals = np.unique(np.abs(F.decode_e4m3(np.arange(128))[:-1]))
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids])
    x = x[np.abs(x) <= 464]  # beyond, torch's cast gives NaN where the reading saturates
    ours = F.round_e4m3(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)


def test_saturation():
    x = np.array([448.0, 463.9, 464.0, 465.0, 1e6, -1e9], dtype=np.float32)
    assert np.array_equal(F.round_e4m3(x), [448, 448, 448, 448, 448, -448])


def test_decode_all_codes_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = F.decode_e4m3(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(ours[fin], ref[fin])


def test_encode_decode_round_trip():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF, 0x80)], dtype=np.uint8)
    assert np.array_equal(F.encode_e4m3(F.decode_e4m3(codes)), codes)


def test_row_quantisation_error_bound_and_scale():
    rng = np.random.default_rng(1)
    for scale in (1e-3, 1.0, 30.0):
        row = (rng.normal(0, scale, 128)).astype(np.float32)
        codes, s = F.quantize_row(row)
        assert s == np.float32(np.max(np.abs(row)) / np.float32(448))
        back = F.decode_e4m3(codes) * np.float64(s)
        big = np.abs(row) >= 2 ** -6 * s   # normal range of the scaled values
        rel = np.abs(back[big] - row[big]) / np.abs(row[big])
        assert rel.max() <= 2 ** -4 + 1e-12
        # the largest element maps to the largest code
        assert np.max(np.abs(F.decode_e4m3(codes))) == 448


def test_zero_row():
    codes, s = F.quantize_row(np.zeros(128, dtype=np.float32))
    assert s == 1.0 and not codes.any()


def test_vectorised_rows_equal_row_by_row():
    rng = np.random.default_rng(2)
    x = (rng.normal(0, 1, (50, 128)) * rng.uniform(0.01, 100, (50, 1))).astype(np.float32)
    x[3] = 0
    codes, s = F.quantize_rows(x)
    for i in range(50):
        c1, s1 = F.quantize_row(x[i])
        assert np.array_equal(codes[i], c1) and s[i] == s1
