"""Float8 (E4M3) KV pools, written out from the format's definition.

TEST INFRASTRUCTURE ONLY (same rules as ``attention64``).

The pages only gesture at compressing the KV cache ("Ultimate Guide to
PagedAttention" and the FlexAttention page mention memory savings, not a
method), so the quantisation is a reading, stated here and kept plain:

* Each stored row (one token's K or V for one KV head, ``head_dim`` values)
  gets its own float32 scale ``s = amax / 448`` (448 is the largest finite
  E4M3 value; ``s = 1`` for an all-zero row), computed in float32.
* A value x is stored as the E4M3 code of ``x / s`` (float32 division),
  rounded to nearest with ties to even and saturated to +-448.
* It reads back as ``decode(code) * s``.

E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 holds
the subnormals ``m * 2**-9``; code 0x7F / 0xFF is NaN (there is no infinity).

Pins (``tests/test_oracle_fp8.py``): rounding against torch's float8_e4m3fn
cast over normals, subnormals and ties; decode against torch's reinterpretation
of all 256 codes; encode(decode(c)) == c; the relative error bound 2**-4.
``kv_append_fp8`` and ``dequantize_pool`` (``tests/test_oracle_fp8_placement.py``):
a worked example with hand-derived codes, scales and read-back values
(``tests/golden/e4m3_append_example.json``), a scalar brute force of the
placement (block ``slot // bs``, row ``slot % bs``, every KV head) and of the
read-back, and planted mistakes (head swapped, block and row swapped, one
pool's scales for both, a scale per block, the scale on the wrong axis).
"""

import numpy as np

E4M3_MAX = 448.0


def _f64(x):
    if hasattr(x, "detach"):
        import torch

        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def round_e4m3(x):
    """Nearest E4M3 value of each element (ties to even), saturated to +-448."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    mant, ex = np.frexp(a)              # a = mant * 2**ex, mant in [0.5, 1)
    e = np.maximum(ex - 1, -6)          # binade [2**e, 2**(e+1)); subnormals share 2**-6's spacing
    ulp = np.ldexp(1.0, (e - 3).astype(np.int64))
    r = np.round(a / ulp) * ulp         # half to even on an exact quotient
    r = np.minimum(r, E4M3_MAX)
    return np.where(x < 0, -r, r)


def decode_e4m3(codes):
    """Values of E4M3 codes (uint8); NaN for 0x7F and 0xFF."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    v = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, (e - 7)))
    v = np.where((e == 15) & (m == 7), np.nan, v)
    return sign * v


def encode_e4m3(values):
    """E4M3 codes (uint8) of values that are exactly representable (finite)."""
    v = np.asarray(values, dtype=np.float64)
    a = np.abs(v)
    sign = np.where(np.signbit(v), 0x80, 0)
    mant, ex = np.frexp(a)
    e = ex - 1 + 7                      # biased exponent of a normal value
    normal = a >= 2.0 ** -6
    m_norm = np.round((a / np.ldexp(1.0, np.where(normal, ex - 1, 0)) - 1.0) * 8.0)
    m_sub = np.round(a / 2.0 ** -9)
    code = np.where(normal, (np.clip(e, 0, 15) << 3) | m_norm.astype(np.int64),
                    m_sub.astype(np.int64))
    return (sign | code).astype(np.uint8)


def row_scale(row):
    """float32 scale of one stored row: amax / 448 in float32 (1 for a zero row)."""
    r = np.asarray(_f64(row), dtype=np.float32)
    amax = np.float32(np.max(np.abs(r))) if r.size else np.float32(0)
    if amax == 0:
        return np.float32(1.0)
    return np.float32(amax / np.float32(E4M3_MAX))


def quantize_row(row):
    """(codes uint8 [d], scale float32) of one row."""
    r = np.asarray(_f64(row), dtype=np.float32)
    s = row_scale(r)
    q = round_e4m3((r / s).astype(np.float32))
    return encode_e4m3(q), s


def kv_append_fp8(k, v, slot_mapping, k_codes, v_codes, k_scale, v_scale):
    """Expected E4M3 pools and scales after appending bf16 tokens (copies).

    k, v: [T, Hkv, d]; pools uint8 [NB, Hkv, bs, d]; scales float32
    [NB, Hkv, bs]. Token t (slot >= 0) writes its quantised rows and their
    scales at block ``slot // bs``, row ``slot % bs``, for every KV head.
    """
    kc = np.array(k_codes, dtype=np.uint8, copy=True)
    vc = np.array(v_codes, dtype=np.uint8, copy=True)
    ks = np.array(k_scale, dtype=np.float32, copy=True)
    vs = np.array(v_scale, dtype=np.float32, copy=True)
    kf, vf = _f64(k), _f64(v)
    bs = kc.shape[2]
    slots = np.asarray(slot_mapping.cpu() if hasattr(slot_mapping, "cpu") else slot_mapping,
                       dtype=np.int64)
    for t, slot in enumerate(slots):
        if slot < 0:
            continue
        for h in range(kc.shape[1]):
            kc[slot // bs, h, slot % bs], ks[slot // bs, h, slot % bs] = quantize_row(kf[t, h])
            vc[slot // bs, h, slot % bs], vs[slot // bs, h, slot % bs] = quantize_row(vf[t, h])
    return kc, vc, ks, vs


def dequantize_pool(codes, scales):
    """float64 values of an E4M3 pool: decode(code) * scale of its row."""
    return decode_e4m3(codes) * np.asarray(scales, dtype=np.float64)[..., None]


def quantize_rows(x):
    """Vectorised ``quantize_row`` over the last axis: (codes uint8, scales float32)."""
    xf = np.asarray(_f64(x), dtype=np.float32)
    amax = np.max(np.abs(xf), axis=-1)
    s = np.where(amax > 0, (amax / np.float32(E4M3_MAX)).astype(np.float32),
                 np.float32(1.0)).astype(np.float32)
    q = round_e4m3((xf / s[..., None]).astype(np.float32))
    return encode_e4m3(q), s
