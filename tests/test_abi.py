"""The C ABI library loads, exports every declared symbol and rejects bad
arguments on the host before any launch (CPU only: no call here reaches the
GPU)."""

import ctypes
import os
import re

import pytest

from paged_kv_cache_gather_b200 import _lib as L
from paged_kv_cache_gather_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.lib()


def header_symbols():
    text = open(os.path.join(ROOT, "include", "pagedkv.h")).read()
    return sorted(set(re.findall(r"PKV_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)))


def test_header_lists_the_exports():
    assert header_symbols() == sorted(L.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    for name in header_symbols():
        assert hasattr(lib, name), name
    assert lib.pkv_version() == 1


def test_internal_symbols_are_hidden():
    out = os.popen(f"nm -D --defined-only {L.LIB_PATH}").read()
    names = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert names == set(L.EXPORTS)


def test_status_strings(lib):
    assert lib.pkv_status_string(0) == b"PKV_OK"
    assert lib.pkv_status_string(-4) == b"PKV_ERR_WORKSPACE_TOO_SMALL"
    assert lib.pkv_status_string(-99) == b"PKV_ERR_UNKNOWN"


FAKE = ctypes.c_void_p(0x10000)  # 16-byte aligned, never dereferenced: calls fail first


def desc(nb=8, bs=16, h=2, d=128, dt=L.PKV_BF16):
    return L.CacheDescC(nb, bs, h, d, dt)


def mask(kind=0, w=0):
    return L.MaskModC(kind, w, None)


def decode(lib, c=None, m=None, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, c=c or desc(), t=FAKE, mb=4, lens=FAKE, B=2, Hq=8,
             scale=0.1, m=m or mask(), out=FAKE, lse=FAKE, ws=FAKE, wsb=1 << 30, dbg=None,
             s=None)
    a.update(kw)
    st = lib.paged_attention_decode(a["q"], a["k"], a["v"], a["c"], a["t"], a["mb"], a["lens"],
                                    a["B"], a["Hq"], a["scale"], a["m"], a["out"], a["lse"],
                                    a["ws"], a["wsb"], a["dbg"], a["s"])
    return st, lib.pkv_last_error().decode()


def test_decode_argument_checks(lib):
    assert decode(lib, c=desc(bs=12))[0] == L.PKV_ERR_INVALID_ARG
    assert "power of two" in decode(lib, c=desc(bs=12))[1]
    assert decode(lib, c=desc(dt=7))[0] == L.PKV_ERR_UNSUPPORTED
    assert decode(lib, c=desc(d=6, dt=L.PKV_BF16))[0] == L.PKV_ERR_UNSUPPORTED
    assert decode(lib, Hq=7)[0] == L.PKV_ERR_INVALID_ARG
    assert decode(lib, m=mask(kind=9))[0] == L.PKV_ERR_INVALID_ARG
    assert decode(lib, q=None)[0] == L.PKV_ERR_INVALID_ARG
    assert decode(lib, out=ctypes.c_void_p(0x10008))[0] == L.PKV_ERR_INVALID_ARG
    assert decode(lib, scale=float("nan"))[0] == L.PKV_ERR_INVALID_ARG
    assert decode(lib, B=-1)[0] == L.PKV_ERR_INVALID_ARG
    assert decode(lib, mb=0)[0] == L.PKV_ERR_INVALID_ARG
    assert decode(lib, c=desc(nb=1 << 20, bs=256, h=16))[0] == L.PKV_ERR_UNSUPPORTED
    assert decode(lib, B=0)[0] == L.PKV_OK  # nothing to do, nothing launched
    st, msg = decode(lib, wsb=16)
    assert st == L.PKV_ERR_WORKSPACE_TOO_SMALL and "workspace" in msg


def test_append_and_gather_argument_checks(lib):
    st = lib.paged_kv_append(FAKE, FAKE, FAKE, 3, FAKE, None, desc(), None, None)
    assert st == L.PKV_ERR_INVALID_ARG
    st = lib.paged_kv_append(FAKE, FAKE, FAKE, -1, FAKE, FAKE, desc(), None, None)
    assert st == L.PKV_ERR_INVALID_ARG
    assert lib.paged_kv_append(FAKE, FAKE, FAKE, 0, FAKE, FAKE, desc(), None, None) == L.PKV_OK
    st = lib.paged_kv_append(ctypes.c_void_p(0x10004), FAKE, FAKE, 2, FAKE, FAKE, desc(), None,
                             None)
    assert st == L.PKV_ERR_INVALID_ARG
    st = lib.paged_kv_gather(FAKE, FAKE, desc(bs=3), FAKE, 4, FAKE, 1, 16, FAKE, FAKE, None,
                             None)
    assert st == L.PKV_ERR_INVALID_ARG
    st = lib.paged_kv_gather(FAKE, FAKE, desc(), FAKE, 0, FAKE, 1, 16, FAKE, FAKE, None, None)
    assert st == L.PKV_ERR_INVALID_ARG


def test_prefill_argument_checks(lib):
    def call(**kw):
        a = dict(c=desc(), mb=4, B=2, T=10, Hq=8, scale=0.0, m=mask(1), out=FAKE)
        a.update(kw)
        return lib.paged_attention_prefill(FAKE, FAKE, FAKE, FAKE, FAKE, a["c"], FAKE, a["mb"],
                                           FAKE, FAKE, a["B"], a["T"], a["Hq"], a["scale"],
                                           a["m"], a["out"], FAKE, None, None)
    assert call(Hq=3) == L.PKV_ERR_INVALID_ARG
    assert call(out=None) == L.PKV_ERR_INVALID_ARG
    assert call(T=-2) == L.PKV_ERR_INVALID_ARG
    assert call(T=0) == L.PKV_OK
    assert call(m=mask(5)) == L.PKV_ERR_INVALID_ARG


def test_workspace_size_is_zero_for_fp32_and_positive_for_bf16(lib):
    assert lib.paged_attention_decode_workspace_size(4, 8, desc(dt=L.PKV_F32, d=64)) == 0
    assert lib.paged_attention_decode_workspace_size(4, 8, desc()) > 0
    assert lib.paged_attention_decode_workspace_size(4, 7, desc()) == 0


E4M3 = getattr(L, "PKV_FP8_E4M3", 2)


def test_fp8_argument_checks(lib):
    fp8 = desc(dt=E4M3)

    def dec(c=fp8, ks=FAKE, vs=FAKE, **kw):
        a = dict(B=2, Hq=8, out=FAKE, m=mask())
        a.update(kw)
        return lib.paged_attention_decode_fp8(FAKE, FAKE, FAKE, ks, vs, c, FAKE, 4, FAKE, a["B"],
                                              a["Hq"], 0.1, a["m"], a["out"], FAKE, FAKE,
                                              1 << 30, None, None)
    assert dec(c=desc()) == L.PKV_ERR_INVALID_ARG            # not an E4M3 pool
    assert dec(ks=None) == L.PKV_ERR_INVALID_ARG             # E4M3 needs the row scales
    assert dec(out=None) == L.PKV_ERR_INVALID_ARG
    assert dec(Hq=7) == L.PKV_ERR_INVALID_ARG
    assert dec(B=0) == L.PKV_OK
    # plain decode refuses row scales; the E4M3 append refuses other pools
    st = lib.paged_attention_decode(FAKE, FAKE, FAKE, fp8, FAKE, 4, FAKE, 2, 8, 0.1, mask(),
                                    FAKE, FAKE, FAKE, 1 << 30, None, None)
    assert st == L.PKV_ERR_INVALID_ARG
    assert lib.paged_kv_append_fp8(FAKE, FAKE, FAKE, 2, FAKE, FAKE, FAKE, FAKE, desc(), None,
                                   None) == L.PKV_ERR_UNSUPPORTED
    assert lib.paged_kv_append_fp8(FAKE, FAKE, FAKE, 2, FAKE, FAKE, FAKE, FAKE,
                                   desc(dt=E4M3, d=64), None, None) == L.PKV_ERR_UNSUPPORTED
    assert lib.paged_kv_append_fp8(FAKE, FAKE, FAKE, 2, FAKE, FAKE, None, FAKE, fp8, None,
                                   None) == L.PKV_ERR_INVALID_ARG
    assert lib.paged_kv_append_fp8(FAKE, FAKE, FAKE, 0, FAKE, FAKE, FAKE, FAKE, fp8, None,
                                   None) == L.PKV_OK
    # E4M3 pools are refused where their row scales would have to move
    assert lib.paged_kv_append(FAKE, FAKE, FAKE, 2, FAKE, FAKE, fp8, None,
                               None) == L.PKV_ERR_UNSUPPORTED
    assert lib.paged_kv_copy_blocks(FAKE, FAKE, fp8, FAKE, 1, None,
                                    None) == L.PKV_ERR_UNSUPPORTED


def test_copy_blocks_argument_checks(lib):
    assert lib.paged_kv_copy_blocks(FAKE, FAKE, desc(), FAKE, -1, None,
                                    None) == L.PKV_ERR_INVALID_ARG
    assert lib.paged_kv_copy_blocks(FAKE, FAKE, desc(), None, 2, None,
                                    None) == L.PKV_ERR_INVALID_ARG
    assert lib.paged_kv_copy_blocks(ctypes.c_void_p(0x10004), FAKE, desc(), FAKE, 2, None,
                                    None) == L.PKV_ERR_INVALID_ARG
    assert lib.paged_kv_copy_blocks(FAKE, FAKE, desc(), FAKE, 0, None, None) == L.PKV_OK


def test_shared_prefix_argument_checks(lib):
    def call(c=None, m=None, **kw):
        a = dict(B=8, Hq=16, groups=2, gmax=4, out=FAKE, scale=0.1, ws=1 << 30)
        a.update(kw)
        return lib.paged_attention_decode_shared_prefix(
            FAKE, FAKE, FAKE, c or desc(), FAKE, 4, FAKE, a["B"], a["Hq"], a["scale"],
            m or mask(1), FAKE, a["groups"], a["gmax"], FAKE, a["out"], FAKE, FAKE, a["ws"],
            None, None)
    assert call(c=desc(d=64)) == L.PKV_ERR_UNSUPPORTED         # bf16, head_dim 128 only
    assert call(c=desc(bs=4)) == L.PKV_ERR_UNSUPPORTED         # block_size >= 8
    assert call(m=mask(2, 64)) == L.PKV_ERR_UNSUPPORTED        # no sliding window
    assert call(Hq=7) == L.PKV_ERR_INVALID_ARG
    assert call(Hq=2 * 33) == L.PKV_ERR_UNSUPPORTED            # > 32 query heads per KV head
    assert call(scale=float("nan")) == L.PKV_ERR_INVALID_ARG
    assert call(groups=0) == L.PKV_ERR_INVALID_ARG
    assert call(groups=9) == L.PKV_ERR_INVALID_ARG             # more groups than sequences
    assert call(Hq=2 * 32, gmax=8) == L.PKV_ERR_UNSUPPORTED    # group rows beyond 128
    assert call(out=None) == L.PKV_ERR_INVALID_ARG
    assert call(ws=16) == L.PKV_ERR_WORKSPACE_TOO_SMALL
    assert call(B=0) == L.PKV_OK
    assert lib.paged_attention_decode_shared_prefix_workspace_size(8, 16, desc()) > 0


def test_block_mask_and_reserve_argument_checks(lib):
    def bm(**kw):
        a = dict(B=2, Hq=8, qt=128, kt=128, nq=4, nk=4, out=FAKE, m=mask(1))
        a.update(kw)
        return lib.paged_attention_block_mask(FAKE, FAKE, a["B"], a["Hq"], a["m"], a["qt"],
                                              a["kt"], a["nq"], a["nk"], a["out"], None)
    assert bm(qt=0) == L.PKV_ERR_INVALID_ARG
    assert bm(B=-1) == L.PKV_ERR_INVALID_ARG
    assert bm(out=None) == L.PKV_ERR_INVALID_ARG
    assert bm(m=mask(7)) == L.PKV_ERR_INVALID_ARG
    assert bm(nq=0) == L.PKV_OK

    def rs(c=None, **kw):
        a = dict(B=4, T=4, mb=8, stack=FAKE)
        a.update(kw)
        return lib.paged_kv_reserve_slots(FAKE, FAKE, c or desc(), FAKE, a["mb"], FAKE, FAKE,
                                          a["B"], a["stack"], FAKE, FAKE, FAKE, FAKE, a["T"],
                                          FAKE, None, None)
    assert rs(c=desc(dt=E4M3)) == L.PKV_ERR_UNSUPPORTED
    assert rs(T=-1) == L.PKV_ERR_INVALID_ARG
    assert rs(mb=0) == L.PKV_ERR_INVALID_ARG
    assert rs(B=8193) == L.PKV_ERR_UNSUPPORTED
    assert rs(stack=None) == L.PKV_ERR_INVALID_ARG
    assert rs(B=0) == L.PKV_OK
    assert lib.paged_kv_reserve_scratch_size(desc()) > 0


def test_debug_entries_reject_bad_arguments(lib):
    assert lib.pkv_debug_wait_timeout(None, None, None) == L.PKV_ERR_INVALID_ARG


def noalloc(lib, B, c=None, Hq=32, q=None):
    return lib.paged_attention_decode_noalloc(q, FAKE, FAKE, c or desc(h=8), FAKE, 4, FAKE, B, Hq,
                                              0.1, mask(), FAKE, FAKE, None, None)


def test_noalloc_scratch_boundary(lib):
    """The no-allocation decode accepts exactly the problems whose scratch
    need (the regular call's workspace size) fits its fixed array: at the
    largest such batch the size check passes (the call then fails later, on
    the null query, never with WORKSPACE_TOO_SMALL); one sequence more is
    rejected by the size check. Sizes are computed for a 148-SM B200, the
    library's count when no device is visible."""
    c = desc(h=8)  # 32 query heads / 8 KV heads, head_dim 128: group 4
    size = lambda b: lib.paged_attention_decode_workspace_size(b, 32, c)
    cap = L.PKV_NOALLOC_SCRATCH_BYTES
    lo, hi = 0, 1 << 24  # size(lo) <= cap < size(hi)
    assert size(lo) <= cap < size(hi)
    while hi - lo > 1:
        mid = (lo + hi) // 2
        lo, hi = (mid, hi) if size(mid) <= cap else (lo, mid)
    assert size(lo) <= cap < size(lo + 1)
    assert lo > 100_000  # the fixed part (per-worker partials) leaves room for a big batch
    assert noalloc(lib, lo) not in (L.PKV_OK, L.PKV_ERR_WORKSPACE_TOO_SMALL)
    assert noalloc(lib, lo + 1) == L.PKV_ERR_WORKSPACE_TOO_SMALL
    assert b"built-in scratch" in lib.pkv_last_error()


def test_noalloc_rejects_a_negative_batch_like_the_regular_call(lib):
    assert noalloc(lib, -5) == L.PKV_ERR_INVALID_ARG
    assert decode(lib, B=-5)[0] == L.PKV_ERR_INVALID_ARG
    assert lib.paged_attention_decode_workspace_size(-5, 32, desc(h=8)) == 0


def test_fp8_copy_and_reserve_argument_checks(lib):
    fp8 = desc(dt=E4M3)

    def cp(c=fp8, ks=FAKE, n=2, pairs=FAKE):
        return lib.paged_kv_copy_blocks_fp8(FAKE, FAKE, ks, FAKE, c, pairs, n, None, None)
    assert cp(c=desc()) == L.PKV_ERR_UNSUPPORTED                    # bf16 pools: plain copy
    assert cp(c=desc(dt=E4M3, bs=2, h=1)) == L.PKV_ERR_UNSUPPORTED  # scale spans of 8 bytes
    assert cp(n=-1) == L.PKV_ERR_INVALID_ARG
    assert cp(ks=None) == L.PKV_ERR_INVALID_ARG
    assert cp(pairs=None) == L.PKV_ERR_INVALID_ARG
    assert cp(ks=ctypes.c_void_p(0x10004)) == L.PKV_ERR_INVALID_ARG
    assert cp(n=0) == L.PKV_OK

    def rs(c=fp8, ks=FAKE, B=4):
        return lib.paged_kv_reserve_slots_fp8(FAKE, FAKE, ks, FAKE, c, FAKE, 8, FAKE, FAKE, B,
                                              FAKE, FAKE, FAKE, FAKE, FAKE, 4, FAKE, None, None)
    assert rs(c=desc()) == L.PKV_ERR_UNSUPPORTED
    assert rs(ks=None) == L.PKV_ERR_INVALID_ARG
    assert rs(B=8193) == L.PKV_ERR_UNSUPPORTED
    assert rs(B=0) == L.PKV_OK
