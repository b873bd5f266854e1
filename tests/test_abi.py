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
