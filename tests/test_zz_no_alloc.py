"""GPU: the no-allocation decode call matches the regular one.

``paged_attention_decode_noalloc`` exists for callers that cannot allocate
device memory (a runtime whose device memory all belongs to its own pool, a C
or embedded host without a device allocator, a loop that cannot afford
cudaMalloc). It keeps its split-KV scratch in a fixed array inside the
library instead of a caller-provided workspace. Here it is called through the
C ABI twice in a row, on two different problems that both split sequences
between workers (so the scratch is really used and the second call runs over
the first call's leftovers), and each result is compared with the regular
call's. This file is collected last so that a failure here does not hide the
other tests' results; it needs no state from them.
"""

import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_gather_b200 as pkv
from paged_kv_cache_gather_b200 import _lib as L
from paged_kv_cache_gather_b200 import inputs as I
from paged_kv_cache_gather_b200.ops import _ptr, cache_desc
from parity import BF16_ATOL, BF16_RTOL, LSE_ATOL, mask_of, to_dev

pytestmark = pytest.mark.gpu


def make_case(seed, mask_kind, window):
    rng = np.random.default_rng(seed)
    lens = rng.integers(1, 3000, size=24).tolist()
    nb = sum(-(-L_ // 16) for L_ in lens) + 16
    return I.make_decode_case("noalloc", lens=lens, num_q_heads=32, num_kv_heads=8, head_dim=128,
                              block_size=16, num_blocks=nb, dtype=torch.bfloat16, seed=seed,
                              mask_kind=mask_kind, window=window, peaky=True)


def regular(case, t):
    return pkv.paged_attention_decode(t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                      t["seq_lens"], case.scale, mask_of(case, t))


def no_alloc(case, t):
    out = torch.empty_like(t["q"])
    lse = torch.empty(t["q"].shape[:2], dtype=torch.float32, device=t["q"].device)
    err = torch.zeros(1, dtype=torch.int32, device=t["q"].device)
    B, Hq, _ = t["q"].shape
    st = L.lib().paged_attention_decode_noalloc(
        _ptr(t["q"]), _ptr(t["k_cache"]), _ptr(t["v_cache"]), cache_desc(t["k_cache"]),
        _ptr(t["block_tables"]), t["block_tables"].shape[1], _ptr(t["seq_lens"]), B, Hq,
        float(case.scale), mask_of(case, t).to_c(B, t["q"].device), _ptr(out), _ptr(lse),
        _ptr(err), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    L.check(st)
    return out, lse, err


def test_noalloc_matches_regular_decode_twice_in_a_row(cuda_device):
    cases = [make_case(31, I.MASK_SLIDING, 700), make_case(32, I.MASK_CAUSAL, 0)]
    devs = [to_dev(c, cuda_device) for c in cases]
    refs = [regular(c, t) for c, t in zip(cases, devs)]
    torch.cuda.synchronize()
    # both calls queued back to back on one stream, one synchronisation at the
    # end: the second call's kernels run right after the first call's, over
    # the scratch the first call has just written
    results = [no_alloc(c, t) for c, t in zip(cases, devs)]
    torch.cuda.synchronize()
    for (ro, rl), (out, lse, err) in zip(refs, results):
        assert err.item() == 0
        o, r = out.float().cpu(), ro.float().cpu()
        assert torch.all((o - r).abs() <= BF16_ATOL + BF16_RTOL * r.abs())
        assert torch.all((lse.cpu() - rl.cpu()).abs() <= LSE_ATOL)
        # same kernels and the same split plan: the results are in fact identical
        assert torch.equal(out.view(torch.int16), ro.view(torch.int16))
        assert torch.equal(lse, rl)


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_device):
    # 3M sequences need more than the 8 MiB scratch for their tile prefix alone;
    # the size check fails before any pointer is touched or kernel launched
    fake = ctypes.c_void_p(0x10000)
    desc = L.CacheDescC(1024, 16, 8, 128, L.PKV_BF16)
    st = L.lib().paged_attention_decode_noalloc(fake, fake, fake, desc, fake, 4, fake, 3_000_000,
                                                32, 0.1, L.MaskModC(1, 0, None), fake, fake,
                                                None, None)
    assert st == L.PKV_ERR_WORKSPACE_TOO_SMALL
    assert b"built-in scratch" in L.lib().pkv_last_error()
