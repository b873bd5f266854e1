"""GPU: the library's FMA-pipe exponential (a building block for taking softmax
exponentials off the MUFU unit) against exp2 in float64: relative error <= 2e-4
on [-126, 8.5] (a softmax with a lazy maximum feeds it values <= 8), exactly 0
below -126 and for -inf."""

import ctypes

import pytest
import torch

from paged_kv_cache_gather_b200 import _lib as L

pytestmark = pytest.mark.gpu


def test_exp2_fma_matches_exp2(cuda_device):
    x = torch.cat([torch.linspace(-126.0, 8.5, 1_000_001),
                   torch.tensor([-126.5, -127.0, -200.0, -1e30, float("-inf"), 0.0, 1.0, -1.0]),
                   torch.randn(100_000) * 20]).float().to(cuda_device)
    x = torch.clamp(x, max=8.5)
    y = torch.empty_like(x)
    L.check(L.lib().pkv_debug_exp2(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(y.data_ptr()),
                                   x.numel(),
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)))
    torch.cuda.synchronize()
    xd, yd = x.double().cpu(), y.double().cpu()
    ref = torch.exp2(xd)
    ok = xd >= -126.0
    rel = ((yd[ok] - ref[ok]).abs() / ref[ok]).max().item()
    assert rel <= 2e-4, rel
    assert torch.all(yd[~ok] == 0)
    assert torch.isfinite(yd).all()
