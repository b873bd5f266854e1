"""GPU: the bounded wait gives up cleanly. One warp waits on an mbarrier that
nothing arrives on, through the same wait the kernels use for their TMA and
MMA barriers; after the limit the kernel sets PKV_DBG_TIMEOUT and returns,
the host reads the flag, and the context keeps working (an append and a decode
run afterwards and match the oracle). No fault, trap or endless loop is
involved: the wait is bounded by the globaltimer."""

import ctypes

import pytest
import torch

import oracle
import paged_kv_cache_gather_b200 as pkv
from paged_kv_cache_gather_b200 import _lib as L
from paged_kv_cache_gather_b200 import inputs as I
from parity import assert_attention_close

pytestmark = pytest.mark.gpu


def test_wait_gives_up_with_flag_and_context_survives(cuda_device):
    dbg = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    elapsed = torch.zeros(1, dtype=torch.int64, device=cuda_device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    L.check(L.lib().pkv_debug_wait_timeout(ctypes.c_void_p(dbg.data_ptr()),
                                           ctypes.c_void_p(elapsed.data_ptr()), stream))
    torch.cuda.synchronize()
    assert int(dbg.item()) == L.PKV_DBG_TIMEOUT
    ns = int(elapsed.item())
    assert 4.0e9 <= ns < 30e9, ns

    # the context is still usable: a small append + decode against the oracle
    case = I.config1()
    kc, vc = case.k_cache.to(cuda_device), case.v_cache.to(cuda_device)
    pkv.paged_kv_append(case.k_new.to(cuda_device), case.v_new.to(cuda_device),
                        case.slot_mapping.to(cuda_device), kc, vc)
    out, lse = pkv.paged_attention_decode(case.q.to(cuda_device), kc, vc,
                                          case.block_tables.to(cuda_device),
                                          case.seq_lens.to(cuda_device), case.scale, pkv.no_mask())
    ek, ev = oracle.kv_append(case.k_new, case.v_new, case.slot_mapping, case.k_cache, case.v_cache)
    ref_o, ref_l = oracle.paged_decode(case.q, ek, ev, case.block_tables, case.seq_lens,
                                       case.scale, oracle.MASK_NONE)
    assert_attention_close(out.cpu(), lse.cpu(), ref_o, ref_l, torch.float32, "after timeout")


def test_null_debug_word_is_rejected(cuda_device):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.lib().pkv_debug_wait_timeout(None, None, stream) == L.PKV_ERR_INVALID_ARG
