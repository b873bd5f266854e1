"""GPU: the fused decode step (paged_attention_decode_append) against the
two-call step it replaces and against the float64 oracle.

The fused call writes each sequence's new token at position seq_lens[b]-1 of
its block table and decodes in the same launch. Its pools and results must be
bit-identical to paged_kv_append (with the slots of those positions) followed
by paged_attention_decode, and within the stated bounds of the oracle (append
then decode, "Ultimate Guide to PagedAttention", dynamic growth). Cases: the
full ragged workload, plain and peaky; lengths at tile and block edges and
empty sequences; block sizes 8..64; head_dim 64; sliding, per-head and
document masks; a length-1 sequence (the new token is its only key).
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_gather_b200 as pkv
from paged_kv_cache_gather_b200 import inputs as I
from parity import (assert_attention_close, mask_of, oracle_after_append, oracle_decode,
                    to_dev)

pytestmark = pytest.mark.gpu


def two_calls(case, t, err):
    pkv.paged_kv_append(t["k_new"], t["v_new"], t["slot_mapping"], t["k_cache"], t["v_cache"],
                        dbg_err=err)
    return pkv.paged_attention_decode(t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                      t["seq_lens"], case.scale, mask_of(case, t), dbg_err=err)


def fused(case, t, err):
    return pkv.paged_attention_decode_append(t["q"], t["k_new"], t["v_new"], t["k_cache"],
                                             t["v_cache"], t["block_tables"], t["seq_lens"],
                                             case.scale, mask_of(case, t), dbg_err=err)


def check(case, dev, rows=None):
    ta, tb = to_dev(case, dev), to_dev(case, dev)
    ea = torch.zeros(1, dtype=torch.int32, device=dev)
    eb = torch.zeros(1, dtype=torch.int32, device=dev)
    oa, la = two_calls(case, ta, ea)
    ob, lb = fused(case, tb, eb)
    torch.cuda.synchronize()
    assert ea.item() == 0 and eb.item() == 0
    # the same pools and the same results, bit for bit
    assert torch.equal(ta["k_cache"].view(torch.int16), tb["k_cache"].view(torch.int16))
    assert torch.equal(ta["v_cache"].view(torch.int16), tb["v_cache"].view(torch.int16))
    assert torch.equal(oa.view(torch.int16), ob.view(torch.int16))
    assert torch.equal(la, lb)
    # and the oracle's append and attention
    kc, vc = oracle_after_append(case)
    assert torch.equal(tb["k_cache"].cpu().view(torch.int16), kc.view(torch.int16))
    assert torch.equal(tb["v_cache"].cpu().view(torch.int16), vc.view(torch.int16))
    if rows is None:
        ref_o, ref_l = oracle_decode(case, kc, vc)
        assert_attention_close(ob.cpu(), lb.cpu(), ref_o, ref_l, case.dtype, case.name)
    else:
        res = oracle_decode(case, kc, vc, rows)
        ro = np.stack([res[r][0] for r in rows])
        rl = np.array([res[r][1] for r in rows])
        go = torch.stack([ob[b, h].cpu() for b, h in rows])
        gl = torch.stack([lb[b, h].cpu() for b, h in rows])
        assert_attention_close(go, gl, ro, rl, case.dtype, case.name)


def ragged(name, lens, bs=16, d=128, hq=32, hkv=8, seed=7, **kw):
    nb = sum(-(-L // bs) for L in lens) + 24
    return I.make_decode_case(name, lens=lens, num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                              block_size=bs, num_blocks=nb, dtype=torch.bfloat16, seed=seed, **kw)


@pytest.mark.slow
@pytest.mark.parametrize("peaky", [False, True])
def test_ragged_workload_full_size(cuda_device, peaky):
    case = I.config3(peaky=peaky)
    rng = np.random.default_rng(3 + int(peaky))
    rows = [(int(b), int(h)) for b, h in zip(rng.integers(0, case.batch, 96),
                                             rng.integers(0, 32, 96))]
    rows += [(b, 0) for b in range(case.batch)]
    check(case, cuda_device, rows=sorted(set(rows)))


EDGE_LENS = [1, 2, 15, 16, 17, 31, 32, 33, 255, 256, 257, 1000, 0, 4097]


@pytest.mark.parametrize("bs", [8, 16, 32, 64])
def test_edge_lengths_and_block_sizes(cuda_device, bs):
    check(ragged(f"append_edges_bs{bs}", EDGE_LENS, bs=bs, mask_kind=I.MASK_CAUSAL),
          cuda_device)


def test_head_dim_64_and_group_8(cuda_device):
    check(ragged("append_d64_g8", [5, 700, 129, 2048], d=64, hq=16, hkv=2,
                 mask_kind=I.MASK_NONE), cuda_device)


@pytest.mark.parametrize("w", [1, 17, 300])
def test_sliding_window(cuda_device, w):
    check(ragged(f"append_win{w}", [1, 40, 333, 1500, 2049], mask_kind=I.MASK_SLIDING,
                 window=w, peaky=True), cuda_device)


def test_per_head_windows_and_documents(cuda_device):
    lens = [3, 250, 1100, 64]
    case = ragged("append_per_head", lens, peaky=True)
    wph = torch.tensor([0, 5, 64, 1000] * 8, dtype=torch.int32)
    check(I.with_mask(case, I.MASK_SLIDING, window_per_head=wph), cuda_device)
    case = ragged("append_docs", lens, seed=9)
    off, st = I.document_starts(lens, 4, mean_doc=90)
    check(I.with_mask(case, I.MASK_DOCUMENT, doc_offsets=off, doc_starts=st), cuda_device)


def test_unsupported_pool_dtype_rejected(cuda_device):
    case = I.config1()
    t = to_dev(case, cuda_device)
    with pytest.raises((ValueError, pkv.PagedKVError)):
        fused(case, t, None)


@pytest.mark.parametrize("d", [64, 128])
def test_short_batch(cuda_device, d):
    # a short list (one tile per warp, segments cut into single-tile pieces),
    # empty sequences among them, plain and with per-head windows
    lens = [1, 17, 100, 160, 0, 33]
    check(ragged(f"append_short_d{d}", lens, d=d, mask_kind=I.MASK_CAUSAL), cuda_device)
    case = ragged(f"append_short_ph_d{d}", lens, d=d, peaky=True)
    wph = torch.tensor([0, 5, 64, 1000] * 8, dtype=torch.int32)
    check(I.with_mask(case, I.MASK_SLIDING, window_per_head=wph), cuda_device)
