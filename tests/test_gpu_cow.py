"""GPU: copy-on-write of shared blocks, end to end with the host block manager.

A sequence whose last block is half full is forked (the blocks are shared by
id); appending to the fork makes the manager hand out a private copy of that
block. The device copies it (paged_kv_copy_blocks), appends the new token, and
both sequences then decode to the oracle's results; the pools match the
oracle's copy + append bit for bit, and the parent's blocks are untouched.
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_gather_b200 as pkv
from paged_kv_cache_gather_b200 import inputs as I
from parity import assert_attention_close

pytestmark = pytest.mark.gpu


def test_fork_copy_on_write_append_decode(cuda_device):
    dev = cuda_device
    nb, hkv, bs, d, hq = 64, 2, 16, 128, 8
    gen = torch.Generator().manual_seed(21)
    kc = I.randn((nb, hkv, bs, d), gen)
    vc = I.randn((nb, hkv, bs, d), gen)
    bm = pkv.BlockManager(nb, bs, seed=4)
    bm.add_sequence(0, 40)                      # 3 blocks, the last one half full
    bm.fork(0, 1)
    slots, copies = bm.append_slots(1, 1)       # writes into the shared last block
    assert len(copies) == 1
    k_new = I.randn((1, hkv, d), gen)
    v_new = I.randn((1, hkv, d), gen)
    # expected pools: copy, then append
    ek, ev = oracle.kv_copy_blocks(kc, vc, copies)
    ek, ev = oracle.kv_append(k_new, v_new, torch.tensor(slots), ek, ev)
    gk, gv = kc.to(dev), vc.to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    pkv.paged_kv_copy_blocks(gk, gv, copies, dbg_err=err)
    pkv.paged_kv_append(k_new.to(dev), v_new.to(dev), torch.tensor(slots, device=dev), gk, gv,
                        dbg_err=err)
    torch.cuda.synchronize()
    pkv.read_dbg(err)
    assert torch.equal(gk.cpu().view(torch.int16), ek.view(torch.int16))
    assert torch.equal(gv.cpu().view(torch.int16), ev.view(torch.int16))
    src = copies[0][0]
    assert torch.equal(gk[src].cpu().view(torch.int16), kc[src].view(torch.int16))  # parent's block
    # decode both sequences from the updated pools
    tabs = bm.block_table_tensor([0, 1])
    lens = bm.seq_lens_tensor([0, 1])
    q = I.randn((2, hq, d), gen)
    out, lse = pkv.paged_attention_decode(q.to(dev), gk, gv, tabs.to(dev), lens.to(dev),
                                          1.0 / np.sqrt(d), pkv.causal())
    ro, rl = oracle.paged_decode(q, ek, ev, tabs, lens, 1.0 / np.sqrt(d), I.MASK_CAUSAL)
    assert_attention_close(out.cpu(), lse.cpu(), ro, rl, torch.bfloat16, "cow")


def test_copy_blocks_bad_id_is_flagged(cuda_device):
    kc = torch.zeros(4, 1, 16, 64, dtype=torch.bfloat16, device=cuda_device)
    vc = torch.zeros_like(kc)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    pkv.paged_kv_copy_blocks(kc, vc, [[0, 9]], dbg_err=err)
    torch.cuda.synchronize()
    assert err.item() & pkv._lib.PKV_DBG_BLOCK_ID
