"""GPU: the block-sparse table of every mask kind, bit-exact against a
classification of the oracle's pairwise visibility (every query-key pair of
every tile tested with ``oracle.visible``)."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_gather_b200 as pkv
from paged_kv_cache_gather_b200 import inputs as I

pytestmark = pytest.mark.gpu


def expected_table(ctx, ql, Hq, kind, window, wps, wph, plen, off, starts, q_tile, k_tile):
    B = len(ctx)
    nqt = -(-max(ql) // q_tile)
    nkt = -(-max(c + q for c, q in zip(ctx, ql)) // k_tile)
    exp = np.zeros((B, Hq, nqt, nkt), dtype=np.uint8)
    for b in range(B):
        n = ctx[b] + ql[b]
        qpos = ctx[b] + np.arange(ql[b])
        kpos = np.arange(n)
        for h in range(Hq):
            w = wph[h] if wph is not None else (wps[b] if wps is not None else window)
            vis = oracle.visible(kind, qpos[:, None], kpos[None, :], w,
                                 plen[b] if plen is not None else 0,
                                 starts[off[b]:off[b + 1]] if off is not None else None)
            for qt in range(nqt):
                for kt in range(nkt):
                    t = vis[qt * q_tile:(qt + 1) * q_tile, kt * k_tile:(kt + 1) * k_tile]
                    if t.size == 0 or not t.any():
                        exp[b, h, qt, kt] = 0
                    elif t.all():
                        exp[b, h, qt, kt] = 2
                    else:
                        exp[b, h, qt, kt] = 1
    return exp


CASES = [
    # kind, q_tile, k_tile
    (I.MASK_NONE, 128, 128),
    (I.MASK_CAUSAL, 128, 128),
    (I.MASK_CAUSAL, 7, 16),
    (I.MASK_SLIDING, 16, 16),
    (I.MASK_PREFIX_LM, 32, 16),
    (I.MASK_DOCUMENT, 64, 16),
    (I.MASK_DOCUMENT, 1, 1),
]


@pytest.mark.parametrize("per_head", [False, True])
@pytest.mark.parametrize("kind,q_tile,k_tile", CASES)
def test_block_mask_matches_pairwise_visibility(cuda_device, kind, q_tile, k_tile, per_head):
    ctx, ql, Hq = [0, 37, 300, 5], [200, 1, 129, 64], 4
    rng = np.random.default_rng(kind * 10 + q_tile)
    wps = np.array([0, 5, 40, 17], dtype=np.int32)
    wph = np.array([1, 0, 33, 300], dtype=np.int32) if per_head else None
    plen = np.array([10, 50, 1000, 0], dtype=np.int32)
    off_t, st_t = I.document_starts([c + q for c, q in zip(ctx, ql)], 3, mean_doc=40)
    off, st = off_t.numpy(), st_t.numpy()
    dev = cuda_device
    mm = pkv.MaskMod(kind, 3, torch.from_numpy(wps).to(dev),
                     torch.from_numpy(wph).to(dev) if per_head else None,
                     torch.from_numpy(plen).to(dev), off_t.to(dev), st_t.to(dev))
    got = pkv.block_mask(torch.tensor(ctx, dtype=torch.int32, device=dev),
                         torch.tensor(ql, dtype=torch.int32, device=dev), Hq, mm, q_tile, k_tile)
    exp = expected_table(ctx, ql, Hq, kind, 3, wps, wph if kind == I.MASK_SLIDING else None,
                         plen, off, st, q_tile, k_tile)
    assert np.array_equal(got.cpu().numpy(), exp)


def test_decode_shaped_table(cuda_device):
    # a decode step: ctx = seq_len - 1, one query; 16-token key tiles
    lens = [1, 16, 17, 4000]
    dev = cuda_device
    ctx = torch.tensor([L - 1 for L in lens], dtype=torch.int32, device=dev)
    ql = torch.ones(4, dtype=torch.int32, device=dev)
    wps = torch.tensor([0, 4, 16, 1000], dtype=torch.int32, device=dev)
    got = pkv.block_mask(ctx, ql, 2, pkv.sliding_window(wps), 1, 16).cpu().numpy()
    exp = expected_table([L - 1 for L in lens], [1] * 4, 2, I.MASK_SLIDING, 0, wps.cpu().numpy(),
                         None, None, None, None, 1, 16)
    assert np.array_equal(got, exp)
    # the tiles a decode reads are exactly the non-skipped ones
    assert (got[3, 0, 0] > 0).sum() == -(-4000 // 16) - (4000 - 1000) // 16
