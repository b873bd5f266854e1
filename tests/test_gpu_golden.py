"""GPU: the library against the hand-derived worked example of
tests/golden/ (float32 pools, block size 2, head_dim 4): decode under each
mask, the append's slot and the gather, through the C ABI."""

import numpy as np
import pytest
import torch

import paged_kv_cache_gather_b200 as pkv
from golden_case import array, load, value

pytestmark = pytest.mark.gpu


def masks(c):
    if c["mask"] == "none":
        return pkv.no_mask()
    if c["mask"] == "causal":
        return pkv.causal()
    return pkv.sliding_window(c["window"])


def test_golden_decode_append_gather(cuda_device):
    g, k, v = load()
    dev = cuda_device
    kc = torch.from_numpy(k).float().to(dev)
    vc = torch.from_numpy(v).float().to(dev)
    tables = torch.tensor([g["block_table"]], dtype=torch.int32, device=dev)
    d = g["decode"]
    lens = torch.tensor([d["seq_len"]], dtype=torch.int32, device=dev)
    q = torch.from_numpy(array(d["q"])).float().reshape(1, 1, -1).to(dev)
    for c in d["cases"]:
        out, lse = pkv.paged_attention_decode(q, kc, vc, tables, lens, d["scale"], masks(c))
        torch.cuda.synchronize()
        assert np.allclose(out[0, 0].double().cpu().numpy(), array(c["out"]), rtol=0,
                           atol=1e-5), c
        assert abs(float(lse[0, 0]) - value(c["lse"])) < 1e-5, c

    ga = g["gather"]
    ko, vo = pkv.paged_kv_gather(kc, vc, tables, lens, ga["out_max_len"])
    torch.cuda.synchronize()
    assert np.array_equal(ko[0, 0].cpu().numpy(), array(ga["k"]).astype(np.float32))
    assert np.array_equal(vo[0, 0].cpu().numpy(), array(ga["v"]).astype(np.float32))

    a = g["append"]
    kn = torch.from_numpy(array(a["k"])).float().reshape(1, 1, -1).to(dev)
    vn = torch.from_numpy(array(a["v"])).float().reshape(1, 1, -1).to(dev)
    pkv.paged_kv_append(kn, vn, torch.tensor([a["slot"]], dtype=torch.int64, device=dev), kc, vc)
    torch.cuda.synchronize()
    ek = torch.from_numpy(k).float()
    ev = torch.from_numpy(v).float()
    ek[a["block"], :, a["row"], :] = kn[0, 0].cpu()
    ev[a["block"], :, a["row"], :] = vn[0, 0].cpu()
    assert torch.equal(kc.cpu(), ek) and torch.equal(vc.cpu(), ev)
