"""GPU: copy-on-write and device-side allocation on E4M3 pools. A copied
block carries its row scales with its codes (bit for bit against the oracle's
copies of both arrays); the reserve step on E4M3 pools does the host block
manager's bookkeeping and copies, and a whole reserve -> quantising append ->
decode step matches the oracle over the dequantised pools."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_gather_b200 as pkv
from oracle import fp8 as F
from paged_kv_cache_gather_b200 import inputs as I
from parity import assert_attention_close
from test_gpu_reserve import BS, D, HKV, compare, device_state, host_step, scenario

pytestmark = pytest.mark.gpu


def e4m3_pools(seed, num_blocks, hkv=HKV, bs=BS, d=D):
    rng = np.random.default_rng(seed)
    shape = (num_blocks, hkv, bs, d)
    codes = [rng.integers(0, 256, size=shape, dtype=np.uint8) for _ in range(2)]
    for c in codes:  # valid codes only (0x7F / 0xFF are NaN)
        c[(c & 0x7F) == 0x7F] ^= 1
    scales = [rng.uniform(1e-3, 2.0, size=shape[:3]).astype(np.float32) for _ in range(2)]
    return codes[0], codes[1], scales[0], scales[1]


def dev_copies(arrs, dev):
    return [torch.from_numpy(a.copy()).to(dev) for a in arrs]


@pytest.mark.parametrize("hkv,bs", [(8, 16), (1, 8), (2, 64)])
def test_copy_blocks_fp8_moves_codes_and_scales(cuda_device, hkv, bs):
    nb = 24
    kc, vc, ks, vs = e4m3_pools(hkv * 100 + bs, nb, hkv, bs)
    dk, dv, dks, dvs = dev_copies((kc, vc, ks, vs), cuda_device)
    pairs = np.array([[3, 10], [5, 11], [3, 12], [0, 23]], dtype=np.int32)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    pkv.paged_kv_copy_blocks_fp8(dk, dv, dks, dvs, torch.from_numpy(pairs).to(cuda_device),
                                 dbg_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ek, ev = oracle.kv_copy_blocks(kc, vc, pairs)
    eks, evs = oracle.kv_copy_blocks(ks, vs, pairs)
    assert np.array_equal(dk.cpu().numpy(), ek) and np.array_equal(dv.cpu().numpy(), ev)
    assert np.array_equal(dks.cpu().numpy().view(np.int32), eks.view(np.int32))
    assert np.array_equal(dvs.cpu().numpy().view(np.int32), evs.view(np.int32))


def test_copy_blocks_fp8_bad_id_is_flagged_and_skipped(cuda_device):
    kc, vc, ks, vs = e4m3_pools(7, 16)
    dk, dv, dks, dvs = dev_copies((kc, vc, ks, vs), cuda_device)
    pairs = np.array([[2, 9], [1, 16], [-1, 3]], dtype=np.int32)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    pkv.paged_kv_copy_blocks_fp8(dk, dv, dks, dvs, torch.from_numpy(pairs).to(cuda_device),
                                 dbg_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pkv._lib.PKV_DBG_BLOCK_ID
    ek, ev = oracle.kv_copy_blocks(kc, vc, pairs[:1])
    eks, evs = oracle.kv_copy_blocks(ks, vs, pairs[:1])
    assert np.array_equal(dk.cpu().numpy(), ek) and np.array_equal(dv.cpu().numpy(), ev)
    assert np.array_equal(dks.cpu().numpy().view(np.int32), eks.view(np.int32))
    assert np.array_equal(dvs.cpu().numpy().view(np.int32), evs.view(np.int32))


@pytest.mark.parametrize("seed", [11, 12])
def test_reserve_fp8_then_append_and_decode(cuda_device, seed):
    mgr, ids = scenario(seed)
    width = 24
    tables, lens, pool = device_state(mgr, ids, width, cuda_device)
    kc, vc, ks, vs = e4m3_pools(seed, mgr.num_blocks)
    dk, dv, dks, dvs = dev_copies((kc, vc, ks, vs), cuda_device)
    rng = np.random.default_rng(seed + 10)
    num_new = rng.integers(0, 40, size=len(ids)).astype(np.int32)
    T = int(num_new.sum())
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    slots, pairs = pkv.paged_kv_reserve_slots(dk, dv, tables, lens,
                                              torch.from_numpy(num_new).to(cuda_device), pool, T,
                                              dbg_err=err, k_scale=dks, v_scale=dvs)
    torch.cuda.synchronize()
    pkv.read_dbg(err)
    exp_slots, exp_pairs = host_step(mgr, ids, num_new)
    assert np.array_equal(slots.cpu().numpy(), exp_slots)
    assert np.array_equal(pairs.cpu().numpy(), exp_pairs)
    compare(mgr, ids, width, tables, lens, pool)
    used = exp_pairs[exp_pairs[:, 0] >= 0]
    assert len(used) > 0
    ek, ev = oracle.kv_copy_blocks(kc, vc, used)
    eks, evs = oracle.kv_copy_blocks(ks, vs, used)
    assert np.array_equal(dk.cpu().numpy(), ek) and np.array_equal(dv.cpu().numpy(), ev)
    assert np.array_equal(dks.cpu().numpy().view(np.int32), eks.view(np.int32))
    assert np.array_equal(dvs.cpu().numpy().view(np.int32), evs.view(np.int32))

    # quantising append of the new tokens into the reserved slots, then decode
    gen = torch.Generator().manual_seed(seed + 20)
    kn = I.randn((T, HKV, D), gen)
    vn = I.randn((T, HKV, D), gen)
    pkv.paged_kv_append_fp8(kn.to(cuda_device), vn.to(cuda_device), slots, dk, dv, dks, dvs)
    ek, ev, eks, evs = F.kv_append_fp8(kn, vn, exp_slots, ek, ev, eks, evs)
    torch.cuda.synchronize()
    assert np.array_equal(dk.cpu().numpy(), ek) and np.array_equal(dv.cpu().numpy(), ev)
    hq = 4 * HKV
    q = I.randn((len(ids), hq, D), gen)
    out, lse = pkv.paged_attention_decode_fp8(q.to(cuda_device), dk, dv, dks, dvs, tables, lens,
                                              1 / D ** 0.5, pkv.causal())
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.paged_decode(q, F.dequantize_pool(ek, eks), F.dequantize_pool(ev, evs),
                                       tables.cpu(), lens.cpu(), 1 / D ** 0.5, oracle.MASK_CAUSAL)
    assert_attention_close(out.cpu(), lse.cpu(), ref_o, ref_l, torch.bfloat16, "reserve fp8 e2e")
