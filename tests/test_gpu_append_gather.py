"""GPU: slot-mapped append and block-table gather are bit-exact against the
oracle, and append leaves every other slot untouched (sentinel pools)."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_gather_b200 as pkv
from paged_kv_cache_gather_b200 import inputs as I

pytestmark = pytest.mark.gpu


def bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


def sentinel_pool(shape, dtype):
    t = torch.empty(shape, dtype=dtype)
    bits(t).fill_(0x7A5C if dtype == torch.bfloat16 else 0x7A5C3E1F)
    return t


def check_append(k, v, slots, kc, vc, dev):
    ek, ev = oracle.kv_append(k, v, slots, kc, vc)
    gk, gv = kc.to(dev), vc.to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    pkv.paged_kv_append(k.to(dev), v.to(dev), slots.to(dev), gk, gv, dbg_err=err)
    torch.cuda.synchronize()
    pkv.read_dbg(err)
    assert torch.equal(bits(gk.cpu()), bits(ek)) and torch.equal(bits(gv.cpu()), bits(ev))


def test_append_tiny_fp32_sentinel(cuda_device):
    case = I.config1()
    kc = sentinel_pool(case.k_cache.shape, torch.float32)
    vc = sentinel_pool(case.v_cache.shape, torch.float32)
    check_append(case.k_new, case.v_new, case.slot_mapping, kc, vc, cuda_device)
    # exactly one row per head changed
    ek, _ = oracle.kv_append(case.k_new, case.v_new, case.slot_mapping, kc, vc)
    changed = (bits(ek) != bits(kc)).any(-1).sum().item()
    assert changed == case.num_kv_heads


@pytest.mark.parametrize("bs", [1, 2, 8, 16, 64])
def test_append_block_sizes_with_padding(cuda_device, bs):
    gen = torch.Generator().manual_seed(bs)
    nb, hkv, d, T = 64, 4, 128, 37
    kc = sentinel_pool((nb, hkv, bs, d), torch.bfloat16)
    vc = sentinel_pool((nb, hkv, bs, d), torch.bfloat16)
    k = I.randn((T, hkv, d), gen)
    v = I.randn((T, hkv, d), gen)
    slots = torch.from_numpy(np.random.default_rng(bs).permutation(nb * bs)[:T].astype(np.int64))
    slots[::5] = -1  # padding tokens
    check_append(k, v, slots, kc, vc, cuda_device)


def test_append_decode_batch_slots(cuda_device):
    case = I.config3()
    check_append(case.k_new, case.v_new, case.slot_mapping, case.k_cache, case.v_cache,
                 cuda_device)


@pytest.mark.slow
def test_append_prefill_chunk_full_size(cuda_device):
    case = I.config5()
    check_append(case.k_new, case.v_new, case.slot_mapping, case.k_cache, case.v_cache,
                 cuda_device)


def test_append_out_of_range_slot_is_flagged_and_skipped(cuda_device):
    kc = sentinel_pool((4, 2, 16, 64), torch.bfloat16)
    vc = sentinel_pool((4, 2, 16, 64), torch.bfloat16)
    gen = torch.Generator().manual_seed(0)
    k = I.randn((2, 2, 64), gen)
    v = I.randn((2, 2, 64), gen)
    slots = torch.tensor([3, 4 * 16 + 2], dtype=torch.int64)
    gk, gv = kc.to(cuda_device), vc.to(cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    pkv.paged_kv_append(k.to(cuda_device), v.to(cuda_device), slots.to(cuda_device), gk, gv,
                        dbg_err=err)
    torch.cuda.synchronize()
    assert err.item() & pkv._lib.PKV_DBG_SLOT
    ek, ev = oracle.kv_append(k[:1], v[:1], slots[:1], kc, vc)
    assert torch.equal(bits(gk.cpu()), bits(ek)) and torch.equal(bits(gv.cpu()), bits(ev))


def check_gather(case, out_max_len, dev):
    ek, ev = oracle.kv_gather(case.k_cache, case.v_cache, case.block_tables, case.seq_lens,
                              out_max_len)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    gk, gv = pkv.paged_kv_gather(case.k_cache.to(dev), case.v_cache.to(dev),
                                 case.block_tables.to(dev), case.seq_lens.to(dev), out_max_len,
                                 dbg_err=err)
    torch.cuda.synchronize()
    pkv.read_dbg(err)
    assert torch.equal(bits(gk.cpu()), bits(ek)) and torch.equal(bits(gv.cpu()), bits(ev))


def test_gather_tiny_fp32(cuda_device):
    check_gather(I.config1(), 160, cuda_device)


@pytest.mark.parametrize("L", I.CONFIG2_LENGTHS)
def test_gather_single_sequence(cuda_device, L):
    check_gather(I.config2(L), L, cuda_device)


def test_gather_ragged_batch(cuda_device):
    case = I.config3()
    check_gather(case, int(case.seq_lens.max()), cuda_device)


def test_gather_cuts_at_out_max_len_and_zero_fills(cuda_device):
    case = I.make_decode_case("g", lens=[0, 5, 33, 70], num_q_heads=2, num_kv_heads=2,
                              head_dim=64, block_size=8, num_blocks=32, dtype=torch.bfloat16,
                              seed=3)
    check_gather(case, 40, cuda_device)


def test_gather_bad_block_id_is_flagged(cuda_device):
    case = I.make_decode_case("g", lens=[20], num_q_heads=2, num_kv_heads=2, head_dim=64,
                              block_size=16, num_blocks=4, dtype=torch.bfloat16, seed=3)
    case.block_tables[0, 1] = 99
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    gk, _ = pkv.paged_kv_gather(case.k_cache.to(cuda_device), case.v_cache.to(cuda_device),
                                case.block_tables.to(cuda_device),
                                case.seq_lens.to(cuda_device), 32, dbg_err=err)
    torch.cuda.synchronize()
    assert err.item() & pkv._lib.PKV_DBG_BLOCK_ID
    with pytest.raises(pkv.PagedKVError):
        pkv.read_dbg(err)
    assert torch.all(gk[0, :, 16:].cpu().float() == 0)  # skipped rows stay zero
