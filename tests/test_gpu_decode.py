"""GPU: paged decode (append + decode step) against the float64 oracle.

Covers the five workloads (tiny fp32; batch-1 sweep 128..4096; ragged batch of
64 with windows on even sequences, at full size; shared-prefix beams, shared
vs copied; plus "peaky" variants whose outputs are O(1) so the tolerance
bites) and the edge cases: empty and one-token sequences, lengths around tile
and block edges, windows of 1 and longer than the sequence, block sizes 8..128,
head_dim 64, group sizes 1..8, many sequences, a bad block id.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_gather_b200 as pkv
from paged_kv_cache_gather_b200 import inputs as I
from parity import (assert_attention_close, oracle_after_append, oracle_decode, run_decode,
                    to_dev, mask_of)

pytestmark = pytest.mark.gpu


def check_case(case, dev, rows=None):
    out, lse, gk, gv = run_decode(case, dev)
    kc, vc = oracle_after_append(case)
    if rows is None:
        ref_o, ref_l = oracle_decode(case, kc, vc)
        assert_attention_close(out, lse, ref_o, ref_l, case.dtype, case.name)
    else:
        res = oracle_decode(case, kc, vc, rows)
        ro = np.stack([res[r][0] for r in rows])
        rl = np.array([res[r][1] for r in rows])
        go = torch.stack([out[b, h] for b, h in rows])
        gl = torch.stack([lse[b, h] for b, h in rows])
        assert_attention_close(go, gl, ro, rl, case.dtype, case.name)
    return out, lse


@pytest.mark.parametrize("L", [128, 129])
def test_cfg1_tiny_fp32(cuda_device, L):
    check_case(I.config1(L=L), cuda_device)


@pytest.mark.parametrize("L", I.CONFIG2_LENGTHS)
@pytest.mark.parametrize("peaky", [False, True])
def test_cfg2_single_sequence_sweep(cuda_device, L, peaky):
    check_case(I.config2(L, peaky=peaky), cuda_device)


@pytest.mark.slow
@pytest.mark.parametrize("peaky", [False, True])
def test_cfg3_ragged_batch_full_size(cuda_device, peaky):
    check_case(I.config3(peaky=peaky), cuda_device)


@pytest.mark.slow
def test_cfg4_shared_prefix_equals_copies(cuda_device):
    sh = I.config4(shared=True)
    cp = I.config4(shared=False)
    o1, l1 = check_case(sh, cuda_device)
    o2, l2 = check_case(cp, cuda_device)
    # same lengths give the same split plan: results are bit-identical
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


def test_cfg4_small_peaky(cuda_device):
    check_case(I.config4(groups=2, beams=4, prefix=512, suffix=64, num_blocks=512, peaky=True),
               cuda_device)


def test_physical_permutation_is_bit_identical(cuda_device):
    case = I.make_decode_case("perm", lens=[1, 300, 1000, 4097, 77], num_q_heads=32,
                              num_kv_heads=8, head_dim=128, block_size=16, num_blocks=512,
                              dtype=torch.bfloat16, seed=5, mask_kind=I.MASK_CAUSAL)
    o1, l1, _, _ = run_decode(case, cuda_device, do_append=False)
    perm = torch.from_numpy(np.random.default_rng(1).permutation(case.num_blocks))
    case2 = I.PagedCase(**{**case.__dict__})
    case2.k_cache = torch.empty_like(case.k_cache)
    case2.v_cache = torch.empty_like(case.v_cache)
    case2.k_cache[perm] = case.k_cache
    case2.v_cache[perm] = case.v_cache
    tab = case.block_tables.clone()
    valid = tab >= 0
    tab[valid] = perm[tab[valid].long()].int()
    case2.block_tables = tab
    o2, l2, _, _ = run_decode(case2, cuda_device, do_append=False)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


def test_repeat_is_deterministic(cuda_device):
    case = I.config3(batch=16, peaky=False)
    o1, l1, _, _ = run_decode(case, cuda_device, do_append=False)
    o2, l2, _, _ = run_decode(case, cuda_device, do_append=False)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


EDGE = [
    # lens, Hq, Hkv, d, bs, mask, window
    ([1, 2, 15, 16, 17, 31, 32, 33], 32, 8, 128, 16, I.MASK_CAUSAL, 0),
    ([0, 5, 0, 40], 8, 2, 128, 16, I.MASK_CAUSAL, 0),
    ([0], 8, 2, 128, 16, I.MASK_NONE, 0),
    ([100, 257, 1000], 8, 8, 128, 16, I.MASK_NONE, 0),           # g = 1
    ([100, 257, 1000], 16, 8, 128, 16, I.MASK_CAUSAL, 0),        # g = 2
    ([100, 257, 1000], 64, 8, 128, 16, I.MASK_CAUSAL, 0),        # g = 8
    ([100, 257, 1000], 24, 8, 128, 16, I.MASK_CAUSAL, 0),        # g = 3
    ([3000, 17, 900], 32, 8, 128, 16, I.MASK_SLIDING, 1),        # W = 1: only self
    ([3000, 17, 900], 32, 8, 128, 16, I.MASK_SLIDING, 37),       # W not tile-aligned
    ([3000, 17, 900], 32, 8, 128, 16, I.MASK_SLIDING, 5000),     # W > L: causal
    ([999, 2048, 3], 32, 8, 64, 16, I.MASK_SLIDING, 300),        # head_dim 64
    ([999, 2048, 3, 45], 32, 8, 128, 8, I.MASK_CAUSAL, 0),       # block 8
    ([999, 2048, 3, 45], 32, 8, 128, 8, I.MASK_SLIDING, 21),
    ([999, 2048, 3, 45], 32, 8, 128, 32, I.MASK_SLIDING, 100),   # block 32
    ([999, 2048, 3, 45], 32, 4, 128, 64, I.MASK_CAUSAL, 0),      # block 64
    ([999, 2048, 3, 45], 32, 4, 64, 128, I.MASK_SLIDING, 700),   # block 128, d 64
]


@pytest.mark.parametrize("lens,hq,hkv,d,bs,kind,w", EDGE)
def test_edge_cases(cuda_device, lens, hq, hkv, d, bs, kind, w):
    nb = sum(-(-L // bs) for L in lens) + 8
    case = I.make_decode_case("edge", lens=lens, num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                              block_size=bs, num_blocks=nb, dtype=torch.bfloat16, seed=len(lens),
                              mask_kind=kind, window=w)
    check_case(case, cuda_device)


def test_many_sequences_and_per_sequence_windows(cuda_device):
    rng = np.random.default_rng(9)
    lens = rng.integers(0, 700, size=300).tolist()
    wps = torch.from_numpy(rng.integers(-5, 400, size=300).astype(np.int32))
    nb = sum(-(-L // 16) for L in lens) + 4
    case = I.make_decode_case("many", lens=lens, num_q_heads=8, num_kv_heads=2, head_dim=128,
                              block_size=16, num_blocks=nb, dtype=torch.bfloat16, seed=9,
                              mask_kind=I.MASK_SLIDING, window_per_seq=wps)
    check_case(case, cuda_device)


def test_fp32_edge_cases(cuda_device):
    case = I.make_decode_case("f32", lens=[0, 1, 200, 513], num_q_heads=8, num_kv_heads=2,
                              head_dim=128, block_size=8, num_blocks=120, dtype=torch.float32,
                              seed=4, mask_kind=I.MASK_SLIDING, window=100)
    check_case(case, cuda_device)


def test_bad_block_id_is_flagged_without_fault(cuda_device):
    case = I.make_decode_case("bad", lens=[100], num_q_heads=8, num_kv_heads=2, head_dim=128,
                              block_size=16, num_blocks=16, dtype=torch.bfloat16, seed=2)
    case.block_tables[0, 3] = 1 << 20
    t = to_dev(case, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    pkv.paged_attention_decode(t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                               t["seq_lens"], case.scale, mask_of(case, t), dbg_err=err)
    torch.cuda.synchronize()
    assert err.item() & pkv._lib.PKV_DBG_BLOCK_ID


def test_unsupported_group_size_is_rejected(cuda_device):
    case = I.make_decode_case("g16", lens=[10], num_q_heads=32, num_kv_heads=2, head_dim=128,
                              block_size=16, num_blocks=4, dtype=torch.bfloat16, seed=2)
    with pytest.raises(pkv.PagedKVError):
        run_decode(case, cuda_device, do_append=False)


def poisoned_dead_rows(case, w=0):
    """Pool rows in the same blocks as visible keys but outside the visible range
    (past the last key, and before a sliding window's first key) set to NaN."""
    bs = case.k_cache.shape[2]
    tab = case.block_tables.numpy()
    n = 0
    for b, L in enumerate(case.seq_lens.tolist()):
        if L <= 0:
            continue
        lo = max(0, L - w) if w > 0 else 0
        dead = list(range(L, -(-L // bs) * bs)) + list(range((lo // bs) * bs, lo))
        for pos in dead:
            blk = int(tab[b, pos // bs])
            case.k_cache[blk, :, pos % bs] = float("nan")
            case.v_cache[blk, :, pos % bs] = float("nan")
            n += 1
    return n


@pytest.mark.parametrize("kind,w", [(I.MASK_CAUSAL, 0), (I.MASK_SLIDING, 100)])
def test_nan_in_rows_outside_the_visible_range(cuda_device, kind, w):
    # the tile that holds a sequence's last key (or a window's first) also loads
    # rows the query must not see; stale or non-finite data there changes nothing
    lens = [5, 17, 300, 1000]
    nb = sum(-(-L // 16) for L in lens) + 8
    case = I.make_decode_case(f"nan_rows_{kind}", lens=lens, num_q_heads=32, num_kv_heads=8,
                              head_dim=128, block_size=16, num_blocks=nb, dtype=torch.bfloat16,
                              seed=31, mask_kind=kind, window=w)
    clean = I.PagedCase(**{**case.__dict__})
    clean.k_cache, clean.v_cache = case.k_cache.clone(), case.v_cache.clone()
    assert poisoned_dead_rows(case, w) > 0
    out, lse, _, _ = run_decode(case, cuda_device)
    # the reference is the attention over the clean pools (the oracle resolves
    # whole blocks, where the NaN rows would reach its P*V even at weight 0)
    kc, vc = oracle_after_append(clean)
    ref_o, ref_l = oracle_decode(clean, kc, vc)
    assert_attention_close(out, lse, ref_o, ref_l, case.dtype, case.name)
