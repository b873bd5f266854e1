"""GPU: shared-prefix (cascade) decode against the float64 oracle.

The call splits each group's attention into the shared prefix (read once per
group and KV head) and every member's own keys, then merges the two by
log-sum-exp; the oracle is plain decode over the whole context. Covers the
beams workload (8 groups x 8 beams, 4096 shared + 256 own tokens) at full
size, ragged groups (sizes 1..32, prefixes that end inside a block, members
with no own tokens, groups with no prefix, empty sequences), block sizes
8..64, both masks a decode query can take, and the argument and device checks.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_gather_b200 as pkv
from paged_kv_cache_gather_b200 import inputs as I
from paged_kv_cache_gather_b200._lib import PagedKVError
from parity import assert_attention_close, oracle_decode, to_dev, mask_of

pytestmark = pytest.mark.gpu


def run_shared(case, dev, max_group_size=None, shared_len=None, group_start=None, dbg=True):
    t = to_dev(case, dev)
    gs = (group_start if group_start is not None else case.extra["group_start"]).to(dev)
    sl = (shared_len if shared_len is not None else case.extra["shared_len"]).to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    out, lse = pkv.paged_attention_decode_shared_prefix(
        t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["seq_lens"], gs, sl,
        max_group_size or case.extra["max_group_size"], case.scale, mask_of(case, t),
        dbg_err=err)
    torch.cuda.synchronize()
    if dbg:
        pkv.read_dbg(err)
    return out.cpu(), lse.cpu(), err


def check(case, dev, **kw):
    out, lse, _ = run_shared(case, dev, **kw)
    ref_o, ref_l = oracle_decode(case, case.k_cache, case.v_cache)
    assert_attention_close(out, lse, ref_o, ref_l, case.dtype, case.name)
    return out, lse


def ragged(name, seed, **kw):
    return I.make_shared_prefix_case(name, seed=seed, **kw)


def test_small_ragged_groups(cuda_device):
    case = ragged("ragged_small", 11, group_sizes=[3, 1, 2], prefix_lens=[40, 0, 32],
                  suffix_lens=[5, 0, 17, 1, 9, 0], num_q_heads=8, num_kv_heads=2)
    check(case, cuda_device)


@pytest.mark.parametrize("peaky", [False, True])
def test_beams_small(cuda_device, peaky):
    check(I.config4(groups=2, beams=4, prefix=512, suffix=64, num_blocks=512, peaky=peaky),
          cuda_device)


@pytest.mark.parametrize("peaky", [False, True])
def test_beams_full_size(cuda_device, peaky):
    case = I.config4(peaky=peaky)
    out, lse = check(case, cuda_device)
    # the same batch through plain decode agrees within the rounding of one bf16 step
    t = to_dev(case, cuda_device)
    o2, l2 = pkv.paged_attention_decode(t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                        t["seq_lens"], case.scale, mask_of(case, t))
    assert torch.allclose(l2.cpu(), lse, atol=1e-3)
    assert torch.allclose(o2.cpu().float(), out.float(), atol=2e-2, rtol=2e-2)


@pytest.mark.parametrize("prefix,suffix_hi", [(1, 3), (15, 17), (16, 16), (127, 130),
                                              (128, 1), (129, 300), (2000, 700)])
def test_prefix_lengths(cuda_device, prefix, suffix_hi):
    rng = np.random.default_rng(prefix)
    sizes = [4, 3, 1]
    suffix = rng.integers(0, suffix_hi + 1, size=sum(sizes)).tolist()
    case = ragged(f"prefix_{prefix}", 100 + prefix, group_sizes=sizes,
                  prefix_lens=[prefix, prefix + 7, prefix], suffix_lens=suffix, peaky=True)
    check(case, cuda_device)


def test_largest_group(cuda_device):
    # 32 members x 4 query heads per KV head fill the 128-row query tile
    rng = np.random.default_rng(3)
    case = ragged("group32", 3, group_sizes=[32, 5], prefix_lens=[1000, 333],
                  suffix_lens=rng.integers(0, 200, size=37).tolist(), peaky=True)
    check(case, cuda_device)


def test_two_row_blocks(cuda_device):
    # 16 members x 4 heads = 64 rows: the prefix is attended in two 32-row blocks
    rng = np.random.default_rng(6)
    case = ragged("rows64", 6, group_sizes=[16, 16, 3], prefix_lens=[700, 1400, 5],
                  suffix_lens=rng.integers(0, 50, size=35).tolist(), peaky=True)
    check(case, cuda_device)


def test_group_too_large_rejected(cuda_device):
    case = ragged("group33", 4, group_sizes=[33], prefix_lens=[64], suffix_lens=[1] * 33)
    with pytest.raises(PagedKVError):
        run_shared(case, cuda_device)


def test_max_group_size_above_sizes(cuda_device):
    case = ragged("loose_bound", 5, group_sizes=[2, 3, 1], prefix_lens=[96, 50, 10],
                  suffix_lens=[3, 4, 5, 6, 7, 8])
    check(case, cuda_device, max_group_size=8)


@pytest.mark.parametrize("bs", [8, 32, 64])
def test_block_sizes(cuda_device, bs):
    case = ragged(f"bs{bs}", 20 + bs, group_sizes=[4, 2], prefix_lens=[3 * bs + 5, 2 * bs],
                  suffix_lens=[1, bs, 2 * bs + 3, 0, 7, 9], block_size=bs, peaky=True)
    check(case, cuda_device)


def test_no_mask_equals_causal(cuda_device):
    case = ragged("nomask", 7, group_sizes=[3, 3], prefix_lens=[200, 64],
                  suffix_lens=[10, 20, 30, 1, 2, 3], mask_kind=I.MASK_NONE)
    check(case, cuda_device)


def test_no_prefix_anywhere_and_empty_sequences(cuda_device):
    case = ragged("noprefix", 8, group_sizes=[2, 1, 3], prefix_lens=[0, 0, 0],
                  suffix_lens=[0, 40, 17, 0, 1, 0])
    out, lse = check(case, cuda_device)
    empty = case.seq_lens == 0
    assert torch.all(out[empty] == 0) and torch.all(torch.isneginf(lse[empty]))


def test_group_query_heads_1_and_8(cuda_device):
    for hq, hkv in ((8, 8), (32, 4)):
        case = ragged(f"g{hq // hkv}", 9, group_sizes=[4, 2], prefix_lens=[100, 48],
                      suffix_lens=[1, 2, 3, 4, 5, 6], num_q_heads=hq, num_kv_heads=hkv,
                      peaky=True)
        check(case, cuda_device, max_group_size=4)


@pytest.mark.parametrize("hq,hkv", [(16, 1), (24, 1), (32, 1), (32, 2)])
def test_group_query_heads_16_to_32(cuda_device, hq, hkv):
    # up to 16 query heads per KV head take 16-row segments, more take 32-row ones;
    # 24 heads make segments that straddle two members
    case = ragged(f"g{hq // hkv}", 12 + hq, group_sizes=[3, 1, 2], prefix_lens=[300, 17, 64],
                  suffix_lens=[0, 9, 40, 1, 16, 33], num_q_heads=hq, num_kv_heads=hkv,
                  peaky=True)
    check(case, cuda_device)


def test_sliding_window_rejected(cuda_device):
    case = ragged("sliding", 10, group_sizes=[2], prefix_lens=[32], suffix_lens=[1, 1])
    case.mask_kind = I.MASK_SLIDING
    case.window = 8
    with pytest.raises(PagedKVError):
        run_shared(case, cuda_device)


def test_inconsistent_shared_len_flagged(cuda_device):
    case = ragged("mismatch", 12, group_sizes=[3], prefix_lens=[64], suffix_lens=[4, 4, 4])
    sl = case.extra["shared_len"].clone()
    sl[1] = 48
    _, _, err = run_shared(case, cuda_device, shared_len=sl, dbg=False)
    assert int(err.item()) & pkv._lib.PKV_DBG_LENGTH


def test_groups_not_covering_batch_flagged(cuda_device):
    case = ragged("cover", 13, group_sizes=[2, 2], prefix_lens=[32, 32], suffix_lens=[1] * 4)
    gs = torch.tensor([0, 2, 3], dtype=torch.int32)
    _, _, err = run_shared(case, cuda_device, group_start=gs, dbg=False)
    assert int(err.item()) & pkv._lib.PKV_DBG_LENGTH


def test_prefix_past_sequence_flagged(cuda_device):
    case = ragged("past", 14, group_sizes=[2], prefix_lens=[32], suffix_lens=[0, 5])
    sl = case.extra["shared_len"].clone()
    sl[:] = 36  # longer than the first member's 32 tokens
    _, _, err = run_shared(case, cuda_device, shared_len=sl, dbg=False)
    assert int(err.item()) & pkv._lib.PKV_DBG_LENGTH


def test_two_calls_in_a_row_share_a_workspace(cuda_device):
    case = ragged("twice", 15, group_sizes=[3, 2], prefix_lens=[77, 300],
                  suffix_lens=[9, 8, 7, 6, 5], peaky=True)
    t = to_dev(case, cuda_device)
    ws = pkv.shared_prefix_workspace(case.batch, case.num_q_heads, t["k_cache"])
    gs = case.extra["group_start"].to(cuda_device)
    sl = case.extra["shared_len"].to(cuda_device)
    res = []
    for _ in range(2):
        o, l = pkv.paged_attention_decode_shared_prefix(
            t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["seq_lens"], gs, sl, 3,
            case.scale, mask_of(case, t), workspace=ws)
        res.append((o.clone(), l.clone()))
    torch.cuda.synchronize()
    assert torch.equal(res[0][0].view(torch.int16), res[1][0].view(torch.int16))
    assert torch.equal(res[0][1], res[1][1])
    ref_o, ref_l = oracle_decode(case, case.k_cache, case.v_cache)
    assert_attention_close(res[1][0].cpu(), res[1][1].cpu(), ref_o, ref_l, case.dtype, "twice")
