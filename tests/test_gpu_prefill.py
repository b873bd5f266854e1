"""GPU: paged chunked prefill (tcgen05 kernel) against the float64 oracle.

Small cases are compared in full: contexts that are empty, shorter than a
tile, not multiples of the block or tile size; chunks of 1 token up to several
tiles; causal, no mask and sliding windows; group sizes with two heads per CTA
(even) and one (odd); block sizes 8..64. The long-context workload (4 x 30720
cached + 2048 new, 32/8 heads) is checked on whole 128-row tiles at all 32
heads (first, middle and last tile of every sequence) and on sampled rows
the oracle computes one by one, plain and "peaky". Also: pool rows past the context end that hold
NaN must not leak into the result, and bad block ids are flagged.
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_gather_b200 as pkv
from paged_kv_cache_gather_b200 import inputs as I
from parity import assert_attention_close, mask_kwargs, mask_of, to_dev

pytestmark = pytest.mark.gpu


def run_prefill(case, dev, append_first=True):
    t = to_dev(case, dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    if append_first:
        pkv.paged_kv_append(t["k_new"], t["v_new"], t["slot_mapping"], t["k_cache"],
                            t["v_cache"], dbg_err=err)
    out, lse = pkv.paged_attention_prefill(t["q"], t["k_new"], t["v_new"], t["k_cache"],
                                           t["v_cache"], t["block_tables"], t["ctx_lens"],
                                           t["q_lens"], mask_of(case, t), case.scale,
                                           dbg_err=err)
    torch.cuda.synchronize()
    pkv.read_dbg(err)
    return out.cpu(), lse.cpu()


def check_full(case, dev):
    out, lse = run_prefill(case, dev)
    ref_o, ref_l = oracle.paged_prefill(case.q, case.k_new, case.v_new, case.k_cache,
                                        case.v_cache, case.block_tables, case.ctx_lens,
                                        case.q_lens, case.scale, case.mask_kind, case.window,
                                        case.window_per_seq, **mask_kwargs(case))
    assert_attention_close(out, lse, ref_o, ref_l, torch.bfloat16, case.name)
    return out, lse


SMALL = [
    # ctx_lens, q_lens, Hq, Hkv, bs, mask, window
    ([0], [128], 8, 2, 16, I.MASK_CAUSAL, 0),
    ([128], [128], 8, 2, 16, I.MASK_CAUSAL, 0),
    ([300, 0, 1000], [200, 77, 1], 8, 2, 16, I.MASK_CAUSAL, 0),
    ([513, 64], [257, 129], 8, 2, 16, I.MASK_NONE, 0),
    ([1000, 250], [300, 140], 8, 2, 16, I.MASK_SLIDING, 200),
    ([1000, 250], [300, 140], 8, 2, 16, I.MASK_SLIDING, 1),
    ([700, 33], [150, 260], 8, 8, 16, I.MASK_CAUSAL, 0),          # g = 1: one head per CTA
    ([700, 33], [150, 260], 12, 4, 16, I.MASK_CAUSAL, 0),         # g = 3
    ([700, 33], [150, 260], 32, 4, 16, I.MASK_CAUSAL, 0),         # g = 8
    ([501, 96], [130, 20], 8, 2, 8, I.MASK_CAUSAL, 0),            # block 8
    ([501, 96], [130, 20], 8, 2, 32, I.MASK_SLIDING, 333),        # block 32
    ([1024, 77], [128, 300], 8, 2, 64, I.MASK_CAUSAL, 0),         # block 64
]


@pytest.mark.parametrize("ctx,ql,hq,hkv,bs,kind,w", SMALL)
def test_small_cases_full_compare(cuda_device, ctx, ql, hq, hkv, bs, kind, w):
    nb = sum(-(-(c + q) // bs) for c, q in zip(ctx, ql)) + 8
    case = I.make_prefill_case("pf", ctx_lens=ctx, q_lens=ql, num_q_heads=hq, num_kv_heads=hkv,
                               head_dim=128, block_size=bs, num_blocks=nb, seed=sum(ctx) + hq,
                               mask_kind=kind, window=w)
    check_full(case, cuda_device)


def test_small_peaky(cuda_device):
    case = I.make_prefill_case("pf_peaky", ctx_lens=[900, 2000], q_lens=[300, 256],
                               num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                               num_blocks=256, seed=3, peaky=True)
    check_full(case, cuda_device)


def test_per_sequence_windows(cuda_device):
    case = I.make_prefill_case("pf_wps", ctx_lens=[400, 900, 0], q_lens=[200, 130, 140],
                               num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                               num_blocks=160, seed=5, mask_kind=I.MASK_SLIDING,
                               window_per_seq=torch.tensor([0, 150, 64], dtype=torch.int32))
    check_full(case, cuda_device)


def test_stale_nan_rows_past_context_end_do_not_leak(cuda_device):
    """The prefill reads the context through the table before the chunk is
    appended; rows of the last context block past the context end hold NaN."""
    case = I.make_prefill_case("pf_nan", ctx_lens=[1003, 77], q_lens=[150, 60], num_q_heads=8,
                               num_kv_heads=2, head_dim=128, block_size=16, num_blocks=128,
                               seed=9)
    tabs = case.block_tables.numpy()
    for b, C in enumerate(case.ctx_lens.tolist()):
        blk = int(tabs[b, C // 16])
        case.v_cache[blk, :, C % 16:] = float("nan")
        case.k_cache[blk, :, C % 16:] = float("nan")
    out, lse = run_prefill(case, cuda_device, append_first=False)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    ref_o, ref_l = oracle.paged_prefill(case.q, case.k_new, case.v_new, case.k_cache,
                                        case.v_cache, case.block_tables, case.ctx_lens,
                                        case.q_lens, case.scale, case.mask_kind)
    assert_attention_close(out, lse, ref_o, ref_l, torch.bfloat16, case.name)


def test_prefill_is_deterministic(cuda_device):
    case = I.make_prefill_case("pf_det", ctx_lens=[777], q_lens=[333], num_q_heads=8,
                               num_kv_heads=2, head_dim=128, block_size=16, num_blocks=80,
                               seed=11)
    o1, l1 = run_prefill(case, cuda_device)
    o2, l2 = run_prefill(case, cuda_device)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


def test_bad_block_id_is_flagged(cuda_device):
    case = I.make_prefill_case("pf_bad", ctx_lens=[300], q_lens=[50], num_q_heads=8,
                               num_kv_heads=2, head_dim=128, block_size=16, num_blocks=40,
                               seed=1)
    case.block_tables[0, 2] = 10_000
    t = to_dev(case, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    pkv.paged_attention_prefill(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"],
                                t["block_tables"], t["ctx_lens"], t["q_lens"],
                                mask_of(case, t), case.scale, dbg_err=err)
    torch.cuda.synchronize()
    assert err.item() & pkv._lib.PKV_DBG_BLOCK_ID


def sampled_rows(case, n_per_seq, seed):
    rng = np.random.default_rng(seed)
    rows = []
    for b in range(case.batch):
        Q = int(case.q_lens[b])
        picks = {0, Q - 1, min(127, Q - 1), min(128, Q - 1)}
        picks |= set(rng.integers(0, Q, size=n_per_seq).tolist())
        for i in sorted(picks):
            rows.append((b, int(rng.integers(0, case.num_q_heads)), int(i)))
    return rows


@pytest.mark.slow
@pytest.mark.parametrize("peaky", [False, True])
def test_long_context_workload_sampled_rows(cuda_device, peaky):
    case = I.config5(peaky=peaky)
    out, lse = run_prefill(case, cuda_device)
    rows = sampled_rows(case, 12, 5 + int(peaky))
    res = oracle.paged_prefill_rows(case.q, case.k_new, case.v_new, case.k_cache, case.v_cache,
                                    case.block_tables, case.ctx_lens, case.q_lens, case.scale,
                                    case.mask_kind, rows=rows)
    starts = np.concatenate([[0], np.cumsum(case.q_lens.numpy())])
    go = torch.stack([out[starts[b] + i, h] for b, h, i in rows])
    gl = torch.stack([lse[starts[b] + i, h] for b, h, i in rows])
    ro = np.stack([res[r][0] for r in rows])
    rl = np.array([res[r][1] for r in rows])
    assert_attention_close(go, gl, ro, rl, torch.bfloat16, case.name)
    # every row is finite and every lse plausible (>= its diagonal score's log-sum)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


@pytest.mark.slow
@pytest.mark.parametrize("peaky", [False, True])
def test_long_context_workload_whole_tiles(cuda_device, peaky):
    """Whole query tiles of the long-context workload, element by element:
    for each of the 4 sequences the first, a middle and the last 128-row tile,
    every one of the 32 query heads (both heads of every GQA pair a CTA runs,
    the full span of ~256 key tiles with the lazy rescale, the causal diagonal
    tile), against the oracle's block-of-rows entry."""
    case = I.config5(peaky=peaky)
    out, lse = run_prefill(case, cuda_device)
    starts = np.concatenate([[0], np.cumsum(case.q_lens.numpy())])
    for b in range(case.batch):
        Q = int(case.q_lens[b])
        n_qt = (Q + 127) // 128
        for qt in sorted({0, n_qt // 2, n_qt - 1}):
            i0, i1 = qt * 128, min(qt * 128 + 128, Q)
            ro, rl = oracle.paged_prefill_tile(case.q, case.k_new, case.v_new, case.k_cache,
                                               case.v_cache, case.block_tables, case.ctx_lens,
                                               case.q_lens, case.scale, case.mask_kind, b, i0, i1)
            go = out[starts[b] + i0:starts[b] + i1]
            gl = lse[starts[b] + i0:starts[b] + i1]
            assert_attention_close(go, gl, ro, rl, torch.bfloat16,
                                   f"{case.name} b{b} tile{qt} peaky={peaky}")


def test_decode_equals_last_row_of_prefill(cuda_device):
    """A one-token-chunk prefill and a decode of the same (appended) token agree."""
    case = I.make_prefill_case("pf_vs_dec", ctx_lens=[999, 130], q_lens=[1, 1], num_q_heads=8,
                               num_kv_heads=2, head_dim=128, block_size=16, num_blocks=80,
                               seed=13)
    out_p, lse_p = run_prefill(case, cuda_device)
    t = to_dev(case, cuda_device)
    pkv.paged_kv_append(t["k_new"], t["v_new"], t["slot_mapping"], t["k_cache"], t["v_cache"])
    out_d, lse_d = pkv.paged_attention_decode(t["q"], t["k_cache"], t["v_cache"],
                                              t["block_tables"], t["seq_lens"], case.scale,
                                              pkv.causal())
    torch.cuda.synchronize()
    assert (out_p.float() - out_d.cpu().float()).abs().max() < 2e-2
    assert (lse_p - lse_d.cpu()).abs().max() < 1e-3
