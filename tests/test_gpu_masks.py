"""GPU: the further mask modifiers against the float64 oracle.

Prefix-LM (a bidirectional prefix, causal after it), packed documents (causal
within each document) and per-head sliding windows, in paged decode (bf16 and
fp32 pools), chunked prefill and the shared-prefix decode. Documents start on
and off tile and block edges, span the context/chunk boundary and are as short
as one token; per-head windows differ inside one unit of the prefill (the two
heads of a pair) and inside one decode segment (the heads of a GQA group).
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_gather_b200 as pkv
from paged_kv_cache_gather_b200 import inputs as I
from parity import (assert_attention_close, mask_kwargs, mask_of, oracle_after_append,
                    oracle_decode, run_decode, to_dev)
from test_gpu_prefill import check_full, run_prefill

pytestmark = pytest.mark.gpu


def check_decode(case, dev):
    out, lse, _, _ = run_decode(case, dev)
    kc, vc = oracle_after_append(case)
    ref_o, ref_l = oracle_decode(case, kc, vc)
    assert_attention_close(out, lse, ref_o, ref_l, case.dtype, case.name)
    return out, lse


def ragged_decode(seed, lens, hq=32, hkv=8, bs=16, peaky=False, dtype=torch.bfloat16, d=128):
    nb = sum((L + bs - 1) // bs for L in lens) + 16
    return I.make_decode_case(f"masks_{seed}", lens=lens, num_q_heads=hq, num_kv_heads=hkv,
                              head_dim=d, block_size=bs, num_blocks=nb, dtype=dtype, seed=seed,
                              peaky=peaky)


# ------------------------------------------------------------------------ decode

@pytest.mark.parametrize("peaky", [False, True])
def test_decode_documents(cuda_device, peaky):
    lens = [1, 15, 16, 17, 300, 1029, 2048, 3333]
    case = ragged_decode(41, lens, peaky=peaky)
    off, st = I.document_starts(lens, 5, mean_doc=150)
    check_decode(I.with_mask(case, I.MASK_DOCUMENT, doc_offsets=off, doc_starts=st), cuda_device)


def test_decode_documents_last_token_alone(cuda_device):
    # every sequence's newest token opens a new document: it sees only itself
    lens = [5, 64, 700]
    case = ragged_decode(42, lens)
    off = torch.tensor([0, 2, 4, 6], dtype=torch.int32)
    st = torch.tensor([0, 4, 0, 63, 0, 699], dtype=torch.int32)
    out, lse = check_decode(I.with_mask(case, I.MASK_DOCUMENT, doc_offsets=off, doc_starts=st),
                            cuda_device)


@pytest.mark.parametrize("bs", [8, 32])
def test_decode_documents_block_sizes(cuda_device, bs):
    lens = [33, 250, 1000]
    case = ragged_decode(43 + bs, lens, bs=bs, peaky=True)
    off, st = I.document_starts(lens, 6, mean_doc=40, first_at_zero=False)
    check_decode(I.with_mask(case, I.MASK_DOCUMENT, doc_offsets=off, doc_starts=st), cuda_device)


def test_decode_prefix_lm(cuda_device):
    lens = [1, 77, 1500]
    case = ragged_decode(44, lens, peaky=True)
    plen = torch.tensor([0, 76, 4000], dtype=torch.int32)
    check_decode(I.with_mask(case, I.MASK_PREFIX_LM, prefix_len=plen), cuda_device)


@pytest.mark.parametrize("peaky", [False, True])
def test_decode_per_head_windows(cuda_device, peaky):
    lens = [1, 2, 16, 100, 1000, 4100]
    case = ragged_decode(45, lens, peaky=peaky)
    rng = np.random.default_rng(9)
    wph = torch.tensor(rng.choice([0, 1, 2, 15, 16, 17, 128, 999, 5000], size=32),
                       dtype=torch.int32)
    case.window = 7  # overridden by the per-head windows
    check_decode(I.with_mask(case, I.MASK_SLIDING, window_per_head=wph), cuda_device)


def test_decode_per_head_windows_override_per_sequence(cuda_device):
    lens = [300, 900]
    case = ragged_decode(46, lens, hq=8, hkv=2)
    case.window_per_seq = torch.tensor([5, 6], dtype=torch.int32)
    wph = torch.tensor([1, 50, 0, 299, 3, 3, 700, 64], dtype=torch.int32)
    check_decode(I.with_mask(case, I.MASK_SLIDING, window_per_head=wph), cuda_device)


def test_decode_fp32_documents_and_per_head_windows(cuda_device):
    lens = [40, 128]
    case = ragged_decode(47, lens, hq=4, hkv=4, d=64, dtype=torch.float32)
    off, st = I.document_starts(lens, 7, mean_doc=30)
    check_decode(I.with_mask(case, I.MASK_DOCUMENT, doc_offsets=off, doc_starts=st), cuda_device)
    case = ragged_decode(48, lens, hq=4, hkv=4, d=64, dtype=torch.float32)
    wph = torch.tensor([1, 0, 33, 7], dtype=torch.int32)
    check_decode(I.with_mask(case, I.MASK_SLIDING, window_per_head=wph), cuda_device)


# ----------------------------------------------------------------------- prefill

def prefill_case(seed, ctx, ql, hq=8, hkv=2, bs=16, peaky=False):
    nb = sum((c + q + bs - 1) // bs for c, q in zip(ctx, ql)) + 8
    return I.make_prefill_case(f"pmask_{seed}", ctx_lens=ctx, q_lens=ql, num_q_heads=hq,
                               num_kv_heads=hkv, head_dim=128, block_size=bs, num_blocks=nb,
                               seed=seed, peaky=peaky)


@pytest.mark.parametrize("peaky", [False, True])
def test_prefill_documents(cuda_device, peaky):
    ctx, ql = [0, 100, 700, 1000], [300, 200, 333, 128]
    case = prefill_case(51, ctx, ql, peaky=peaky)
    off, st = I.document_starts([c + q for c, q in zip(ctx, ql)], 8, mean_doc=90)
    check_full(I.with_mask(case, I.MASK_DOCUMENT, doc_offsets=off, doc_starts=st), cuda_device)


def test_prefill_documents_on_tile_edges_and_single_tokens(cuda_device):
    ctx, ql = [256, 128], [384, 257]
    case = prefill_case(52, ctx, ql, hq=4, hkv=4)
    off = torch.tensor([0, 7, 12], dtype=torch.int32)
    st = torch.tensor([0, 127, 128, 129, 256, 257, 511,   # sequence 0 (640 tokens)
                       0, 1, 2, 128, 384], dtype=torch.int32)
    check_full(I.with_mask(case, I.MASK_DOCUMENT, doc_offsets=off, doc_starts=st), cuda_device)


@pytest.mark.parametrize("plen", [[0, 0, 0], [50, 300, 1000], [5000, 5000, 5000],
                                  [100, 129, 700]])
def test_prefill_prefix_lm(cuda_device, plen):
    ctx, ql = [0, 200, 600], [300, 257, 140]
    case = prefill_case(53, ctx, ql, peaky=True)
    check_full(I.with_mask(case, I.MASK_PREFIX_LM,
                           prefix_len=torch.tensor(plen, dtype=torch.int32)), cuda_device)


@pytest.mark.parametrize("hq,hkv", [(8, 2), (6, 2), (4, 4)])
def test_prefill_per_head_windows(cuda_device, hq, hkv):
    ctx, ql = [0, 300, 900], [260, 129, 200]
    case = prefill_case(54 + hq, ctx, ql, hq=hq, hkv=hkv, peaky=True)
    rng = np.random.default_rng(hq)
    wph = torch.tensor(rng.choice([0, 1, 100, 128, 129, 700], size=hq), dtype=torch.int32)
    check_full(I.with_mask(case, I.MASK_SLIDING, window_per_head=wph), cuda_device)


def test_prefill_long_documents_sampled_rows(cuda_device):
    import oracle
    ctx, ql = [6000, 3000], [1024, 2048]
    case = prefill_case(55, ctx, ql, hq=32, hkv=8, peaky=True)
    off, st = I.document_starts([c + q for c, q in zip(ctx, ql)], 9, mean_doc=1500)
    I.with_mask(case, I.MASK_DOCUMENT, doc_offsets=off, doc_starts=st)
    out, lse = run_prefill(case, cuda_device)
    rng = np.random.default_rng(3)
    rows = [(b, int(rng.integers(0, 32)), int(rng.integers(0, ql[b]))) for b in (0, 1)
            for _ in range(16)]
    res = oracle.paged_prefill_rows(case.q, case.k_new, case.v_new, case.k_cache, case.v_cache,
                                    case.block_tables, case.ctx_lens, case.q_lens, case.scale,
                                    case.mask_kind, rows=rows, **mask_kwargs(case))
    starts = np.concatenate([[0], np.cumsum(ql)])
    go = torch.stack([out[starts[b] + i, h] for b, h, i in rows])
    gl = torch.stack([lse[starts[b] + i, h] for b, h, i in rows])
    assert_attention_close(go, gl, np.stack([res[r][0] for r in rows]),
                           np.array([res[r][1] for r in rows]), torch.bfloat16, case.name)


def test_prefill_mask_arrays_required(cuda_device):
    case = prefill_case(56, [10], [10])
    t = to_dev(case, cuda_device)
    with pytest.raises(ValueError):
        pkv.paged_attention_prefill(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"],
                                    t["block_tables"], t["ctx_lens"], t["q_lens"],
                                    pkv.MaskMod(pkv.MaskMod.DOCUMENT))


# ------------------------------------------------------------ shared-prefix decode

def test_shared_prefix_with_prefix_lm_equals_causal(cuda_device):
    case = I.make_shared_prefix_case("sp_plm", group_sizes=[3, 2], prefix_lens=[100, 37],
                                     suffix_lens=[4, 5, 6, 7, 8], seed=57, peaky=True)
    I.with_mask(case, I.MASK_PREFIX_LM, prefix_len=torch.tensor([50] * 5, dtype=torch.int32))
    t = to_dev(case, cuda_device)
    out, lse = pkv.paged_attention_decode_shared_prefix(
        t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["seq_lens"],
        case.extra["group_start"].to(cuda_device), case.extra["shared_len"].to(cuda_device),
        3, case.scale, mask_of(case, t))
    ref_o, ref_l = oracle_decode(case, case.k_cache, case.v_cache)
    assert_attention_close(out.cpu(), lse.cpu(), ref_o, ref_l, case.dtype, case.name)
