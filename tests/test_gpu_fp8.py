"""GPU: E4M3 KV pools (one float32 scale per stored row).

Append: the codes and scales the GPU writes equal the oracle's quantisation
bit for bit (rounding ties, saturation, zero rows, subnormal codes), and every
other byte of the pools keeps its sentinel. Decode: attention over the decoded
values (code x row scale) matches the float64 oracle at the bf16 bounds, for
ragged lengths, block sizes 8..64, group sizes 1..8, every mask kind, peaky
queries, the full ragged workload on sampled rows, and pools whose codes and
scales were written by the append (a whole quantise -> decode step).
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_gather_b200 as pkv
from oracle import fp8 as F
from paged_kv_cache_gather_b200 import inputs as I
from parity import assert_attention_close, mask_kwargs, mask_of, to_dev

pytestmark = pytest.mark.gpu


def quantised_case(case):
    """E4M3 codes and scales of a bf16 decode case's pools (host, oracle rules)."""
    kc, ks = F.quantize_rows(case.k_cache)
    vc, vs = F.quantize_rows(case.v_cache)
    return kc, vc, ks, vs


def run_fp8(case, kc, vc, ks, vs, dev, dbg=True):
    t = to_dev(case, dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    out, lse = pkv.paged_attention_decode_fp8(
        t["q"], torch.from_numpy(kc).to(dev), torch.from_numpy(vc).to(dev),
        torch.from_numpy(ks).to(dev), torch.from_numpy(vs).to(dev), t["block_tables"],
        t["seq_lens"], case.scale, mask_of(case, t), dbg_err=err)
    torch.cuda.synchronize()
    if dbg:
        pkv.read_dbg(err)
    return out.cpu(), lse.cpu()


def oracle_fp8(case, kc, vc, ks, vs, rows=None):
    kd, vd = F.dequantize_pool(kc, ks), F.dequantize_pool(vc, vs)
    if rows is None:
        return oracle.paged_decode(case.q, kd, vd, case.block_tables, case.seq_lens, case.scale,
                                   case.mask_kind, case.window, case.window_per_seq,
                                   **mask_kwargs(case))
    return oracle.paged_decode_rows(case.q, kd, vd, case.block_tables, case.seq_lens, case.scale,
                                    case.mask_kind, case.window, case.window_per_seq, rows=rows,
                                    **mask_kwargs(case))


def check(case, dev):
    kc, vc, ks, vs = quantised_case(case)
    out, lse = run_fp8(case, kc, vc, ks, vs, dev)
    ref_o, ref_l = oracle_fp8(case, kc, vc, ks, vs)
    assert_attention_close(out, lse, ref_o, ref_l, torch.bfloat16, case.name + "_fp8")
    return out, lse


def case_of(seed, lens, hq=32, hkv=8, bs=16, peaky=False, mask=I.MASK_CAUSAL, window=0,
            wps=None):
    nb = sum((L + bs - 1) // bs for L in lens) + 8
    return I.make_decode_case(f"fp8_{seed}", lens=lens, num_q_heads=hq, num_kv_heads=hkv,
                              head_dim=128, block_size=bs, num_blocks=nb, dtype=torch.bfloat16,
                              seed=seed, mask_kind=mask, window=window, window_per_seq=wps,
                              peaky=peaky)


# ------------------------------------------------------------------------ append

def test_append_codes_and_scales_bit_exact(cuda_device):
    rng = np.random.default_rng(1)
    NB, Hkv, bs, d, T = 12, 2, 16, 128, 70
    gen = torch.Generator().manual_seed(1)
    k = (torch.randn(T, Hkv, d, generator=gen) *
         torch.from_numpy(rng.uniform(1e-3, 300, (T, Hkv, 1)).astype(np.float32))).bfloat16()
    v = (torch.randn(T, Hkv, d, generator=gen) * 3).bfloat16()
    k[5] = 0                                              # all-zero rows: scale 1, codes 0
    k[6, 0, :4] = torch.tensor([448.0, -448.0, 464.0, 1e-30]).bfloat16()  # saturation, tiny
    v[7, 1] = torch.linspace(-2, 2, d).bfloat16()         # many exact halfway points
    slots = torch.from_numpy(rng.permutation(NB * bs)[:T].astype(np.int64))
    slots[3] = -1                                          # padding
    kc0 = np.full((NB, Hkv, bs, d), 0x5A, dtype=np.uint8)
    ks0 = np.full((NB, Hkv, bs), -7.0, dtype=np.float32)
    dev = cuda_device
    kc, vc = torch.from_numpy(kc0.copy()).to(dev), torch.from_numpy(kc0.copy()).to(dev)
    ks, vs = torch.from_numpy(ks0.copy()).to(dev), torch.from_numpy(ks0.copy()).to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    pkv.paged_kv_append_fp8(k.to(dev), v.to(dev), slots.to(dev), kc, vc, ks, vs, dbg_err=err)
    torch.cuda.synchronize()
    pkv.read_dbg(err)
    ekc, evc, eks, evs = F.kv_append_fp8(k, v, slots, kc0, kc0, ks0, ks0)
    assert np.array_equal(kc.cpu().numpy(), ekc)
    assert np.array_equal(vc.cpu().numpy(), evc)
    assert np.array_equal(ks.cpu().numpy().view(np.int32), eks.view(np.int32))
    assert np.array_equal(vs.cpu().numpy().view(np.int32), evs.view(np.int32))


def test_append_bad_slot_flagged(cuda_device):
    dev = cuda_device
    kc = torch.zeros(2, 1, 16, 128, dtype=torch.uint8, device=dev)
    ks = torch.zeros(2, 1, 16, dtype=torch.float32, device=dev)
    k = torch.ones(2, 1, 128, dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    pkv.paged_kv_append_fp8(k, k, torch.tensor([5, 32], device=dev), kc, kc.clone(), ks,
                            ks.clone(), dbg_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pkv._lib.PKV_DBG_SLOT


# ------------------------------------------------------------------------ decode

@pytest.mark.parametrize("peaky", [False, True])
def test_decode_ragged(cuda_device, peaky):
    check(case_of(3, [1, 2, 15, 16, 17, 100, 1000, 3000], peaky=peaky), cuda_device)


@pytest.mark.parametrize("bs", [8, 32, 64])
def test_decode_block_sizes(cuda_device, bs):
    check(case_of(4 + bs, [7, 64, 500, 1111], bs=bs, peaky=True), cuda_device)


@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 8), (24, 4), (64, 8)])
def test_decode_group_sizes(cuda_device, hq, hkv):
    check(case_of(5 + hq, [33, 700], hq=hq, hkv=hkv, peaky=True), cuda_device)


def test_decode_masks(cuda_device):
    lens = [1, 300, 2000]
    wps = torch.tensor([0, 50, 1000], dtype=torch.int32)
    check(case_of(6, lens, mask=I.MASK_SLIDING, wps=wps, peaky=True), cuda_device)
    case = case_of(7, lens, peaky=True)
    off, st = I.document_starts(lens, 7, mean_doc=200)
    check(I.with_mask(case, I.MASK_DOCUMENT, doc_offsets=off, doc_starts=st), cuda_device)
    case = case_of(8, lens, peaky=True)
    wph = torch.tensor([1, 0, 16, 17, 300] * 6 + [2, 64], dtype=torch.int32)
    check(I.with_mask(case, I.MASK_SLIDING, window_per_head=wph), cuda_device)
    case = case_of(9, lens, mask=I.MASK_NONE, peaky=True)
    check(case, cuda_device)


def test_decode_empty_sequence(cuda_device):
    out, lse = check(case_of(10, [0, 5]), cuda_device)
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))


def test_quantise_then_decode_step(cuda_device):
    # the append writes every row of the pool, the decode reads them back; the
    # oracle quantises the same bf16 rows by its own rules
    case = case_of(11, [40, 333, 1024], peaky=True)
    dev = cuda_device
    NB, Hkv, bs, d = case.k_cache.shape
    rows = case.k_cache.permute(0, 2, 1, 3).reshape(NB * bs, Hkv, d).contiguous()
    vrows = case.v_cache.permute(0, 2, 1, 3).reshape(NB * bs, Hkv, d).contiguous()
    slots = torch.arange(NB * bs, dtype=torch.int64)
    kc = torch.zeros(NB, Hkv, bs, d, dtype=torch.uint8, device=dev)
    vc = torch.zeros_like(kc)
    ks = torch.zeros(NB, Hkv, bs, dtype=torch.float32, device=dev)
    vs = torch.zeros_like(ks)
    pkv.paged_kv_append_fp8(rows.to(dev), vrows.to(dev), slots.to(dev), kc, vc, ks, vs)
    t = to_dev(case, dev)
    out, lse = pkv.paged_attention_decode_fp8(t["q"], kc, vc, ks, vs, t["block_tables"],
                                              t["seq_lens"], case.scale, mask_of(case, t))
    torch.cuda.synchronize()
    qk, qv, sk, sv = quantised_case(case)
    ref_o, ref_l = oracle_fp8(case, qk, qv, sk, sv)
    assert_attention_close(out.cpu(), lse.cpu(), ref_o, ref_l, torch.bfloat16, "fp8 step")
    # and the bf16 result of the unquantised pools is close (E4M3 error ~2^-4)
    ref_b, _ = oracle.paged_decode(case.q, case.k_cache, case.v_cache, case.block_tables,
                                   case.seq_lens, case.scale, case.mask_kind)
    rel = np.linalg.norm(out.cpu().float().numpy() - ref_b) / np.linalg.norm(ref_b)
    assert rel < 0.1


@pytest.mark.slow
def test_decode_ragged_workload_sampled_rows(cuda_device):
    # the ragged workload at full size; the pools hold random valid E4M3 codes
    # with random row scales (a valid pool without quantising 1.3 G values on
    # the host); the oracle decodes only the blocks of the sampled sequences
    case = I.config3(peaky=False)
    rng = np.random.default_rng(12)
    shape = tuple(case.k_cache.shape)
    kc = rng.integers(0, 256, size=shape, dtype=np.uint8)
    vc = rng.integers(0, 256, size=shape, dtype=np.uint8)
    for c in (kc, vc):
        c[c == 0x7F] = 0x7E
        c[c == 0xFF] = 0xFE
    ks = rng.uniform(1e-3, 1e-2, size=shape[:3]).astype(np.float32)
    vs = rng.uniform(1e-3, 1e-2, size=shape[:3]).astype(np.float32)
    out, lse = run_fp8(case, kc, vc, ks, vs, cuda_device)
    seqs = rng.choice(case.batch, 12, replace=False)
    tabs = case.block_tables.numpy()
    lens = case.seq_lens.numpy()
    for b in seqs:
        nblk = -(-int(lens[b]) // shape[2])
        used = tabs[b, :nblk]
        kd = F.dequantize_pool(kc[used], ks[used])
        vd = F.dequantize_pool(vc[used], vs[used])
        sub_tab = np.arange(nblk)[None, :]
        h = int(rng.integers(0, case.num_q_heads))
        res = oracle.paged_decode_rows(case.q[b:b + 1], kd, vd, sub_tab, case.seq_lens[b:b + 1],
                                       case.scale, case.mask_kind, case.window,
                                       None if case.window_per_seq is None
                                       else case.window_per_seq[b:b + 1], rows=[(0, h)])
        ro, rl = res[(0, h)]
        assert_attention_close(out[b, h][None], lse[b, h][None], ro[None], np.array([rl]),
                               torch.bfloat16, f"fp8 cfg3 b{b} h{h}")


def test_plain_calls_reject_e4m3_pools(cuda_device):
    case = case_of(13, [20])
    kc, vc, ks, vs = quantised_case(case)
    t = to_dev(case, cuda_device)
    with pytest.raises((ValueError, pkv.PagedKVError)):
        pkv.paged_attention_decode(t["q"], torch.from_numpy(kc).to(cuda_device),
                                   torch.from_numpy(vc).to(cuda_device), t["block_tables"],
                                   t["seq_lens"])


@pytest.mark.parametrize("w", [0, 100])
def test_nan_codes_and_scales_outside_the_visible_range(cuda_device, w):
    # rows of a visible key's tile that the query must not see hold NaN codes
    # (0x7f) and NaN scales: the decode zeroes them before the P*V product
    lens = [5, 17, 300, 1000]
    case = case_of(14 + w, lens, mask=I.MASK_SLIDING if w else I.MASK_CAUSAL, window=w,
                   peaky=True)
    kc, vc, ks, vs = quantised_case(case)
    ref_o, ref_l = oracle_fp8(case, kc, vc, ks, vs)  # on the clean pools
    bs = kc.shape[2]
    tab = case.block_tables.numpy()
    n = 0
    for b, L in enumerate(lens):
        lo = max(0, L - w) if w else 0
        for pos in list(range(L, -(-L // bs) * bs)) + list(range((lo // bs) * bs, lo)):
            blk = int(tab[b, pos // bs])
            kc[blk, :, pos % bs] = 0x7F
            vc[blk, :, pos % bs] = 0x7F
            ks[blk, :, pos % bs] = np.nan
            vs[blk, :, pos % bs] = np.nan
            n += 1
    assert n > 0
    out, lse = run_fp8(case, kc, vc, ks, vs, cuda_device)
    assert_attention_close(out, lse, ref_o, ref_l, torch.bfloat16, "fp8 nan rows")
