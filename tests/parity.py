"""Helpers shared by the GPU parity tests: move a workload to the device, run
the library's calls, compare with the float64 oracle at the stated bounds."""

import numpy as np
import torch

import oracle
import paged_kv_cache_gather_b200 as pkv

# Tolerances: fp32 max-abs 1e-5; bf16 |out-ref| <= 2e-2 + 2e-2|ref|; LSE 1e-3;
# and, because N(0,1) outputs over thousands of keys are ~1e-2 in size, a
# normwise relative bound of 1e-2 per (row, head).
FP32_ATOL = 1e-5
BF16_ATOL = 2e-2
BF16_RTOL = 2e-2
LSE_ATOL = 1e-3
NORM_RTOL = 1e-2


MASK_EXTRA = ("window_per_head", "prefix_len", "doc_offsets", "doc_starts")


def to_dev(case, dev):
    d = {}
    for name in ("k_cache", "v_cache", "block_tables", "seq_lens", "q", "k_new", "v_new",
                 "slot_mapping", "ctx_lens", "q_lens", "window_per_seq"):
        t = getattr(case, name)
        d[name] = None if t is None else t.to(dev).contiguous()
    extra = case.extra.get("mask", {})
    for name in MASK_EXTRA:
        t = extra.get(name)
        d[name] = None if t is None else t.to(dev).contiguous()
    return d


def mask_of(case, dev_tensors):
    return pkv.MaskMod(case.mask_kind, case.window, dev_tensors["window_per_seq"],
                       *(dev_tensors.get(n) for n in MASK_EXTRA))


def mask_kwargs(case):
    """The further mask arguments of the oracle calls (CPU tensors or None)."""
    extra = case.extra.get("mask", {})
    return {n: extra.get(n) for n in MASK_EXTRA}


def assert_attention_close(out, lse, ref_out, ref_lse, dtype, what=""):
    """out/lse: GPU results moved to CPU (any float dtype); refs: float64 arrays."""
    o = out.float().double().numpy().reshape(ref_out.shape)
    l = lse.double().numpy().reshape(ref_lse.shape)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(l), fin), f"{what}: lse finiteness differs"
    assert np.all(np.abs(l[fin] - ref_lse[fin]) <= LSE_ATOL), \
        f"{what}: lse max err {np.max(np.abs(l[fin] - ref_lse[fin]))}"
    err = np.abs(o - ref_out)
    if dtype == torch.float32:
        assert err.max() <= FP32_ATOL, f"{what}: max abs err {err.max()}"
        return
    bound = BF16_ATOL + BF16_RTOL * np.abs(ref_out)
    assert np.all(err <= bound), f"{what}: worst excess {np.max(err - bound)}"
    # normwise relative error per row/head (rows with a zero reference are exact zeros)
    num = np.linalg.norm((o - ref_out).reshape(-1, ref_out.shape[-1]), axis=1)
    den = np.linalg.norm(ref_out.reshape(-1, ref_out.shape[-1]), axis=1)
    nz = den > 0
    assert np.all(num[~nz] == 0), f"{what}: nonzero output where the reference is zero"
    if nz.any():
        rel = num[nz] / den[nz]
        assert rel.max() <= NORM_RTOL, f"{what}: normwise rel err {rel.max()}"


def run_decode(case, dev, do_append=True, dbg=True):
    """Append each sequence's newest token (when the case has one), then decode.
    Returns (out, lse, k_cache_after, v_cache_after) on the CPU."""
    t = to_dev(case, dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev) if dbg else None
    if do_append and case.k_new is not None:
        pkv.paged_kv_append(t["k_new"], t["v_new"], t["slot_mapping"], t["k_cache"],
                            t["v_cache"], dbg_err=err)
    out, lse = pkv.paged_attention_decode(t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                          t["seq_lens"], case.scale, mask_of(case, t),
                                          dbg_err=err)
    torch.cuda.synchronize()
    if dbg:
        pkv.read_dbg(err)
    return out.cpu(), lse.cpu(), t["k_cache"], t["v_cache"]


def oracle_after_append(case):
    if case.k_new is None:
        return case.k_cache, case.v_cache
    return oracle.kv_append(case.k_new, case.v_new, case.slot_mapping, case.k_cache,
                            case.v_cache)


def oracle_decode(case, kc, vc, rows=None):
    if rows is None:
        return oracle.paged_decode(case.q, kc, vc, case.block_tables, case.seq_lens, case.scale,
                                   case.mask_kind, case.window, case.window_per_seq,
                                   **mask_kwargs(case))
    return oracle.paged_decode_rows(case.q, kc, vc, case.block_tables, case.seq_lens, case.scale,
                                    case.mask_kind, case.window, case.window_per_seq, rows=rows,
                                    **mask_kwargs(case))
