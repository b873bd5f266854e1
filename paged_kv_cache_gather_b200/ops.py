"""Python binding of the paged KV-cache calls: argument marshalling only.

Each function checks devices, dtypes and shapes, allocates outputs with torch
when the caller passes none, and calls the C ABI of ``libpagedkv.so`` on the
current CUDA stream. Every step of the computation runs in the library's
CUDA kernels; nothing here computes attention.
"""

import ctypes
import math
from dataclasses import dataclass
from typing import Optional, Union

import numpy as np
import torch

from . import _lib as L

_DTYPES = {torch.float32: L.PKV_F32, torch.bfloat16: L.PKV_BF16, torch.uint8: L.PKV_FP8_E4M3,
           torch.float8_e4m3fn: L.PKV_FP8_E4M3}


@dataclass
class MaskMod:
    """FlexAttention-style mask modifier as data.

    kind: ``MaskMod.NONE``, ``CAUSAL``, ``SLIDING``, ``PREFIX_LM`` or
    ``DOCUMENT``. ``window`` (sliding) keeps keys with ``q_pos - k_pos <
    window``; ``<= 0`` means causal only. ``window_per_seq`` (int32 [batch])
    and ``window_per_head`` (int32 [num_q_heads]) override it, per head first.
    ``prefix_len`` (int32 [batch], prefix-LM): keys below it are visible to
    every query. ``doc_offsets`` (int32 [batch + 1]) and ``doc_starts``
    (int32, ascending per sequence): document start positions of sequence b
    are ``doc_starts[doc_offsets[b]:doc_offsets[b + 1]]``. All tensors live
    on the cache's device.
    """

    kind: int = L.PKV_MASK_NONE
    window: int = 0
    window_per_seq: Optional[torch.Tensor] = None
    window_per_head: Optional[torch.Tensor] = None
    prefix_len: Optional[torch.Tensor] = None
    doc_offsets: Optional[torch.Tensor] = None
    doc_starts: Optional[torch.Tensor] = None

    NONE = L.PKV_MASK_NONE
    CAUSAL = L.PKV_MASK_CAUSAL
    SLIDING = L.PKV_MASK_SLIDING
    PREFIX_LM = L.PKV_MASK_PREFIX_LM
    DOCUMENT = L.PKV_MASK_DOCUMENT

    def to_c(self, batch, device, num_q_heads=None):
        def arr(t, n, name):
            if t is None:
                return None
            _check(t.dtype == torch.int32 and t.device == device and t.is_contiguous()
                   and (n is None or t.numel() >= n), f"{name} must be int32 [{n}] on the device")
            return t.data_ptr()

        wph = arr(self.window_per_head, num_q_heads, "window_per_head")
        if self.kind == L.PKV_MASK_PREFIX_LM:
            _check(self.prefix_len is not None, "prefix-LM mask needs prefix_len")
        if self.kind == L.PKV_MASK_DOCUMENT:
            _check(self.doc_offsets is not None and self.doc_starts is not None,
                   "document mask needs doc_offsets and doc_starts")
        return L.MaskModC(int(self.kind), int(self.window),
                          arr(self.window_per_seq, batch, "window_per_seq"), wph,
                          arr(self.prefix_len, batch, "prefix_len"),
                          arr(self.doc_offsets, batch + 1, "doc_offsets"),
                          arr(self.doc_starts, None, "doc_starts"))


def no_mask() -> MaskMod:
    return MaskMod(L.PKV_MASK_NONE)


def causal() -> MaskMod:
    return MaskMod(L.PKV_MASK_CAUSAL)


def sliding_window(window: Union[int, torch.Tensor], per_head: Optional[torch.Tensor] = None
                   ) -> MaskMod:
    """Sliding window: a scalar, a per-sequence tensor, and/or per-head windows."""
    if isinstance(window, torch.Tensor):
        return MaskMod(L.PKV_MASK_SLIDING, 0, window, per_head)
    return MaskMod(L.PKV_MASK_SLIDING, int(window), None, per_head)


def prefix_lm(prefix_len: torch.Tensor) -> MaskMod:
    """Bidirectional prefix of ``prefix_len[b]`` keys, causal after it."""
    return MaskMod(L.PKV_MASK_PREFIX_LM, prefix_len=prefix_len)


def document(doc_offsets: torch.Tensor, doc_starts: torch.Tensor) -> MaskMod:
    """Causal within documents packed into each sequence (CSR of start positions)."""
    return MaskMod(L.PKV_MASK_DOCUMENT, doc_offsets=doc_offsets, doc_starts=doc_starts)


def _check(cond, msg):
    if not cond:
        raise ValueError(msg)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def cache_desc(k_cache: torch.Tensor) -> L.CacheDescC:
    _check(k_cache.dim() == 4, "cache must be [num_blocks, num_kv_heads, block_size, head_dim]")
    _check(k_cache.dtype in _DTYPES, f"cache dtype {k_cache.dtype} not supported")
    nb, hkv, bs, d = k_cache.shape
    return L.CacheDescC(nb, bs, hkv, d, _DTYPES[k_cache.dtype])


def _check_pool(k_cache, v_cache):
    _check(k_cache.is_cuda and v_cache.device == k_cache.device, "caches must be on one GPU")
    _check(k_cache.shape == v_cache.shape and k_cache.dtype == v_cache.dtype,
           "k_cache and v_cache must match")
    _check(k_cache.is_contiguous() and v_cache.is_contiguous(), "caches must be contiguous")


def _i32(t, name, device):
    _check(t.dtype == torch.int32 and t.device == device and t.is_contiguous(),
           f"{name} must be a contiguous int32 tensor on {device}")
    return t


def paged_kv_append(k, v, slot_mapping, k_cache, v_cache, dbg_err=None):
    """Write K/V of new tokens into their slots (exact copy; slot < 0 skips)."""
    _check_pool(k_cache, v_cache)
    dev = k_cache.device
    T = k.shape[0]
    _check(k.shape == (T, k_cache.shape[1], k_cache.shape[3]) and v.shape == k.shape,
           "k, v must be [num_tokens, num_kv_heads, head_dim]")
    _check(k.dtype == k_cache.dtype and v.dtype == k_cache.dtype, "k/v dtype must match cache")
    _check(k.is_contiguous() and v.is_contiguous() and k.device == dev and v.device == dev,
           "k, v must be contiguous on the cache's device")
    _check(slot_mapping.dtype == torch.int64 and slot_mapping.device == dev
           and slot_mapping.numel() == T and slot_mapping.is_contiguous(),
           "slot_mapping must be int64 [num_tokens] on the device")
    L.check(L.lib().paged_kv_append(_ptr(k), _ptr(v), _ptr(slot_mapping), T, _ptr(k_cache),
                                    _ptr(v_cache), cache_desc(k_cache), _ptr(dbg_err), _stream()))


def _check_scales(k_scale, v_scale, k_cache):
    nb, hkv, bs, _ = k_cache.shape
    for t, name in ((k_scale, "k_scale"), (v_scale, "v_scale")):
        _check(t is not None and t.dtype == torch.float32 and t.device == k_cache.device and
               t.is_contiguous() and t.numel() >= nb * hkv * bs,
               f"{name} must be float32 [num_blocks, num_kv_heads, block_size] on the device")


def paged_kv_append_fp8(k, v, slot_mapping, k_cache, v_cache, k_scale, v_scale, dbg_err=None):
    """Quantise bf16 tokens into E4M3 pools (one float32 scale per stored row)."""
    _check_pool(k_cache, v_cache)
    _check(k_cache.dtype in (torch.uint8, torch.float8_e4m3fn), "pools must hold E4M3 codes")
    _check_scales(k_scale, v_scale, k_cache)
    dev = k_cache.device
    T = k.shape[0]
    _check(k.shape == (T, k_cache.shape[1], k_cache.shape[3]) and v.shape == k.shape and
           k.dtype == torch.bfloat16 and v.dtype == torch.bfloat16 and k.is_contiguous() and
           v.is_contiguous() and k.device == dev and v.device == dev,
           "k, v must be contiguous bf16 [num_tokens, num_kv_heads, head_dim] on the device")
    _check(slot_mapping.dtype == torch.int64 and slot_mapping.device == dev and
           slot_mapping.numel() == T and slot_mapping.is_contiguous(),
           "slot_mapping must be int64 [num_tokens] on the device")
    L.check(L.lib().paged_kv_append_fp8(_ptr(k), _ptr(v), _ptr(slot_mapping), T, _ptr(k_cache),
                                        _ptr(v_cache), _ptr(k_scale), _ptr(v_scale),
                                        cache_desc(k_cache), _ptr(dbg_err), _stream()))


def paged_attention_decode_fp8(q, k_cache, v_cache, k_scale, v_scale, block_tables, seq_lens,
                               scale=None, mask_mod: Optional[MaskMod] = None, *, out=None,
                               lse=None, workspace=None, dbg_err=None):
    """Decode over E4M3 pools (bf16 q and out). Returns (out, lse)."""
    _check_pool(k_cache, v_cache)
    _check(k_cache.dtype in (torch.uint8, torch.float8_e4m3fn), "pools must hold E4M3 codes")
    _check_scales(k_scale, v_scale, k_cache)
    dev = k_cache.device
    _i32(block_tables, "block_tables", dev)
    _i32(seq_lens, "seq_lens", dev)
    B, Hq, d = q.shape
    _check(q.dtype == torch.bfloat16 and q.device == dev and q.is_contiguous(),
           "q must be contiguous bf16 on the cache's device")
    _check(d == k_cache.shape[3], "head_dim mismatch")
    _check(block_tables.dim() == 2 and block_tables.shape[0] == B and seq_lens.numel() == B,
           "block_tables [B, M] and seq_lens [B] must match q's batch")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    mask_mod = mask_mod or no_mask()
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = decode_workspace(B, Hq, k_cache)
    L.check(L.lib().paged_attention_decode_fp8(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), cache_desc(k_cache),
        _ptr(block_tables), block_tables.shape[1], _ptr(seq_lens), B, Hq, float(scale),
        mask_mod.to_c(B, dev, Hq), _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
        _ptr(dbg_err), _stream()))
    return out, lse


def paged_kv_gather(k_cache, v_cache, block_tables, seq_lens, out_max_len, dbg_err=None):
    """Contiguous [B, Hkv, out_max_len, d] copies of each sequence's K and V."""
    _check_pool(k_cache, v_cache)
    dev = k_cache.device
    _i32(block_tables, "block_tables", dev)
    _i32(seq_lens, "seq_lens", dev)
    B = seq_lens.numel()
    _check(block_tables.dim() == 2 and block_tables.shape[0] == B, "block_tables must be [B, M]")
    nb, hkv, bs, d = k_cache.shape
    ko = torch.empty(B, hkv, out_max_len, d, dtype=k_cache.dtype, device=dev)
    vo = torch.empty_like(ko)
    L.check(L.lib().paged_kv_gather(_ptr(k_cache), _ptr(v_cache), cache_desc(k_cache),
                                    _ptr(block_tables), block_tables.shape[1], _ptr(seq_lens), B,
                                    int(out_max_len), _ptr(ko), _ptr(vo), _ptr(dbg_err),
                                    _stream()))
    return ko, vo


def paged_kv_copy_blocks(k_cache, v_cache, block_pairs, dbg_err=None):
    """Copy-on-write: copy every KV head of block src to block dst for each
    (src, dst) row of ``block_pairs`` (int32 [n, 2] on the device)."""
    _check_pool(k_cache, v_cache)
    dev = k_cache.device
    if isinstance(block_pairs, (list, tuple)):
        block_pairs = torch.tensor(block_pairs, dtype=torch.int32, device=dev).view(-1, 2)
    _check(block_pairs.dtype == torch.int32 and block_pairs.device == dev and
           block_pairs.is_contiguous() and block_pairs.dim() == 2 and block_pairs.shape[1] == 2,
           "block_pairs must be a contiguous int32 [n, 2] tensor on the device")
    L.check(L.lib().paged_kv_copy_blocks(_ptr(k_cache), _ptr(v_cache), cache_desc(k_cache),
                                         _ptr(block_pairs), block_pairs.shape[0], _ptr(dbg_err),
                                         _stream()))


def paged_kv_copy_blocks_fp8(k_cache, v_cache, k_scale, v_scale, block_pairs, dbg_err=None):
    """Copy-on-write on E4M3 pools: the codes and the row scales of block src
    go to block dst for each (src, dst) row of ``block_pairs``."""
    _check_pool(k_cache, v_cache)
    _check(k_cache.dtype in (torch.uint8, torch.float8_e4m3fn), "pools must hold E4M3 codes")
    _check_scales(k_scale, v_scale, k_cache)
    dev = k_cache.device
    if isinstance(block_pairs, (list, tuple)):
        block_pairs = torch.tensor(block_pairs, dtype=torch.int32, device=dev).view(-1, 2)
    _check(block_pairs.dtype == torch.int32 and block_pairs.device == dev and
           block_pairs.is_contiguous() and block_pairs.dim() == 2 and block_pairs.shape[1] == 2,
           "block_pairs must be a contiguous int32 [n, 2] tensor on the device")
    L.check(L.lib().paged_kv_copy_blocks_fp8(_ptr(k_cache), _ptr(v_cache), _ptr(k_scale),
                                             _ptr(v_scale), cache_desc(k_cache),
                                             _ptr(block_pairs), block_pairs.shape[0],
                                             _ptr(dbg_err), _stream()))


def decode_workspace_size(batch, num_q_heads, k_cache):
    return int(L.lib().paged_attention_decode_workspace_size(batch, num_q_heads,
                                                             cache_desc(k_cache)))


def decode_workspace(batch, num_q_heads, k_cache):
    n = decode_workspace_size(batch, num_q_heads, k_cache)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=k_cache.device)


def paged_attention_decode(q, k_cache, v_cache, block_tables, seq_lens, scale=None,
                           mask_mod: Optional[MaskMod] = None, *, out=None, lse=None,
                           workspace=None, dbg_err=None):
    """One query token per sequence over its paged context. Returns (out, lse)."""
    _check_pool(k_cache, v_cache)
    dev = k_cache.device
    _i32(block_tables, "block_tables", dev)
    _i32(seq_lens, "seq_lens", dev)
    B, Hq, d = q.shape
    _check(q.dtype == k_cache.dtype and q.device == dev and q.is_contiguous(),
           "q must be contiguous, on the cache's device, in the cache dtype")
    _check(d == k_cache.shape[3], "head_dim mismatch")
    _check(block_tables.dim() == 2 and block_tables.shape[0] == B and seq_lens.numel() == B,
           "block_tables [B, M] and seq_lens [B] must match q's batch")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    mask_mod = mask_mod or no_mask()
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = decode_workspace(B, Hq, k_cache)
    L.check(L.lib().paged_attention_decode(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), cache_desc(k_cache), _ptr(block_tables),
        block_tables.shape[1], _ptr(seq_lens), B, Hq, float(scale), mask_mod.to_c(B, dev, Hq),
        _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), _ptr(dbg_err), _stream()))
    return out, lse


def paged_attention_decode_append(q, k_new, v_new, k_cache, v_cache, block_tables, seq_lens,
                                  scale=None, mask_mod: Optional[MaskMod] = None, *, out=None,
                                  lse=None, workspace=None, dbg_err=None):
    """One decode step in one launch: sequence b's new token (k_new[b], v_new[b],
    [B, Hkv, d]) is written at position seq_lens[b]-1 of its block table, then
    the queries attend to the cache including it. Returns (out, lse)."""
    _check_pool(k_cache, v_cache)
    dev = k_cache.device
    B, Hq, d = q.shape
    _check(k_cache.dtype == torch.bfloat16, "bf16 pools only")
    for t, name in ((k_new, "k_new"), (v_new, "v_new")):
        _check(t.dtype == k_cache.dtype and t.device == dev and t.is_contiguous() and
               tuple(t.shape) == (B, k_cache.shape[1], d),
               f"{name} must be contiguous [B, num_kv_heads, head_dim] in the cache dtype")
    _i32(block_tables, "block_tables", dev)
    _i32(seq_lens, "seq_lens", dev)
    _check(q.dtype == k_cache.dtype and q.device == dev and q.is_contiguous(),
           "q must be contiguous, on the cache's device, in the cache dtype")
    _check(d == k_cache.shape[3], "head_dim mismatch")
    _check(block_tables.dim() == 2 and block_tables.shape[0] == B and seq_lens.numel() == B,
           "block_tables [B, M] and seq_lens [B] must match q's batch")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    mask_mod = mask_mod or no_mask()
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = decode_workspace(B, Hq, k_cache)
    L.check(L.lib().paged_attention_decode_append(
        _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), cache_desc(k_cache),
        _ptr(block_tables), block_tables.shape[1], _ptr(seq_lens), B, Hq, float(scale),
        mask_mod.to_c(B, dev, Hq), _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
        _ptr(dbg_err), _stream()))
    return out, lse


def shared_prefix_workspace_size(batch, num_q_heads, k_cache):
    return int(L.lib().paged_attention_decode_shared_prefix_workspace_size(
        batch, num_q_heads, cache_desc(k_cache)))


def shared_prefix_workspace(batch, num_q_heads, k_cache):
    n = shared_prefix_workspace_size(batch, num_q_heads, k_cache)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=k_cache.device)


def paged_attention_decode_shared_prefix(q, k_cache, v_cache, block_tables, seq_lens,
                                         group_start, shared_len, max_group_size, scale=None,
                                         mask_mod: Optional[MaskMod] = None, *, out=None,
                                         lse=None, workspace=None, dbg_err=None):
    """Decode for groups of sequences (beams, samples) that share a prefix.

    ``group_start`` (int32 [G+1] on the device) splits the batch into
    consecutive groups; ``shared_len`` (int32 [B]) is the length of each
    sequence's shared prefix, the same within a group. ``max_group_size`` is a
    host int bounding every group's size. Returns (out, lse) equal to
    ``paged_attention_decode`` on the same inputs."""
    _check_pool(k_cache, v_cache)
    dev = k_cache.device
    _i32(block_tables, "block_tables", dev)
    _i32(seq_lens, "seq_lens", dev)
    _i32(group_start, "group_start", dev)
    _i32(shared_len, "shared_len", dev)
    B, Hq, d = q.shape
    _check(q.dtype == k_cache.dtype and q.device == dev and q.is_contiguous(),
           "q must be contiguous, on the cache's device, in the cache dtype")
    _check(d == k_cache.shape[3], "head_dim mismatch")
    _check(block_tables.dim() == 2 and block_tables.shape[0] == B and seq_lens.numel() == B
           and shared_len.numel() == B, "block_tables, seq_lens and shared_len must match q")
    _check(group_start.dim() == 1 and group_start.numel() >= 2, "group_start must be [G + 1]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    mask_mod = mask_mod or no_mask()
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = shared_prefix_workspace(B, Hq, k_cache)
    L.check(L.lib().paged_attention_decode_shared_prefix(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), cache_desc(k_cache), _ptr(block_tables),
        block_tables.shape[1], _ptr(seq_lens), B, Hq, float(scale), mask_mod.to_c(B, dev, Hq),
        _ptr(group_start), group_start.numel() - 1, int(max_group_size), _ptr(shared_len),
        _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), _ptr(dbg_err), _stream()))
    return out, lse


def paged_attention_prefill(q, k_new, v_new, k_cache, v_cache, block_tables, ctx_lens, q_lens,
                            mask_mod: Optional[MaskMod] = None, scale=None, *, out=None,
                            lse=None, dbg_err=None):
    """A chunk of new queries per sequence over its paged context plus the
    chunk itself. q/k_new/v_new are packed by sequence. Returns (out, lse)."""
    _check_pool(k_cache, v_cache)
    dev = k_cache.device
    _i32(block_tables, "block_tables", dev)
    _i32(ctx_lens, "ctx_lens", dev)
    _i32(q_lens, "q_lens", dev)
    T, Hq, d = q.shape
    B = ctx_lens.numel()
    _check(q_lens.numel() == B and block_tables.dim() == 2 and block_tables.shape[0] == B,
           "ctx_lens, q_lens and block_tables must agree on the batch")
    for t, name in ((q, "q"), (k_new, "k_new"), (v_new, "v_new")):
        _check(t.dtype == k_cache.dtype and t.device == dev and t.is_contiguous(),
               f"{name} must be contiguous, on the cache's device, in the cache dtype")
    _check(k_new.shape == (T, k_cache.shape[1], d) and v_new.shape == k_new.shape,
           "k_new/v_new must be [total_q, num_kv_heads, head_dim]")
    mask_mod = mask_mod or no_mask()
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(T, Hq, dtype=torch.float32, device=dev)
    L.check(L.lib().paged_attention_prefill(
        _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), cache_desc(k_cache),
        _ptr(block_tables), block_tables.shape[1], _ptr(ctx_lens), _ptr(q_lens), B, T, Hq,
        float(scale) if scale is not None else 0.0, mask_mod.to_c(B, dev, Hq), _ptr(out), _ptr(lse),
        _ptr(dbg_err), _stream()))
    return out, lse


@dataclass
class DevicePool:
    """Device-side allocation state of one KV pool: a free stack (top at
    ``free_stack[free_top - 1]``), per-block reference counts and the scratch
    the reserve call keeps at zero. ``from_manager`` copies a host
    ``BlockManager``'s state (its free list pops from the end, as here)."""

    free_stack: torch.Tensor   # int32 [num_blocks]
    free_top: torch.Tensor     # int32 [1]
    refcount: torch.Tensor     # int32 [num_blocks]
    scratch: torch.Tensor      # int32 [2 * num_blocks], zero

    @staticmethod
    def from_manager(mgr, device):
        nb = mgr.num_blocks
        stack = torch.zeros(nb, dtype=torch.int32)
        free = list(mgr._free)
        if free:
            stack[:len(free)] = torch.tensor(free, dtype=torch.int32)
        return DevicePool(stack.to(device), torch.tensor([len(free)], dtype=torch.int32,
                                                         device=device),
                          torch.from_numpy(mgr.refcount.astype(np.int32)).to(device),
                          torch.zeros(2 * nb, dtype=torch.int32, device=device))


def paged_kv_reserve_slots(k_cache, v_cache, block_tables, seq_lens, num_new, pool: DevicePool,
                           num_tokens, dbg_err=None, k_scale=None, v_scale=None):
    """Reserve slots for ``num_new[b]`` new tokens of every sequence on the
    device (new blocks from the pool, copy-on-write of shared partly filled
    blocks). Updates block_tables, seq_lens and the pool in place. Returns
    (slot_mapping int64 [num_tokens], cow_pairs int32 [B, 2]). E4M3 pools pass
    their row scales, which are copied with the codes."""
    _check_pool(k_cache, v_cache)
    fp8 = k_cache.dtype in (torch.uint8, torch.float8_e4m3fn)
    if fp8 or k_scale is not None or v_scale is not None:
        _check(fp8, "row scales belong to E4M3 pools")
        _check_scales(k_scale, v_scale, k_cache)
    dev = k_cache.device
    for t, name in ((block_tables, "block_tables"), (seq_lens, "seq_lens"), (num_new, "num_new"),
                    (pool.free_stack, "free_stack"), (pool.free_top, "free_top"),
                    (pool.refcount, "refcount"), (pool.scratch, "scratch")):
        _i32(t, name, dev)
    B = seq_lens.numel()
    _check(block_tables.dim() == 2 and block_tables.shape[0] == B and num_new.numel() == B,
           "block_tables [B, M], seq_lens [B] and num_new [B] must agree")
    nb = k_cache.shape[0]
    _check(pool.free_stack.numel() >= nb and pool.refcount.numel() >= nb and
           pool.scratch.numel() >= 2 * nb, "pool arrays are smaller than the pool")
    slots = torch.empty(max(int(num_tokens), 1), dtype=torch.int64, device=dev)
    pairs = torch.empty(B, 2, dtype=torch.int32, device=dev)
    tail = (cache_desc(k_cache), _ptr(block_tables), block_tables.shape[1], _ptr(seq_lens),
            _ptr(num_new), B, _ptr(pool.free_stack), _ptr(pool.free_top), _ptr(pool.refcount),
            _ptr(pool.scratch), _ptr(slots), int(num_tokens), _ptr(pairs), _ptr(dbg_err),
            _stream())
    if fp8:
        L.check(L.lib().paged_kv_reserve_slots_fp8(_ptr(k_cache), _ptr(v_cache), _ptr(k_scale),
                                                   _ptr(v_scale), *tail))
    else:
        L.check(L.lib().paged_kv_reserve_slots(_ptr(k_cache), _ptr(v_cache), *tail))
    return slots[:int(num_tokens)], pairs


def block_mask(ctx_lens, q_lens, num_q_heads, mask_mod: MaskMod, q_tile=128, k_tile=128):
    """Block-sparse table of a mask: uint8 [B, Hq, n_q_tiles, n_k_tiles] with
    0 = skipped, 1 = partial, 2 = every pair visible (see the C header)."""
    dev = ctx_lens.device
    _i32(ctx_lens, "ctx_lens", dev)
    _i32(q_lens, "q_lens", dev)
    B = ctx_lens.numel()
    _check(q_lens.numel() == B, "ctx_lens and q_lens must agree on the batch")
    n_q = int(q_lens.max().item()) if B else 0
    n_k = int((ctx_lens + q_lens).max().item()) if B else 0
    nqt, nkt = -(-n_q // q_tile), -(-n_k // k_tile)
    out = torch.empty(B, num_q_heads, nqt, nkt, dtype=torch.uint8, device=dev)
    L.check(L.lib().paged_attention_block_mask(
        _ptr(ctx_lens), _ptr(q_lens), B, num_q_heads, mask_mod.to_c(B, dev, num_q_heads),
        int(q_tile), int(k_tile), nqt, nkt, _ptr(out), _stream()))
    return out


def read_dbg(dbg_err):
    """Raise PagedKVError if a kernel flagged an index error in ``dbg_err``."""
    v = int(dbg_err.item())
    if v:
        names = [n for n, bit in (("block id", L.PKV_DBG_BLOCK_ID), ("slot", L.PKV_DBG_SLOT),
                                  ("length", L.PKV_DBG_LENGTH), ("timeout", L.PKV_DBG_TIMEOUT),
                                  ("q_lens sum", L.PKV_DBG_QLEN_SUM)) if v & bit]
        raise L.PagedKVError(L.PKV_ERR_BAD_INDEX, "device flagged: " + ", ".join(names))
