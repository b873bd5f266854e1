"""B200-native paged KV-cache attention.

Calls (thin bindings over the C ABI in ``include/pagedkv.h``):

* ``paged_kv_append``         slot-mapped write of new tokens' K/V
* ``paged_kv_gather``         block tables resolved to contiguous K/V
* ``paged_kv_append_fp8`` / ``paged_attention_decode_fp8``  E4M3 pools with
  per-row scales (half the bytes per token)
* ``paged_kv_copy_blocks``    copy-on-write of shared blocks (``_fp8``: E4M3
  pools, row scales copied with the codes)
* ``paged_kv_reserve_slots``  device-side block allocation (growth + copy-on-write;
  E4M3 pools pass their row scales)
* ``paged_attention_decode``  one query per sequence over paged KV
* ``paged_attention_prefill`` a chunk of queries over paged context + chunk
* ``paged_attention_decode_shared_prefix``  decode for groups (beams,
  samples) sharing a prefix, each shared block read once per group
* ``block_mask``              block-sparse table of a mask modifier

Host helpers: ``BlockManager`` (free list, tables, refcounts, copy-on-write)
and the seeded workload generators in ``inputs``.
"""

from .blockmgr import BlockManager, OutOfBlocks  # noqa: F401
from .ops import (  # noqa: F401
    DevicePool,
    MaskMod,
    block_mask,
    causal,
    decode_workspace,
    decode_workspace_size,
    document,
    no_mask,
    paged_attention_decode,
    paged_attention_decode_append,
    paged_attention_decode_fp8,
    paged_attention_decode_shared_prefix,
    paged_attention_prefill,
    paged_kv_append,
    paged_kv_append_fp8,
    paged_kv_copy_blocks,
    paged_kv_copy_blocks_fp8,
    paged_kv_gather,
    paged_kv_reserve_slots,
    prefix_lm,
    read_dbg,
    shared_prefix_workspace,
    shared_prefix_workspace_size,
    sliding_window,
)
from ._lib import PagedKVError  # noqa: F401
