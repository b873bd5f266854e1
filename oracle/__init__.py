"""Float64 CPU oracle for paged KV-cache attention (test infrastructure only).

This package is the independent checker of the CUDA library. Only the test
suite, the smoke check in ``__graft_entry__`` and the CPU-baseline leg of
``bench.py`` may import it; the product path never does. It shares no code
with the CUDA path (no kernels, headers, helpers or tables).

Sources followed (titles of the pages the method is described on):

* "Paged Attention Meets FlexAttention: Unlocking Long-Context Efficiency in
  Deployed Inference" (abstract): a fused attention kernel that gathers
  scattered, non-contiguous KV blocks and applies FlexAttention masks.
* "Ultimate Guide to PagedAttention", sections on KV blocks and the block
  table: fixed-size blocks (16 tokens typical), a per-request block table that
  maps logical positions to physical blocks, growth by appending blocks, and
  prefix sharing with copy-on-write.
* "FlashAttention: Fast and Memory-Efficient Exact Attention with
  IO-Awareness" (abstract): attention is computed exactly; tiling only changes
  the order of memory traffic, never the result.

Because the method is exact, the oracle is the plain definition: resolve each
block table into a contiguous K/V, then masked softmax attention in float64.

Pins (see ``tests/test_oracle_pins.py``): dense attention from a different
library routine on a contiguous layout, invariance under permutation of the
physical blocks, closed forms (identical keys, a dominant key, W >= L), a
pure-Python brute force on tiny inputs, split-and-merge of the softmax, and
shared-vs-copied prefixes; ``tests/test_golden.py`` checks decode, prefill,
append and gather against a worked example with hand-derived exact answers
(``tests/golden/``). The E4M3 pools of ``oracle.fp8`` are pinned by
``tests/test_oracle_fp8.py`` (rounding and decoding against torch's
float8_e4m3fn, a separate implementation of the format) and
``tests/test_oracle_fp8_placement.py`` (a hand-derived worked example in
``tests/golden/``, a scalar brute force of the placement and the read-back,
and planted mistakes that those checks reject). No function here is
parity-unpinned.
"""

from .attention64 import (  # noqa: F401
    MASK_NONE,
    MASK_CAUSAL,
    MASK_SLIDING,
    MASK_PREFIX_LM,
    MASK_DOCUMENT,
    document_of,
    visible,
    resolve_block_table,
    masked_attention,
    paged_decode,
    paged_prefill,
    paged_prefill_rows,
    paged_prefill_tile,
    paged_decode_rows,
    kv_append,
    kv_gather,
    kv_copy_blocks,
)
