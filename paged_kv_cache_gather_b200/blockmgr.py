"""Host-side block manager: free list, per-sequence block tables, refcounts.

Follows "Ultimate Guide to PagedAttention": the KV cache is cut into
fixed-size blocks (16 tokens is the usual size); a per-request block table
maps logical positions to physical blocks; a request that grows takes a new
block and appends it to its table without moving data; requests with a common
prefix point at the same physical blocks, which are stored once and copied
only when written (copy-on-write); freed blocks are handed out again at once.

The manager never touches device memory. It produces the int32 block tables
and int64 slot mappings that the CUDA calls consume, and, for copy-on-write,
the list of (src, dst) block copies a caller must perform before appending.
"""

from typing import Dict, List, Optional, Tuple

import numpy as np
import torch


class OutOfBlocks(RuntimeError):
    pass


class BlockManager:
    """Pool of ``num_blocks`` physical blocks of ``block_size`` tokens.

    The free list starts as a seeded permutation of the pool (``seed=None``
    keeps it in order); allocation pops from its front and freeing pushes to
    the front, so a freed block is reused first.
    """

    def __init__(self, num_blocks: int, block_size: int = 16, seed: Optional[int] = None):
        if block_size <= 0 or block_size & (block_size - 1):
            raise ValueError("block_size must be a power of two")
        self.num_blocks = num_blocks
        self.block_size = block_size
        order = (np.random.default_rng(seed).permutation(num_blocks) if seed is not None
                 else np.arange(num_blocks))
        self._free: List[int] = [int(x) for x in order][::-1]  # stack: pop() = front
        self.refcount = np.zeros(num_blocks, dtype=np.int64)
        self.tables: Dict[int, List[int]] = {}
        self.lengths: Dict[int, int] = {}

    # ------------------------------------------------------------------ basics
    @property
    def num_free(self) -> int:
        return len(self._free)

    def _pop(self) -> int:
        if not self._free:
            raise OutOfBlocks("no free KV blocks")
        blk = self._free.pop()
        self.refcount[blk] = 1
        return blk

    def _release(self, blk: int) -> None:
        self.refcount[blk] -= 1
        if self.refcount[blk] < 0:
            raise RuntimeError(f"block {blk} released twice")
        if self.refcount[blk] == 0:
            self._free.append(blk)

    def add_sequence(self, seq_id: int, num_tokens: int = 0) -> List[int]:
        """Create a sequence holding ``num_tokens`` tokens (blocks allocated now)."""
        if seq_id in self.tables:
            raise KeyError(f"sequence {seq_id} exists")
        n = -(-num_tokens // self.block_size)
        if n > len(self._free):
            raise OutOfBlocks("not enough free KV blocks")
        self.tables[seq_id] = [self._pop() for _ in range(n)]
        self.lengths[seq_id] = num_tokens
        return list(self.tables[seq_id])

    def fork(self, parent: int, child: int) -> None:
        """New sequence sharing all of ``parent``'s blocks (refcount + 1 each)."""
        if child in self.tables:
            raise KeyError(f"sequence {child} exists")
        self.tables[child] = list(self.tables[parent])
        self.lengths[child] = self.lengths[parent]
        for blk in self.tables[child]:
            self.refcount[blk] += 1

    def free(self, seq_id: int) -> None:
        for blk in self.tables.pop(seq_id):
            self._release(blk)
        del self.lengths[seq_id]

    # ------------------------------------------------------------------ growth
    def append_slots(self, seq_id: int, n: int = 1) -> Tuple[List[int], List[Tuple[int, int]]]:
        """Reserve the next ``n`` positions of a sequence.

        Returns their slots (``block * block_size + row``) and the copy-on-write
        block copies ``(src, dst)`` that must happen before the K/V writes:
        a partly filled last block that is shared is replaced by a private copy.
        """
        table = self.tables[seq_id]
        L = self.lengths[seq_id]
        bs = self.block_size
        copies: List[Tuple[int, int]] = []
        slots: List[int] = []
        for p in range(L, L + n):
            j = p // bs
            if j == len(table):
                table.append(self._pop())
            elif self.refcount[table[j]] > 1:
                src = table[j]
                dst = self._pop()
                copies.append((src, dst))
                self._release(src)
                table[j] = dst
            slots.append(table[j] * bs + p % bs)
        self.lengths[seq_id] = L + n
        return slots, copies

    # ------------------------------------------------------------------ export
    def block_table_tensor(self, seq_ids, width: Optional[int] = None) -> torch.Tensor:
        rows = [self.tables[s] for s in seq_ids]
        width = width or max(1, max(len(r) for r in rows))
        t = np.full((len(rows), width), -1, dtype=np.int32)
        for i, r in enumerate(rows):
            if len(r) > width:
                raise ValueError("table width too small")
            t[i, :len(r)] = r
        return torch.from_numpy(t)

    def seq_lens_tensor(self, seq_ids) -> torch.Tensor:
        return torch.tensor([self.lengths[s] for s in seq_ids], dtype=torch.int32)

    def fragmentation(self) -> float:
        """Share of allocated token slots that hold no token (internal waste)."""
        used = sum(self.lengths.values())
        blocks = set(b for t in self.tables.values() for b in t)
        cap = len(blocks) * self.block_size
        # shared blocks count once; logical tokens in shared blocks count once per holder,
        # so bound the used count by the capacity
        return 0.0 if cap == 0 else max(0.0, 1.0 - min(used, cap) / cap)
