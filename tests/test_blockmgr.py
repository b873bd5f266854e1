"""Host block manager: allocation order, growth, sharing, copy-on-write, reuse (CPU)."""

import numpy as np
import pytest

from paged_kv_cache_gather_b200 import inputs as I
from paged_kv_cache_gather_b200.blockmgr import BlockManager, OutOfBlocks


def test_first_fit_matches_workload_tables():
    """The manager, seeded like the ragged-batch workload, hands out the same tables."""
    case = I.make_decode_case("t", lens=[5, 40, 1, 33], num_q_heads=2, num_kv_heads=1,
                              head_dim=8, block_size=16, num_blocks=64, dtype=I.torch.float32,
                              seed=77)
    bm = BlockManager(64, 16, seed=77)
    for s, L in enumerate([5, 40, 1, 33]):
        bm.add_sequence(s, L)
    t = bm.block_table_tensor(range(4), width=case.block_tables.shape[1])
    assert np.array_equal(t.numpy(), case.block_tables.numpy())


def test_growth_allocates_only_at_block_boundaries_and_moves_nothing():
    bm = BlockManager(8, 4, seed=None)
    bm.add_sequence(0, 3)
    before = list(bm.tables[0])
    slots, copies = bm.append_slots(0, 1)           # position 3: same block
    assert slots == [before[0] * 4 + 3] and copies == [] and bm.tables[0] == before
    slots, _ = bm.append_slots(0, 2)                # positions 4, 5: one new block
    assert len(bm.tables[0]) == 2 and bm.tables[0][0] == before[0]
    assert slots == [bm.tables[0][1] * 4 + 0, bm.tables[0][1] * 4 + 1]
    assert bm.lengths[0] == 6


def test_fork_shares_blocks_and_copy_on_write():
    bm = BlockManager(16, 4, seed=3)
    bm.add_sequence(0, 6)                           # 2 blocks, the last half full
    bm.fork(0, 1)
    assert bm.tables[0] == bm.tables[1]
    assert all(bm.refcount[b] == 2 for b in bm.tables[0])
    last = bm.tables[1][1]
    slots, copies = bm.append_slots(1, 1)           # writes into the shared last block
    assert copies == [(last, bm.tables[1][1])] and bm.tables[1][1] != last
    assert bm.refcount[last] == 1 and bm.tables[0][1] == last
    assert slots == [bm.tables[1][1] * 4 + 2]
    # full shared blocks stay shared
    assert bm.tables[0][0] == bm.tables[1][0] and bm.refcount[bm.tables[0][0]] == 2


def test_freed_blocks_are_reused_first():
    bm = BlockManager(6, 4, seed=5)
    bm.add_sequence(0, 8)
    freed = list(bm.tables[0])
    bm.free(0)
    bm.add_sequence(1, 4)
    assert bm.tables[1][0] in freed
    assert bm.num_free == 5


def test_out_of_blocks_and_bad_block_size():
    bm = BlockManager(2, 4)
    with pytest.raises(OutOfBlocks):
        bm.add_sequence(0, 9)
    with pytest.raises(ValueError):
        BlockManager(4, 12)


def test_fragmentation_below_one_block_per_sequence():
    bm = BlockManager(40000, 16, seed=1)
    lens = np.random.default_rng(0).integers(1, 8193, size=64)
    for s, L in enumerate(lens):
        bm.add_sequence(s, int(L))
    waste = bm.fragmentation()
    assert 0 <= waste < 64 * 16 / lens.sum() + 1e-12
