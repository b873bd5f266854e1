"""Host checks of the shared-prefix workload generator: every member of a group
holds the same K/V over the shared prefix, its own blocks after it, and the
group description tiles the batch."""

import numpy as np
import torch

from paged_kv_cache_gather_b200 import inputs as I


def _kv_at(case, b, t):
    bs = case.block_size
    blk = int(case.block_tables[b, t // bs])
    return case.k_cache[blk, :, t % bs], case.v_cache[blk, :, t % bs]


def test_members_share_prefix_and_own_the_rest():
    case = I.make_shared_prefix_case("t", group_sizes=[3, 1, 4], prefix_lens=[40, 0, 35],
                                     suffix_lens=[5, 0, 17, 1, 9, 0, 30, 2], num_q_heads=8,
                                     num_kv_heads=2, seed=5, peaky=True)
    gs = case.extra["group_start"].tolist()
    sl = case.extra["shared_len"].tolist()
    assert gs == [0, 3, 4, 8] and case.extra["max_group_size"] == 4
    for gi in range(3):
        lead = gs[gi]
        P = sl[lead]
        for b in range(gs[gi], gs[gi + 1]):
            assert sl[b] == P and int(case.seq_lens[b]) >= P
            for t in range(P):
                k0, v0 = _kv_at(case, lead, t)
                k1, v1 = _kv_at(case, b, t)
                assert torch.equal(k0, k1) and torch.equal(v0, v1)
    # blocks after the full prefix blocks belong to one sequence only
    bs = case.block_size
    owner = {}
    for b in range(case.batch):
        P = sl[b]
        n = (int(case.seq_lens[b]) + bs - 1) // bs
        for j in range(P // bs, n):
            blk = int(case.block_tables[b, j])
            assert owner.setdefault(blk, b) == b
    # groups with a shared prefix use fewer unique blocks than copies would
    copies = sum((int(L) + bs - 1) // bs for L in case.seq_lens)
    assert case.extra["unique_blocks"] < copies


def test_beams_config_describes_groups():
    case = I.config4(groups=2, beams=3, prefix=64, suffix=16, num_blocks=64)
    assert case.extra["group_start"].tolist() == [0, 3, 6]
    assert case.extra["shared_len"].tolist() == [64] * 6
    tabs = case.block_tables.numpy()
    assert np.array_equal(tabs[0, :4], tabs[2, :4]) and not np.array_equal(tabs[0, :4], tabs[3, :4])
