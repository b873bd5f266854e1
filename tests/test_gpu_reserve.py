"""GPU: device-side block allocation (paged_kv_reserve_slots) against the host
BlockManager, which serves the same requests one by one in batch order.

Tables, lengths, refcounts, the free stack, the slots and the copy-on-write
pairs must be identical (integers, bit for bit), the pools after the copies
must equal the oracle's copy of the blocks, and a full step (reserve, append,
decode) must match the oracle. Covers growth inside a block and across block
edges, forks whose holders append all or only in part, sequences that do not
append, several steps in a row (the scratch stays zero), a step replayed from
a CUDA graph, and the failure cases (pool exhausted, inconsistent count),
which must change nothing.
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_gather_b200 as pkv
from paged_kv_cache_gather_b200 import BlockManager
from paged_kv_cache_gather_b200 import inputs as I
from parity import assert_attention_close

pytestmark = pytest.mark.gpu

BS, HKV, D = 16, 2, 128


def scenario(seed, num_blocks=200):
    """A manager with plain sequences and forked families (shared partly filled
    last blocks); returns (manager, seq ids in batch order)."""
    rng = np.random.default_rng(seed)
    mgr = BlockManager(num_blocks, BS, seed=seed)
    ids = []
    nxt = 0
    for L in (0, 1, 15, 16, 17, 40, 100):
        mgr.add_sequence(nxt, L)
        ids.append(nxt)
        nxt += 1
    for L, kids in ((37, 3), (48, 2), (5, 4)):
        root = nxt
        mgr.add_sequence(root, L)
        ids.append(root)
        nxt += 1
        for _ in range(kids):
            mgr.fork(root, nxt)
            ids.append(nxt)
            nxt += 1
    order = rng.permutation(len(ids))
    return mgr, [ids[i] for i in order]


def device_state(mgr, ids, width, dev):
    tables = mgr.block_table_tensor(ids, width).to(dev)
    lens = mgr.seq_lens_tensor(ids).to(dev)
    return tables, lens, pkv.DevicePool.from_manager(mgr, dev)


def host_step(mgr, ids, num_new):
    slots, pairs = [], []
    for s, n in zip(ids, num_new):
        sl, cp = mgr.append_slots(s, int(n))
        slots += sl
        assert len(cp) <= 1
        pairs.append(cp[0] if cp else (-1, -1))
    return np.array(slots, dtype=np.int64), np.array(pairs, dtype=np.int32)


def compare(mgr, ids, width, tables, lens, pool):
    assert torch.equal(tables.cpu(), mgr.block_table_tensor(ids, width))
    assert torch.equal(lens.cpu(), mgr.seq_lens_tensor(ids))
    assert torch.equal(pool.refcount.cpu(), torch.from_numpy(mgr.refcount.astype(np.int32)))
    top = int(pool.free_top.item())
    assert top == mgr.num_free
    assert pool.free_stack[:top].cpu().tolist() == list(mgr._free)
    assert int(pool.scratch.abs().sum().item()) == 0


def pools(seed, num_blocks, dev):
    gen = torch.Generator().manual_seed(seed)
    kc = I.randn((num_blocks, HKV, BS, D), gen)
    vc = I.randn((num_blocks, HKV, BS, D), gen)
    return kc, vc, kc.to(dev), vc.to(dev)


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_reserve_matches_block_manager(cuda_device, seed):
    mgr, ids = scenario(seed)
    width = 24
    tables, lens, pool = device_state(mgr, ids, width, cuda_device)
    rng = np.random.default_rng(seed + 10)
    num_new = rng.integers(0, 40, size=len(ids)).astype(np.int32)
    num_new[rng.integers(0, len(ids))] = 0
    kc_h, vc_h, kc, vc = pools(seed, mgr.num_blocks, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    slots, pairs = pkv.paged_kv_reserve_slots(kc, vc, tables, lens,
                                              torch.from_numpy(num_new).to(cuda_device), pool,
                                              int(num_new.sum()), dbg_err=err)
    torch.cuda.synchronize()
    pkv.read_dbg(err)
    exp_slots, exp_pairs = host_step(mgr, ids, num_new)
    assert np.array_equal(slots.cpu().numpy(), exp_slots)
    assert np.array_equal(pairs.cpu().numpy(), exp_pairs)
    compare(mgr, ids, width, tables, lens, pool)
    used = exp_pairs[exp_pairs[:, 0] >= 0]
    ek, ev = oracle.kv_copy_blocks(kc_h, vc_h, used)
    assert torch.equal(kc.cpu().view(torch.int16), ek.view(torch.int16))
    assert torch.equal(vc.cpu().view(torch.int16), ev.view(torch.int16))


def test_all_holders_append_last_keeps_block(cuda_device):
    mgr = BlockManager(40, BS, seed=7)
    mgr.add_sequence(0, 21)
    for c in (1, 2, 3):
        mgr.fork(0, c)
    ids = [2, 0, 3, 1]
    tables, lens, pool = device_state(mgr, ids, 4, cuda_device)
    _, _, kc, vc = pools(7, 40, cuda_device)
    num_new = torch.ones(4, dtype=torch.int32, device=cuda_device)
    slots, pairs = pkv.paged_kv_reserve_slots(kc, vc, tables, lens, num_new, pool, 4)
    exp_slots, exp_pairs = host_step(mgr, ids, [1, 1, 1, 1])
    assert np.array_equal(pairs.cpu().numpy(), exp_pairs)
    assert (exp_pairs[:3, 0] >= 0).all() and exp_pairs[3, 0] == -1  # last in batch order keeps
    assert np.array_equal(slots.cpu().numpy(), exp_slots)
    compare(mgr, ids, 4, tables, lens, pool)


def test_steps_in_a_row_and_end_to_end_decode(cuda_device):
    mgr, ids = scenario(4, num_blocks=300)
    width = 40
    tables, lens, pool = device_state(mgr, ids, width, cuda_device)
    kc_h, vc_h, kc, vc = pools(4, mgr.num_blocks, cuda_device)
    gen = torch.Generator().manual_seed(44)
    rng = np.random.default_rng(4)
    for step in range(5):
        num_new = rng.integers(0, 20, size=len(ids)).astype(np.int32)
        T = int(num_new.sum())
        slots, pairs = pkv.paged_kv_reserve_slots(kc, vc, tables, lens,
                                                  torch.from_numpy(num_new).to(cuda_device),
                                                  pool, T)
        exp_slots, exp_pairs = host_step(mgr, ids, num_new)
        assert np.array_equal(slots.cpu().numpy(), exp_slots), step
        kn = I.randn((T, HKV, D), gen)
        vn = I.randn((T, HKV, D), gen)
        pkv.paged_kv_append(kn.to(cuda_device), vn.to(cuda_device), slots, kc, vc)
        used = exp_pairs[exp_pairs[:, 0] >= 0]
        kc_h, vc_h = oracle.kv_copy_blocks(kc_h, vc_h, used)
        kc_h, vc_h = oracle.kv_append(kn, vn, torch.from_numpy(exp_slots), kc_h, vc_h)
    torch.cuda.synchronize()
    compare(mgr, ids, width, tables, lens, pool)
    assert torch.equal(kc.cpu().view(torch.int16), kc_h.view(torch.int16))
    assert torch.equal(vc.cpu().view(torch.int16), vc_h.view(torch.int16))
    q = I.randn((len(ids), 8, D), gen)
    live = lens > 0
    out, lse = pkv.paged_attention_decode(q.to(cuda_device), kc, vc, tables, lens, None,
                                          pkv.causal())
    ref_o, ref_l = oracle.paged_decode(q, kc_h, vc_h, tables.cpu(), lens.cpu(), 1 / D ** 0.5,
                                       oracle.MASK_CAUSAL)
    assert_attention_close(out.cpu(), lse.cpu(), ref_o, ref_l, torch.bfloat16, "reserve e2e")
    assert live.any()


def test_graph_replayed_decode_steps(cuda_device):
    # one growth step (reserve + append + decode) captured once, replayed 20
    # times: the device state advances as the host manager does step by step
    mgr, ids = scenario(5, num_blocks=300)
    width = 16
    tables, lens, pool = device_state(mgr, ids, width, cuda_device)
    _, _, kc, vc = pools(5, mgr.num_blocks, cuda_device)
    B = len(ids)
    num_new = torch.ones(B, dtype=torch.int32, device=cuda_device)
    kn = torch.zeros(B, HKV, D, dtype=torch.bfloat16, device=cuda_device)
    vn = torch.zeros_like(kn)
    q = torch.zeros(B, 8, D, dtype=torch.bfloat16, device=cuda_device)
    out = torch.empty_like(q)
    lse = torch.empty(B, 8, dtype=torch.float32, device=cuda_device)
    ws = pkv.decode_workspace(B, 8, kc)
    state = {}

    def step():
        slots, _ = pkv.paged_kv_reserve_slots(kc, vc, tables, lens, num_new, pool, B)
        pkv.paged_kv_append(kn, vn, slots, kc, vc)
        pkv.paged_attention_decode(q, kc, vc, tables, lens, None, pkv.causal(), out=out,
                                   lse=lse, workspace=ws)
        state["slots"] = slots

    step()  # eager first call (sets kernel attributes before capture)
    host_step(mgr, ids, [1] * B)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            step()
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(20):
        g.replay()
        host_step(mgr, ids, [1] * B)
    torch.cuda.synchronize()
    compare(mgr, ids, width, tables, lens, pool)


def test_pool_exhausted_changes_nothing(cuda_device):
    mgr, ids = scenario(6, num_blocks=60)
    width = 24
    tables, lens, pool = device_state(mgr, ids, width, cuda_device)
    _, _, kc, vc = pools(6, mgr.num_blocks, cuda_device)
    before = (tables.clone(), lens.clone(), pool.refcount.clone(), pool.free_stack.clone(),
              pool.free_top.clone())
    num_new = torch.full((len(ids),), 200, dtype=torch.int32, device=cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    slots, pairs = pkv.paged_kv_reserve_slots(kc, vc, tables, lens, num_new, pool,
                                              200 * len(ids), dbg_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pkv._lib.PKV_DBG_OUT_OF_BLOCKS
    assert bool((slots == -1).all()) and bool((pairs == -1).all())
    after = (tables, lens, pool.refcount, pool.free_stack, pool.free_top)
    assert all(torch.equal(a, b) for a, b in zip(before, after))
    assert int(pool.scratch.abs().sum().item()) == 0


def test_token_count_mismatch_is_flagged(cuda_device):
    mgr, ids = scenario(8)
    tables, lens, pool = device_state(mgr, ids, 24, cuda_device)
    _, _, kc, vc = pools(8, mgr.num_blocks, cuda_device)
    lens0 = lens.clone()
    num_new = torch.ones(len(ids), dtype=torch.int32, device=cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    slots, _ = pkv.paged_kv_reserve_slots(kc, vc, tables, lens, num_new, pool, len(ids) - 1,
                                          dbg_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pkv._lib.PKV_DBG_LENGTH
    assert bool((slots == -1).all()) and torch.equal(lens, lens0)
