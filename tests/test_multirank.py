"""The benchmark's multi-process plumbing on CPU: two gloo ranks set up from
torchrun-style environment variables, a barrier, and the max-over-ranks
reduction used for every timed number (no GPU, no collective on the data
path)."""

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2",
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench

    ws, r, local = bench.dist_setup(backend="gloo")
    assert (ws, r, local) == (2, rank, rank)
    bench.barrier(ws)
    t = bench.max_over_ranks(10.0 + 5.0 * rank, ws, torch.device("cpu"))
    out.put((rank, t))
    torch.distributed.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got == {0: 15.0, 1: 15.0}


def test_single_rank_needs_no_process_group():
    import bench

    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert bench.dist_setup(backend="gloo") == (1, 0, 0)
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
