"""The N > 1 path of bench.py on the CPU: two ranks over gloo.  The data path
has no collective (independent replicas); what the ranks share is the timing
aggregation, which must give every rank the max over ranks, and the whole-job
value, which counts every rank's bytes against that max."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 20.0 - rank, 3.0 * (rank + 1)]     # elapsed, e2e, decode ms of this rank
        got = bench.max_over_ranks(dist, mine)
        dist.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = [11.0, 20.0, 6.0]
    assert res[0] == want and res[1] == want


def test_max_over_ranks_single_process_is_identity():
    assert bench.max_over_ranks(None, [1.5, 2.5]) == [1.5, 2.5]


def test_weak_scaling_value_counts_every_rank():
    one = bench.weak_scaling_gbs(1, 4.83e9, 1.4)
    assert one == pytest.approx(4.83e9 / 1.4e-3 / 1e9)
    assert bench.weak_scaling_gbs(8, 4.83e9, 1.4) == pytest.approx(8 * one)
