"""Multi-rank host logic of the benchmark, on CPU with the gloo backend (world size 2).

The path shards over batch items with no data-path collective (weak scaling): the only
cross-rank steps are the max over ranks of the elapsed time and the whole-job throughput.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [3.5, 7.25][rank]
        m = bench.max_over_ranks(mine, world)
        v = bench.job_throughput(1e9, m, world)
        # the reference arm runs on rank 0 only: other ranks leave at once with status 0
        os.environ["RANK"] = str(rank)
        rc = bench.reference_arm(type("A", (), {"steps": 1, "warmup": 0})(), world, rank) if rank else 0
        q.put((rank, m, v, rc))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, m, v, rc in got:
        assert m == 7.25                       # every rank sees the slowest rank's time
        assert v == pytest.approx(2 * 1e9 / 7.25e-3 / 1e9)
        assert rc == 0


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(4.0, 1) == 4.0
    assert bench.job_throughput(2e9, 2.0, 1) == pytest.approx(1000.0)
