"""The multi-GPU path is replicas only: host-side rank logic as world-size-2 gloo ranks on CPU."""
import multiprocessing as mp
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, ms, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        slowest = bench.max_over_ranks(ms[rank], world, device="cpu")
        value = bench.replica_throughput(4, 100, world, slowest)
        out.put((rank, slowest, value, bench.rank_master(0x5EED0002, rank)))
    finally:
        dist.destroy_process_group()


def test_two_replicas_agree_on_the_slowest_rank():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port, world, ms = _free_port(), 2, [10.0, 12.5]
    procs = [ctx.Process(target=_rank, args=(r, world, port, ms, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank sees the slowest rank's time; whole-job tokens/s counts every rank's tokens
    assert [r[1] for r in res] == [12.5, 12.5]
    assert res[0][2] == res[1][2] == pytest.approx(4 * 100 * 2 / 0.0125)
    # each replica draws its own weights and inputs
    assert res[0][3] != res[1][3]


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.replica_throughput(8192, 10, 1, 20.0) == pytest.approx(8192 * 10 / 0.02)
