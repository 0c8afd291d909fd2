"""The benchmark's multi-rank plumbing on CPU with two gloo ranks: every rank must see the
slowest rank's time and the same whole-job throughput (weak scaling, no data-path
collective)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, q):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench

    local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
    ms = bench.max_over_ranks(local_ms, dist, "cpu")
    q.put((rank, ms, bench.job_throughput(ms, world)))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    import bench

    for rank, ms, value in got:
        assert ms == 15.0
        assert value == pytest.approx(2 * bench.L / 15e-3)


def test_single_rank_is_identity():
    import bench

    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(10.0, 1) == pytest.approx(bench.L / 1e-2)
