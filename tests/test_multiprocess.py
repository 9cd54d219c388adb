"""Multi-process host logic of the bench (replicas only): ranks on CPU with the
gloo backend, world_size 2.  The attention itself has no exchange step; the
only cross-rank operations are the max of per-rank times and the whole-job rate."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        per_rank_ms = [12.5, 17.25][rank]
        slowest = bench.max_across_ranks(per_rank_ms, world, "cpu")
        rate = bench.whole_job_rate(1.0e12, world, slowest * 1e-3)
        q.put((rank, slowest, rate))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, slowest, rate in res:
        assert slowest == 17.25                       # every rank sees the slowest rank's time
        assert rate == pytest.approx(2 * 1.0e12 / 17.25e-3)   # both replicas' work / that time


def test_single_rank_is_identity():
    assert bench.max_across_ranks(3.5, 1, "cpu") == 3.5
    assert bench.whole_job_rate(10.0, 1, 2.0) == 5.0
