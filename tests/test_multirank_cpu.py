"""The multi-rank path of bench.py (replicas, weak scaling) with world size 2 over gloo on CPU:
each rank draws its own batch, the job time is the slowest rank's, and the job throughput
counts the work of every rank."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from workloads import WORKLOADS, make_inputs
        wl = WORKLOADS["tiny"]
        x = make_inputs(wl, seed=bench.replica_seed(wl, rank))
        t = bench.reduce_max(10.0 + rank, world)          # per-rank "step times"
        digest = float(x["H"].float().sum())
        q.put((rank, t, digest, bench.job_tflops(6.0e12, world, t)))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, t0, h0, v0), (r1, t1, h1, v1) = res
    assert t0 == t1 == 11.0                 # the max over ranks, seen by every rank
    assert h0 != h1                         # each replica has its own seeded batch
    assert v0 == v1 == pytest.approx(6.0e12 * 2 / 11e-3 / 1e12)


def test_single_rank_helpers():
    import bench
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.job_tflops(1e12, 1, 1.0) == pytest.approx(1000.0)
