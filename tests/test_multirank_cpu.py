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


@pytest.mark.parametrize("entry", ["fused_ce", "ce_separate"])
def test_reference_arm_json_line(entry):
    # bench.py --impl reference: the oracle on the host cores, one JSON line with the keys the
    # reference arm reports (no GPU needed)
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    wl = "tiny"
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", wl,
                        "--entry", entry, "--steps", "1", "--warmup", "1",
                        "--ref-seconds", "4"],
                       capture_output=True, text=True, timeout=600, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["value"] > 0 and line["dtype"] == "f64"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["config"]["entry"] == entry
