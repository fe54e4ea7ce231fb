"""The row data-parallel path's host logic on CPU: DataParallelCE's exchange steps (the global
valid count, the rank-ordered sum of the loss shares and of dW) with world size 2 and 3 over
gloo, the compute steps restated from the oracle (tests/dp_oracle_ops.py). Every rank's outputs
for its own rows, the global mean and count, and the summed dW must equal the one-device
oracle on the concatenated batch."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q, case):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import torch
        from lm_head_cross_tcgen05_b200.data_parallel import DataParallelCE
        from oracle import lmh_oracle as O
        from tests.dp_oracle_ops import DataParallelOracleOps
        from workloads import make_inputs, ragged
        split, d, V, ign, tau, weighted, mean = case
        N = sum(split)
        x = make_inputs(ragged(N, d, V, n_ignored=ign, seed=55 + N + V), device="cpu")
        H, W, y = x["H"], x["W"], x["labels"].clone()
        a = sum(split[:rank])
        b = a + split[rank]
        g = np.linspace(-1.0, 2.0, N) if weighted else None
        dp = DataParallelCE(ops=DataParallelOracleOps(), temperature=tau, mean=mean)
        out = dp.forward_backward(H[a:b], W, y[a:b],
                                  grad=None if g is None else torch.from_numpy(g[a:b]),
                                  mode=O.BWD_LOGPROB if weighted else O.BWD_CE)
        f = O.ce_forward(H, W, y, tau)
        n = f["n_valid"]
        # per-row weights are taken as given; the mean divides the unit weight
        w = g if weighted else (np.full(N, 1.0 / n if n else 0.0) if mean else np.ones(N))
        rb = O.backward(O.BWD_LOGPROB if weighted else O.BWD_CE, H, W, y, w, tau=tau)
        rel = lambda u, r: np.abs(u.numpy() - r).max() / max(np.abs(r).max(), 1e-300) if r.size else 0.0
        q.put(dict(rank=rank,
                   rows=max(np.abs(out["loss_rows"].numpy() - f["loss_rows"][a:b]).max(initial=0),
                            np.abs(out["lse"].numpy() - f["lse"][a:b]).max(initial=0),
                            np.abs(out["logprob"].numpy() - f["logprob"][a:b]).max(initial=0)),
                   argmax=bool((out["argmax"].numpy() == f["argmax"][a:b]).all()),
                   mean=abs(float(out["loss_mean"][0]) - f["loss_mean"]),
                   nvalid=int(out["n_valid"][0]) == n,
                   dH=rel(out["dH"], rb["dH"][a:b]), dW=rel(out["dW"], rb["dW"]),
                   dW_digest=float(out["dW"].sum())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,case", [
    (2, ((17, 20), 64, 700, 5, None, False, True)),      # ragged split, ignored rows
    (3, ((9, 0, 14), 64, 1030, 3, 0.7, False, True)),    # a rank with no rows, temperature
    (3, ((8, 8, 7), 64, 600, 0, None, False, False)),    # summed loss
    (2, ((12, 11), 64, 512, 4, None, True, True)),       # weighted log-prob objective
    (3, ((0, 5, 9), 64, 300, 14, None, False, True)),    # no valid row: mean and grads 0
])
def test_data_parallel_exchange_gloo(world, case):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, world, port, q, case)) for r in range(world)]
    for p in ps:
        p.start()
    res = sorted((q.get(timeout=180) for _ in ps), key=lambda r: r["rank"])
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in res:
        assert r["rows"] < 1e-9 and r["mean"] < 1e-9, r
        assert r["nvalid"] and r["argmax"], r
        assert r["dH"] < 1e-9 and r["dW"] < 1e-9, r
    assert len({r["dW_digest"] for r in res}) == 1   # every rank holds the same dW


def _absent_rank_worker(rank, world, port, q):
    import datetime
    import time
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=3))
    try:
        if rank == 1:            # leaves between steps: never joins the step's collectives
            time.sleep(10)
            q.put(dict(rank=rank))
            return
        from lm_head_cross_tcgen05_b200.data_parallel import DataParallelCE
        from tests.dp_oracle_ops import DataParallelOracleOps
        from workloads import make_inputs, ragged
        x = make_inputs(ragged(8, 64, 300, seed=5), device="cpu")
        dp = DataParallelCE(ops=DataParallelOracleOps())
        t0 = time.monotonic()
        try:
            dp.forward_backward(x["H"], x["W"], x["labels"])
            q.put(dict(rank=rank, error=None))
        except Exception as e:   # the group's timeout ends the first collective
            q.put(dict(rank=rank, error=type(e).__name__, after=time.monotonic() - t0))
    finally:
        dist.destroy_process_group()


def test_absent_rank_ends_the_step_with_an_error():
    # a rank that never joins: the others' first exchange (the global count) fails after the
    # process group's timeout instead of waiting for ever
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_absent_rank_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted((q.get(timeout=120) for _ in ps), key=lambda r: r["rank"])
    for p in ps:
        p.join(timeout=60)
    assert res[0]["error"] is not None, res
    assert res[0]["after"] < 9.0, res


def _p2p_chunk_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from lm_head_cross_tcgen05_b200.data_parallel import DataParallelCE
        from tests.dp_oracle_ops import DataParallelOracleOps
        try:
            DataParallelCE(ops=DataParallelOracleOps(), p2p=True, chunk_rows=128)
            refused = None
        except ValueError as e:
            refused = str(e)
        ok = DataParallelCE(ops=DataParallelOracleOps(), p2p=True)   # one chunk: accepted
        q.put(dict(rank=rank, refused=refused, p2p=ok.p2p))
    finally:
        dist.destroy_process_group()


def test_peer_memory_exchange_refuses_a_chunk_plan():
    # the peer-memory dW exchange runs each rank's rows as one chunk: a chunk_rows budget
    # cannot be honoured, so it is refused instead of ignored (two gloo ranks: p2p is only
    # active with more than one rank)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_p2p_chunk_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = [q.get(timeout=120) for _ in ps]
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in res:
        assert r["refused"] and "chunk_rows" in r["refused"], r
        assert r["p2p"] is True
