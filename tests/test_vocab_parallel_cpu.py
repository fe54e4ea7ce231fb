"""The vocabulary-parallel path's host logic on CPU: the shard plan, the row slices of the dH
reduction, and VocabParallelCE's exchange steps with world size 2 and 3 over gloo, the compute
steps restated from the oracle (tests/vp_oracle_ops.py). Every rank's forward outputs, its dH
and the concatenated dW shards must equal the one-device oracle."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from lm_head_cross_tcgen05_b200.vocab_parallel import row_slices, shard_plan


@pytest.mark.parametrize("V,R", [(1000, 4), (128256, 8), (151936, 8), (600, 2), (1025, 4),
                                 (7, 7), (300, 2), (2048, 3)])
def test_shard_plan_covers_vocabulary(V, R):
    plan = shard_plan(V, R)
    assert len(plan) == R and plan[0][0] == 0 and plan[-1][1] == V
    for (a, b), (c, _) in zip(plan, plan[1:]):
        assert b == c                            # contiguous, ascending
    assert all(b > a for a, b in plan)           # non-empty
    sizes = [b - a for a, b in plan]
    if sizes[0] >= 256 and sizes[0] % 256 == 0:
        assert all(s % 256 == 0 for s in sizes[:-1])
    assert max(sizes[:-1] or [0]) == sizes[0]    # equal up to the last


def test_shard_plan_rejects_more_ranks_than_words():
    with pytest.raises(ValueError):
        shard_plan(3, 4)


@pytest.mark.parametrize("N,R", [(10, 3), (8192, 8), (1, 2), (0, 2), (7, 7)])
def test_row_slices(N, R):
    sl = row_slices(N, R)
    assert sl[0][0] == 0 and sl[-1][1] == N
    assert all(b - a in (N // R, N // R + 1) for a, b in sl)
    assert all(sl[j][1] == sl[j + 1][0] for j in range(R - 1))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q, case):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from lm_head_cross_tcgen05_b200.vocab_parallel import VocabParallelCE
        from oracle import lmh_oracle as O
        from tests.vp_oracle_ops import OracleOps
        from workloads import make_inputs, ragged
        N, d, V, ign, tau = case
        x = make_inputs(ragged(N, d, V, n_ignored=ign, seed=77 + N + V), device="cpu")
        H, W, y = x["H"], x["W"], x["labels"]
        vp = VocabParallelCE(V, ops=OracleOps(), temperature=tau)
        Ws = W[vp.v0:vp.v1]
        f = vp.forward(H, Ws, y)
        b = vp.backward(H, Ws, y, f["lse"])
        fb = vp.forward_backward(H, Ws, y)
        assert np.array_equal(fb["lse"].numpy(), f["lse"].numpy())
        assert np.allclose(fb["dH"].numpy(), b["dH"].numpy(), rtol=1e-12, atol=1e-15)
        assert np.allclose(fb["dW"].numpy(), b["dW"].numpy(), rtol=1e-12, atol=1e-15)
        ref = O.ce_fused(H, W, y, tau=tau)
        res = dict(rank=rank, v=(vp.v0, vp.v1),
                   lse=np.abs(f["lse"].numpy() - ref["lse"]).max(),
                   loss=np.abs(f["loss_rows"].numpy() - ref["loss_rows"]).max(),
                   logprob=np.abs(f["logprob"].numpy() - ref["logprob"]).max(),
                   mean=abs(float(f["loss_mean"][0]) - ref["loss_mean"]),
                   nvalid=int(f["n_valid"][0]) == ref["n_valid"],
                   argmax=bool((f["argmax"].numpy() == ref["argmax"]).all()),
                   dH=np.abs(b["dH"].numpy() - ref["dH"]).max() / max(np.abs(ref["dH"]).max(), 1e-300),
                   dW=np.abs(b["dW"].numpy() - ref["dW"][vp.v0:vp.v1]).max()
                   / max(np.abs(ref["dW"]).max(), 1e-300),
                   dH_digest=float(b["dH"].sum()))
        q.put(res)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,case", [
    (2, (37, 64, 700, 5, None)),       # ragged rows over 2 ranks, a shard of 350 words
    (3, (20, 64, 1030, 3, 0.7)),       # 3 ranks, shards 344/344/342, scalar temperature
    (2, (40, 64, 512, 0, None)),       # rows divide evenly: no padding in the dH gather
    (3, (2, 64, 900, 0, None)),        # fewer rows than ranks: one rank reduces no row
])
def test_vocab_parallel_exchange_gloo(world, case):
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
    assert [r["v"] for r in res] == shard_plan(case[2], world)
    for r in res:
        assert r["lse"] < 1e-9 and r["loss"] < 1e-9 and r["logprob"] < 1e-9 and r["mean"] < 1e-9
        assert r["nvalid"] and r["argmax"]
        assert r["dH"] < 1e-9 and r["dW"] < 1e-9
    assert len({r["dH_digest"] for r in res}) == 1   # every rank holds the same dH


def _support_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from lm_head_cross_tcgen05_b200.vocab_parallel import VocabParallelSupport
        from oracle import lmh_oracle as O
        from tests.vp_oracle_ops import OracleOps
        from workloads import make_inputs, ragged
        N, d, V, K = 24, 64, 900, 6
        x = make_inputs(ragged(N, d, V, seed=91, K=K), device="cpu")
        H, W, ids, ref = x["H"], x["W"], x["ids"].clone(), x["ref_logp"]
        ids[0, -1] = -1                       # padding
        ids[1, 1] = ids[1, 0]                 # a repeated id
        vp = VocabParallelSupport(V, ops=OracleOps())
        Ws = W[vp.v0:vp.v1]
        f = vp.forward(H, Ws, ids, ref)
        b = vp.backward(H, Ws, ids, f["lse"], mode=O.BWD_SUPPORT_KL, ref_logp=ref)
        g = np.linspace(-1, 1, N * K).reshape(N, K)
        b2 = vp.backward(H, Ws, ids, f["lse"], mode=O.BWD_SUPPORT_LOGPROB,
                         grad=torch.from_numpy(g))
        rk = O.support_kl(H, W, ids, ref)
        rb = O.backward(O.BWD_SUPPORT_KL, H, W, ids, np.full(N, 1.0 / N), ref)
        rb2 = O.backward(O.BWD_SUPPORT_LOGPROB, H, W, ids, g)
        err = lambda a, r: np.abs(a.numpy() - r).max() / max(np.abs(r).max(), 1e-300)
        q.put(dict(rank=rank, lp=err(f["lp"], rk["lp"]), lse=err(f["lse"], rk["lse"]),
                   kl=err(f["kl_rows"], rk["kl_rows"]),
                   dH=err(b["dH"], rb["dH"]), dW=err(b["dW"], rb["dW"][vp.v0:vp.v1]),
                   dH2=err(b2["dH"], rb2["dH"]), dW2=err(b2["dW"], rb2["dW"][vp.v0:vp.v1])))
    finally:
        dist.destroy_process_group()


def test_vocab_parallel_support_exchange_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_support_worker, args=(r, 3, port, q)) for r in range(3)]
    for p in ps:
        p.start()
    res = [q.get(timeout=180) for _ in ps]
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in res:
        for k in ("lp", "lse", "kl", "dH", "dW", "dH2", "dW2"):
            assert r[k] < 1e-9, (r["rank"], k, r[k])
