"""GPU parity of the vocabulary-parallel entries (through the C ABI) against the fp64 oracle.

One GPU stands in for R ranks: the R shards' steps run one after another and the exchange is a
concatenation in rank order. No kernel of one shard waits for another shard, so this runs the
same device code each rank would run, in the same order of additions. (The exchange logic of
VocabParallelCE itself is covered on CPU ranks over gloo, and on one rank here.)"""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch

import lm_head_cross_tcgen05_b200 as L
from lm_head_cross_tcgen05_b200.vocab_parallel import CudaOps, VocabParallelCE, shard_plan
from tests.gpu_common import O, check_ce_fused, check_grad, check_rows, device_inputs
from workloads import ragged

pytestmark = pytest.mark.gpu


def _wl(N, d, V, ign):
    return ragged(N, d, V, n_ignored=ign, seed=3000 + N + d + V)


def _emulate(x, V, R, chunk=0, tau=None, mode=L.BWD_CE, grad=None, mean=True):
    H, W, y = x["H"], x["W"], x["labels"]
    d = H.shape[1]
    ops = CudaOps()
    plan = shard_plan(V, R)
    recs = [ops.partials(H, W[a:b], y, a, V, chunk, tau) for a, b in plan]
    f = ops.combine(torch.stack(recs), y, V, d)
    parts, dWs = [], []
    for a, b in plan:
        p, w = ops.backward(mode, H, W[a:b], y, f["lse"], grad, a, V, chunk, mean, tau)
        parts.append(p)
        dWs.append(w)
    f["dH"] = ops.reduce_rows(torch.stack(parts))
    f["dW"] = torch.cat(dWs)
    torch.cuda.synchronize()
    return f


def _emulate_fused(x, V, R, tau=None, mean=True, n_given=None):
    H, W, y = x["H"], x["W"], x["labels"]
    ops = CudaOps()
    plan = shard_plan(V, R)
    recs, states = zip(*[ops.partials_fused(H, W[a:b], y, a, V, mean, tau) for a, b in plan])
    f = ops.combine(torch.stack(recs), y, V, H.shape[1], n_given)
    parts, dWs = zip(*[ops.fused_backward(st, H, W[a:b], y, f["lse"], a, V, n_given)
                       for st, (a, b) in zip(states, plan)])
    f["dH"] = ops.reduce_rows(torch.stack(parts))
    f["dW"] = torch.cat(dWs)
    torch.cuda.synchronize()
    return f


@pytest.mark.parametrize("N,d,V,ign,R", [
    (300, 192, 1000, 5, 2),
    (200, 512, 70000, 10, 4),
    (64, 256, 2048, 8, 8),
])
def test_vocab_parallel_fused_matches_oracle_and_recompute(N, d, V, ign, R):
    x, xc = device_inputs(_wl(N, d, V, ign))
    out = _emulate_fused(x, V, R)
    check_ce_fused(out, O.ce_fused(xc["H"], xc["W"], xc["labels"]))
    rec = _emulate(x, V, R)
    assert torch.equal(out["lse"], rec["lse"]) and torch.equal(out["argmax"], rec["argmax"])
    check_grad(out["dH"], rec["dH"], "dH fused vs recompute")
    check_grad(out["dW"], rec["dW"], "dW fused vs recompute")
    again = _emulate_fused(x, V, R)
    assert torch.equal(again["dH"], out["dH"]) and torch.equal(again["dW"], out["dW"])


def test_vocab_parallel_fused_sum_row_temperature_given_count():
    N, d, V = 140, 128, 2600
    x, xc = device_inputs(_wl(N, d, V, 6))
    t = torch.linspace(0.6, 1.4, N, dtype=torch.float32)
    out = _emulate_fused(x, V, 3, tau=t.cuda(), mean=False)
    check_ce_fused(out, O.ce_fused(xc["H"], xc["W"], xc["labels"], mean=False, tau=t.numpy()))
    n = torch.tensor([50], dtype=torch.int32, device="cuda")
    out = _emulate_fused(x, V, 2, n_given=n)
    f = O.ce_forward(xc["H"], xc["W"], xc["labels"])
    g = np.where(xc["labels"].numpy() >= 0, 1.0 / 50, 0.0)
    ref = O.backward(O.BWD_CE, xc["H"], xc["W"], xc["labels"], g)
    check_rows(out["loss_mean"], np.array([f["loss_rows"].sum() / 50]), what="mean, given count")
    check_grad(out["dH"], ref["dH"], "dH given count")
    check_grad(out["dW"], ref["dW"], "dW given count")


def test_vocab_parallel_fused_needs_one_chunk():
    N, d, V = 300, 64, 800
    x, _ = device_inputs(_wl(N, d, V, 0))
    shard = L.make_shape(N, d, 400, 0, 128, L.F_FUSED_BWD)   # 3 chunks
    ws = L.workspace(shard, L.ENTRY_VP_PARTIALS, "cuda")
    rec = torch.empty(N, 4, dtype=torch.float32, device="cuda")
    with pytest.raises(L.LmhError):
        L.lmh_vp_partials(shard, 0, V, x["H"], x["W"][:400], x["labels"], rec, workspace=ws)
    plain = L.make_shape(N, d, 400, 0, N, 0)                  # fused backward needs the flag
    with pytest.raises(L.LmhError):
        L.lmh_vp_fused_bwd(plain, 0, V, x["H"], x["W"][:400], x["labels"],
                           torch.zeros(N, dtype=torch.float32, device="cuda"), workspace=ws)


@pytest.mark.parametrize("N,d,V,ign,R,chunk", [
    (300, 192, 1000, 5, 2, 0),       # 2 shards of 500 words: ragged vocabulary tiles
    (129, 64, 4100, 3, 3, 100),      # 3 shards of 1367/1367/1366, two row chunks
    (200, 512, 70000, 10, 4, 128),   # 4 shards of 17664 (+ 17008), several K blocks
    (64, 256, 2048, 8, 8, 0),        # the tiny workload on 8 shards of 256
])
def test_vocab_parallel_matches_oracle(N, d, V, ign, R, chunk):
    x, xc = device_inputs(_wl(N, d, V, ign))
    out = _emulate(x, V, R, chunk)
    ref = O.ce_fused(xc["H"], xc["W"], xc["labels"])
    check_ce_fused(out, ref)
    again = _emulate(x, V, R, chunk)
    for k in ("lse", "loss_rows", "logprob", "argmax", "loss_mean", "dH", "dW"):
        assert torch.equal(again[k], out[k]), k
    one = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=chunk, grads=True)
    assert torch.equal(one["argmax"], out["argmax"])
    assert (one["lse"] - out["lse"]).abs().max().item() < 1e-4   # fp32 grouping differs


@pytest.mark.parametrize("kind", ["scalar", "rows"])
def test_vocab_parallel_temperature_and_logprob_objective(kind):
    N, d, V = 150, 128, 3000
    x, xc = device_inputs(_wl(N, d, V, 6))
    if kind == "scalar":
        tau, tau_ref = 0.8, 0.8
    else:
        t = torch.linspace(0.5, 1.5, N, dtype=torch.float32)
        tau, tau_ref = t.cuda(), t.numpy()
    g = torch.linspace(-1.0, 1.0, N, dtype=torch.float32)
    out = _emulate(x, V, 3, 64, tau, mode=L.BWD_LOGPROB, grad=g.cuda())
    lp = O.logprob_forward(xc["H"], xc["W"], xc["labels"], tau=tau_ref)
    check_rows(out["logprob"], lp["logprob"], what="logprob")
    check_rows(out["lse"], lp["lse"], what="lse")
    ref = O.backward(O.BWD_LOGPROB, xc["H"], xc["W"], xc["labels"], g.numpy(), tau=tau_ref)
    check_grad(out["dH"], ref["dH"], "dH")
    check_grad(out["dW"], ref["dW"], "dW")


def test_vocab_parallel_label_errors_and_ignored_rows():
    N, d, V = 96, 64, 1200
    x, xc = device_inputs(_wl(N, d, V, 0))
    y = x["labels"].clone()
    y[:10] = -100
    y[10] = -7
    y[11] = V + 5                      # out of range: flagged, row ignored
    xs = dict(x, labels=y)
    ops = CudaOps()
    plan = shard_plan(V, 2)
    recs = torch.stack([ops.partials(x["H"], x["W"][a:b], y, a, V) for a, b in plan])
    shape = L.make_shape(N, d, V)
    ws = L.workspace(shape, L.ENTRY_VP_COMBINE, "cuda")
    f32 = torch.float32
    loss, lse = torch.empty(N, dtype=f32, device="cuda"), torch.empty(N, dtype=f32, device="cuda")
    nv = torch.empty(1, dtype=torch.int32, device="cuda")
    L.lmh_vp_combine(shape, 2, recs, y, loss, lse, n_valid=nv, workspace=ws)
    assert L.lmh_read_errors(ws) & L.DEVERR_LABEL_RANGE
    assert int(nv.item()) == N - 12
    assert torch.all(loss[:12] == 0)
    out = _emulate(xs, V, 2)
    ref = O.ce_fused(xc["H"], xc["W"], y.cpu())
    check_rows(out["loss_rows"], ref["loss_rows"], what="loss_rows")
    check_grad(out["dH"], ref["dH"], "dH")
    check_grad(out["dW"], ref["dW"], "dW")


def test_vocab_parallel_caller_accumulator_and_host_rejections():
    N, d, V = 80, 64, 900
    x, xc = device_inputs(_wl(N, d, V, 2))
    plan = shard_plan(V, 2)
    ops = CudaOps()
    f = ops.combine(torch.stack([ops.partials(x["H"], x["W"][a:b], x["labels"], a, V)
                                 for a, b in plan]), x["labels"], V, d)
    accs = []
    for a, b in plan:
        acc = torch.zeros(b - a, d, dtype=torch.float32, device="cuda")
        _, dw = ops.backward(L.BWD_CE, x["H"], x["W"][a:b], x["labels"], f["lse"], None, a, V,
                             32, True, None, acc)
        assert torch.equal(dw, acc.to(torch.bfloat16))
        accs.append(acc)
    ref = O.ce_fused(xc["H"], xc["W"], xc["labels"])
    check_grad(torch.cat(accs), ref["dW"], "dW_acc shards")
    # a shard that runs past V_total, and a negative offset, are refused before any launch
    shard = L.make_shape(N, d, plan[1][1] - plan[1][0])
    ws = L.workspace(shard, L.ENTRY_VP_PARTIALS, "cuda")
    rec = torch.empty(N, 4, dtype=torch.float32, device="cuda")
    for v0 in (V - 10, -1):
        with pytest.raises(L.LmhError):
            L.lmh_vp_partials(shard, v0, V, x["H"], x["W"][plan[1][0]:], x["labels"], rec,
                              workspace=ws)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_vocab_parallel_class_on_one_rank():
    # the class's collectives over one NCCL rank: the same results as the one-device entries
    import torch.distributed as dist
    N, d, V = 130, 128, 2100
    x, xc = device_inputs(_wl(N, d, V, 4))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        vp = VocabParallelCE(V)
        f = vp.forward(x["H"], x["W"], x["labels"])
        b = vp.backward(x["H"], x["W"], x["labels"], f["lse"])
        fb = vp.forward_backward(x["H"], x["W"], x["labels"])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref = O.ce_fused(xc["H"], xc["W"], xc["labels"])
    check_ce_fused(dict(f, dH=b["dH"], dW=b["dW"]), ref)
    check_ce_fused(fb, ref)


def _scatter_buffers(N, d, R):
    """Stand-ins for the ranks' symmetric buffers on this one GPU: R receive buffers (NaN, so
    a row never written shows) and R full dH outputs, with their address tables."""
    from lm_head_cross_tcgen05_b200.vocab_parallel import row_slices
    sizes = [b - a for a, b in row_slices(N, R)]
    recv = [torch.full((R * max(sizes) * d,), float("nan"), device="cuda") for _ in range(R)]
    outs = [torch.zeros(N, d, dtype=torch.bfloat16, device="cuda") for _ in range(R)]
    rt = torch.tensor([t.data_ptr() for t in recv], dtype=torch.int64, device="cuda")
    ot = torch.tensor([t.data_ptr() for t in outs], dtype=torch.int64, device="cuda")
    return sizes, recv, outs, rt, ot


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("N,d,V,R", [
    (300, 192, 1000, 2),
    (129, 128, 4100, 3),       # ragged row slices (43 each)
    (64, 256, 2048, 8),
    (5, 64, 900, 8),           # fewer rows than ranks: three ranks reduce nothing
])
def test_row_scatter_exchange_matches_collective_path(fused, N, d, V, R):
    # the dH GEMM epilogue writes every fp32 row into its reducing rank's buffer (local buffers
    # stand in for peer memory); each rank's reduce stores its bf16 slice into every dH:
    # the same bits as the gathered, rank-ordered sum
    x, xc = device_inputs(_wl(N, d, V, 3 if N > 10 else 0))
    ref = (_emulate_fused if fused else _emulate)(x, V, R)
    H, W, y = x["H"], x["W"], x["labels"]
    ops = CudaOps()
    plan = shard_plan(V, R)
    sizes, recv, outs, rt, ot = _scatter_buffers(N, d, R)
    if fused:
        recs, states = zip(*[ops.partials_fused(H, W[a:b], y, a, V) for a, b in plan])
    else:
        recs = [ops.partials(H, W[a:b], y, a, V) for a, b in plan]
    f = ops.combine(torch.stack(list(recs)), y, V, d)
    dWs = []
    for r, (a, b) in enumerate(plan):
        if fused:
            part, dw = ops.fused_backward(states[r], H, W[a:b], y, f["lse"], a, V,
                                          dest=(rt, R, r))
        else:
            part, dw = ops.backward(L.BWD_CE, H, W[a:b], y, f["lse"], None, a, V,
                                    dest=(rt, R, r))
        assert part is None
        dWs.append(dw)
    for j in range(R):
        parts = recv[j][: R * sizes[j] * d].view(R, sizes[j], d)
        L.lmh_vp_reduce_rows_to(parts, ot, R, sum(sizes[:j]))
    torch.cuda.synchronize()
    for k in range(R):
        assert torch.equal(outs[k], ref["dH"]), k
    assert torch.equal(torch.cat(dWs), ref["dW"])
    check_grad(outs[0], O.ce_fused(xc["H"], xc["W"], xc["labels"])["dH"], "dH")


def test_row_scatter_argument_checks():
    N, d, V = 40, 64, 600
    x, _ = device_inputs(_wl(N, d, V, 0))
    shard = L.make_shape(N, d, 300, 0, 0, L.F_MEAN)
    ws = L.workspace(shard, L.ENTRY_VP_BWD, "cuda")
    lse = torch.zeros(N, dtype=torch.float32, device="cuda")
    _, recv, _, rt, _ = _scatter_buffers(N, d, 2)
    part = torch.empty(N, d, dtype=torch.float32, device="cuda")
    for dest, dh in [((rt, 2, 2), None), ((rt, 2, -1), None), ((rt, 2, 0), part)]:
        with pytest.raises(L.LmhError, match="INVALID_ARG"):
            L.lmh_vp_loss_bwd(shard, L.BWD_CE, 0, V, x["H"], x["W"][:300], x["labels"], lse,
                              None, dh, None, None, dest, workspace=ws)


def _emulate_support(x, ids, V, R, mode, grad=None, ref=None, tau=None, chunk=0):
    H, W = x["H"], x["W"]
    d = H.shape[1]
    ops = CudaOps()
    plan = shard_plan(V, R)
    recs = [ops.support_partials(H, W[a:b], ids, a, V, chunk, tau) for a, b in plan]
    f = ops.support_combine(torch.stack(recs), ids, ref, V, d)
    parts, dWs = zip(*[ops.support_backward(mode, H, W[a:b], ids, f["lse"], grad, ref, a, V,
                                            chunk, True, tau) for a, b in plan])
    f["dH"] = ops.reduce_rows(torch.stack(list(parts)))
    f["dW"] = torch.cat(dWs)
    torch.cuda.synchronize()
    return f


@pytest.mark.parametrize("N,d,V,K,R,chunk,tau", [
    (150, 128, 2500, 16, 2, 0, None),
    (96, 256, 5000, 8, 3, 40, "scalar"),    # three row chunks, a temperature
    (64, 128, 2048, 64, 8, 0, None),        # 8 shards of 256: most candidates off-shard
])
def test_vocab_parallel_support_matches_oracle(N, d, V, K, R, chunk, tau):
    x, xc = device_inputs(ragged(N, d, V, seed=5000 + N, K=K))
    ids = x["ids"].clone()
    ids[0, -1] = -1                  # padding
    ids[1, 1] = ids[1, 0]            # a repeated id counts once per slot
    ids[2, 0] = V + 3                # out of range: padding (and flagged)
    ids_c = ids.cpu()
    t_dev, t_ref = (0.75, 0.75) if tau else (None, None)
    out = _emulate_support(x, ids, V, R, L.BWD_SUPPORT_KL, ref=x["ref_logp"], tau=t_dev,
                           chunk=chunk)
    rk = O.support_kl(xc["H"], xc["W"], ids_c, xc["ref_logp"], tau=t_ref)
    check_rows(out["lp"], rk["lp"], what="lp")
    check_rows(out["lse"], rk["lse"], what="lse")
    check_rows(out["kl_rows"], rk["kl_rows"], what="kl_rows")
    check_rows(out["kl_mean"], np.array([rk["kl_mean"]]), what="kl_mean")
    ref = O.backward(O.BWD_SUPPORT_KL, xc["H"], xc["W"], ids_c, np.full(N, 1.0 / N),
                     xc["ref_logp"], tau=t_ref)
    check_grad(out["dH"], ref["dH"], "dH KL")
    check_grad(out["dW"], ref["dW"], "dW KL")
    again = _emulate_support(x, ids, V, R, L.BWD_SUPPORT_KL, ref=x["ref_logp"], tau=t_dev,
                             chunk=chunk)
    assert torch.equal(again["dH"], out["dH"]) and torch.equal(again["lp"], out["lp"])
    gam = torch.linspace(-1.0, 1.0, N * K, dtype=torch.float32).view(N, K)
    lpo = _emulate_support(x, ids, V, R, L.BWD_SUPPORT_LOGPROB, grad=gam.cuda(), tau=t_dev,
                           chunk=chunk)
    ref2 = O.backward(O.BWD_SUPPORT_LOGPROB, xc["H"], xc["W"], ids_c, gam.numpy(), tau=t_ref)
    check_grad(lpo["dH"], ref2["dH"], "dH support log-prob")
    check_grad(lpo["dW"], ref2["dW"], "dW support log-prob")
    one = L.support_logprob(x["H"], x["W"], ids, chunk_rows=chunk, temperature=t_dev)
    assert (one["lse"] - out["lse"]).abs().max().item() < 1e-4


def test_vocab_parallel_support_refuses_renorm():
    N, d, V, K = 16, 64, 600, 4
    x, _ = device_inputs(ragged(N, d, V, seed=5100, K=K))
    shard = L.make_shape(N, d, 300, K, 0, L.F_SUPPORT_RENORM)
    ws = L.workspace(L.make_shape(N, d, 300, K), L.ENTRY_VP_SUPPORT_PARTIALS, "cuda")
    rec = torch.empty(N, K + 1, dtype=torch.float32, device="cuda")
    with pytest.raises(L.LmhError, match="INVALID_ARG"):
        L.lmh_vp_support_partials(shard, 0, V, x["H"], x["W"][:300], x["ids"], rec, workspace=ws)


def test_peer_memory_dh_exchange_runs_on_one_rank():
    # The vocabulary-parallel dH exchange over peer memory on one NCCL rank, p2p forced on:
    # symmetric buffers, the barrier kernel, the dH GEMM's row scatter and the reduce into the
    # symmetric output, twice. The results must be the collective path's bits.
    import torch.distributed as dist
    N, d, V = 130, 128, 2100
    x, xc = device_inputs(_wl(N, d, V, 4))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        ref = VocabParallelCE(V).forward_backward(x["H"], x["W"], x["labels"])
        vp = VocabParallelCE(V)
        vp.p2p = True
        outs = [vp.forward_backward(x["H"], x["W"], x["labels"]) for _ in range(2)]
        torch.cuda.synchronize()
        vp.check_exchange()
        assert vp._sym["epoch"] == 6
        vp._sym = None
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    for out in outs:
        assert torch.equal(out["dH"], ref["dH"]) and torch.equal(out["dW"], ref["dW"])
        assert torch.equal(out["lse"], ref["lse"])
    check_ce_fused(outs[0], O.ce_fused(xc["H"], xc["W"], xc["labels"]))
