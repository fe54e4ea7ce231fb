"""GPU parity of the row data-parallel steps (through the C ABI) against the fp64 oracle on the
concatenated batch, and of the two entries and the accumulator flag they add.

One GPU stands in for R ranks: each rank's steps run one after another on its own rows, the
integer all-reduce of the valid counts is a sum of R one-element tensors, and each exchange is
a stack in rank order. No kernel of one rank waits for another, so this runs the device code
each rank would run, with the same order of additions. (DataParallelCE's exchange logic itself
is covered on CPU ranks over gloo, and on one NCCL rank here.)"""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch

import lm_head_cross_tcgen05_b200 as L
from lm_head_cross_tcgen05_b200.data_parallel import CudaOps, DataParallelCE
from tests.gpu_common import O, check_ce_fused, check_grad, device_inputs
from workloads import ragged

pytestmark = pytest.mark.gpu


def _bounds(split):
    out, a = [], 0
    for n in split:
        out.append((a, a + n))
        a += n
    return out


def _emulate(x, split, tau=None, mean=True, chunk=0, mode=L.BWD_CE, grad=None, scalar=False):
    H, W, y = x["H"], x["W"], x["labels"]
    V = W.shape[0]
    ops = CudaOps()
    bounds = _bounds(split)
    n = torch.stack([ops.count_valid(y[a:b], V) for a, b in bounds]).sum(0).to(torch.int32)
    outs = [ops.fused(H[a:b], W, y[a:b], n, mode=mode,
                      grad=None if grad is None else grad if scalar else grad[a:b].contiguous(),
                      weighted=grad is not None, mean=mean, scalar_grad=scalar, chunk_rows=chunk,
                      temperature=tau)
            for a, b in bounds]
    f = {k: torch.cat([o[k] for o in outs]) for k in ("loss_rows", "lse", "logprob", "argmax",
                                                       "dH")}
    f["loss_mean"] = ops.sum_ranks(torch.stack([o["loss_mean"] for o in outs]))
    f["dW"] = ops.reduce_rows(torch.stack([o["dW_part"] for o in outs]))
    f["n_valid"] = n
    torch.cuda.synchronize()
    return f


@pytest.mark.parametrize("split,d,V,ign,chunk", [
    ((150, 150), 192, 1000, 5, 0),
    ((300, 0, 129, 71), 256, 2048, 9, 0),      # a rank without rows
    ((200, 57), 128, 70000, 6, 0),             # V >= 65536: dH splits the vocabulary
    ((500, 333, 16), 128, 4100, 0, 128),       # several chunks per rank
    ((37,) * 8, 64, 3000, 4, 0),
])
def test_data_parallel_matches_oracle_on_concatenated_batch(split, d, V, ign, chunk):
    N = sum(split)
    x, xc = device_inputs(ragged(N, d, V, n_ignored=ign, seed=4100 + N + d + V))
    out = _emulate(x, split, chunk=chunk)
    check_ce_fused(out, O.ce_fused(xc["H"], xc["W"], xc["labels"]))
    # per-row results do not depend on how the rows are split over ranks
    one = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True, chunk_rows=chunk)
    for k in ("loss_rows", "lse", "logprob", "argmax"):
        assert torch.equal(out[k], one[k]), k
    check_grad(out["dH"], one["dH"].float(), "dH ranks vs one device")
    check_grad(out["dW"], one["dW"].float(), "dW ranks vs one device")
    again = _emulate(x, split, chunk=chunk)
    for k in ("dH", "dW", "loss_mean"):
        assert torch.equal(again[k], out[k]), k


@pytest.mark.parametrize("kind", ["sum", "weighted", "scalar", "temperature"])
def test_data_parallel_objectives(kind):
    split, d, V = (90, 45, 121), 128, 5000
    N = sum(split)
    x, xc = device_inputs(ragged(N, d, V, n_ignored=7, seed=4200))
    if kind == "sum":
        out = _emulate(x, split, mean=False)
        check_ce_fused(out, O.ce_fused(xc["H"], xc["W"], xc["labels"], mean=False))
    elif kind == "temperature":
        out = _emulate(x, split, tau=0.7)
        check_ce_fused(out, O.ce_fused(xc["H"], xc["W"], xc["labels"], tau=0.7))
    elif kind == "scalar":  # an upstream gradient g of the global mean: weights g / n
        g = torch.tensor([2.5], device="cuda")
        out = _emulate(x, split, grad=g, scalar=True)
        ref = O.ce_fused(xc["H"], xc["W"], xc["labels"])
        check_ce_fused(dict(out, dH=None, dW=None), ref, grads=False)
        check_grad(out["dH"], 2.5 * ref["dH"], "dH scalar")
        check_grad(out["dW"], 2.5 * ref["dW"], "dW scalar")
    else:  # policy-gradient style: -sum_i A_i logprob_i, the per-row weights as given
        A = torch.linspace(-1.0, 2.0, N, dtype=torch.float32)
        out = _emulate(x, split, mode=L.BWD_LOGPROB, grad=(-A).cuda())
        f = O.ce_forward(xc["H"], xc["W"], xc["labels"])
        rb = O.backward(O.BWD_LOGPROB, xc["H"], xc["W"], xc["labels"], -A.double().numpy())
        check_ce_fused(dict(out, dH=None, dW=None), f, grads=False)
        check_grad(out["dH"], rb["dH"], "dH weighted")
        check_grad(out["dW"], rb["dW"], "dW weighted")


def test_count_valid_and_rank_sum_entries():
    y = torch.tensor([-100, 0, 5, 99, 100, 7, -1, 250], dtype=torch.int32, device="cuda")
    n = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    L.lmh_count_valid(y, 100, n)
    assert int(n.item()) == 4                            # 0, 5, 99, 7
    L.lmh_count_valid(y[:0], 100, n)
    assert int(n.item()) == 0
    g = torch.Generator().manual_seed(5)
    big = torch.randint(-3, 1003, (1_000_003,), generator=g, dtype=torch.int32)
    L.lmh_count_valid(big.cuda(), 1000, n)
    assert int(n.item()) == int(((big >= 0) & (big < 1000)).sum())
    for R, m in ((1, 1), (3, 7), (8, 100_003)):
        parts = (torch.randn(R, m, generator=g) * torch.logspace(-30, 30, m)).float()
        out = torch.full((m,), float("nan"), device="cuda")
        L.lmh_reduce_ranks_f32(parts.cuda(), out)
        ref = parts.numpy()[0].copy()
        for r in range(1, R):                                  # fp32 adds in rank order
            ref = (ref + parts.numpy()[r]).astype(np.float32)
        assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("chunk", [0, 100])
def test_dw_acc_store_flag_overwrites(chunk):
    # the store flag gives the same accumulator bits as adding into zeros, whatever the
    # buffer held before, for the fused forward, the recompute backward, the renormalised
    # support backward and a call without rows
    N, d, V, K = 333, 128, 3000, 5
    x, _ = device_inputs(ragged(N, d, V, n_ignored=4, seed=4300, K=K))
    H, W, y = x["H"], x["W"], x["labels"]
    base = L.F_FUSED_BWD | L.F_DW_ACC_GIVEN | L.F_MEAN

    def fwd(acc, flags, rows=N):
        sh = L.make_shape(rows, d, V, 0, chunk, flags)
        ws = L.workspace(sh, L.ENTRY_LOSS_FWD, "cuda")
        f32 = dict(dtype=torch.float32, device="cuda")
        dW = torch.empty(V, d, dtype=torch.bfloat16, device="cuda")
        L.lmh_loss_fwd(sh, H[:rows], W, y[:rows], torch.empty(rows, **f32),
                       torch.empty(rows, **f32), dH=torch.empty(rows, d, dtype=torch.bfloat16,
                                                                device="cuda"),
                       dW=dW, dW_acc=acc, workspace=ws)
        return dW

    zero = torch.zeros(V, d, device="cuda")
    junk = torch.full((V, d), float("nan"), device="cuda")
    a = fwd(zero, base)
    b = fwd(junk, base | L.F_DW_ACC_STORE)
    assert torch.equal(zero, junk) and torch.equal(a, b)
    junk.fill_(3.0)
    fwd(junk, base | L.F_DW_ACC_STORE, rows=0)
    assert not junk.any()

    lse = L.loss_fwd(H, W, y)["lse"]

    def bwd(acc, flags, mode, targets, renorm=False):
        fl = flags | (L.F_SUPPORT_RENORM if renorm else 0)
        sh = L.make_shape(N, d, V, K if targets.dim() == 2 else 0, chunk, fl)
        ws = L.workspace(sh, L.ENTRY_LOSS_BWD, "cuda")
        grad = (torch.linspace(-1, 1, targets.numel(), device="cuda")
                .reshape(targets.shape).contiguous())
        lse_ = (L.support_logprob(H, W, targets, renorm=True)["lse"] if renorm else lse)
        L.lmh_loss_bwd(sh, mode, H, W, targets, lse_, grad, dW_acc=acc, workspace=ws)

    for mode, targets, renorm in ((L.BWD_CE, y, False),
                                  (L.BWD_SUPPORT_LOGPROB, x["ids"], True)):
        zero.zero_()
        junk.fill_(float("nan"))
        bwd(zero, L.F_DW_ACC_GIVEN, mode, targets, renorm)
        bwd(junk, L.F_DW_ACC_GIVEN | L.F_DW_ACC_STORE, mode, targets, renorm)
        torch.cuda.synchronize()
        assert torch.equal(zero, junk), (mode, renorm)


@pytest.mark.parametrize("split,d,V,weighted", [
    ((150, 150), 192, 1000, False),
    ((300, 0, 129, 71), 256, 2048, False),     # a rank without rows zeroes its slots
    ((37,) * 8, 64, 3000, False),
    ((40, 21, 7), 128, 70000, False),
    ((90, 45, 121), 128, 5000, True),          # weighted log-prob objective, temperature
])
def test_dw_row_scatter_matches_collective_path(split, d, V, weighted):
    # the dW GEMM storing fp32 rows into the reducing ranks' receive buffers (stand-ins on
    # this GPU, NaN so a row never written shows), then each slice reduced into every rank's
    # dW: the collective path's bits
    from lm_head_cross_tcgen05_b200._ranks import row_slices
    N, R = sum(split), len(split)
    x, _ = device_inputs(ragged(N, d, V, n_ignored=3, seed=4500 + N + V))
    kw = {}
    if weighted:
        kw = dict(mode=L.BWD_LOGPROB, tau=0.8,
                  grad=torch.linspace(-1.0, 2.0, N, device="cuda").contiguous())
    ref = _emulate(x, split, **kw)
    H, W, y = x["H"], x["W"], x["labels"]
    sizes = [b - a for a, b in row_slices(V, R)]
    recv = [torch.full((R * max(sizes) * d,), float("nan"), device="cuda") for _ in range(R)]
    outs = [torch.zeros(V, d, dtype=torch.bfloat16, device="cuda") for _ in range(R)]
    rt = torch.tensor([t.data_ptr() for t in recv], dtype=torch.int64, device="cuda")
    ot = torch.tensor([t.data_ptr() for t in outs], dtype=torch.int64, device="cuda")
    ops = CudaOps()
    got = [ops.fused_scatter(H[a:b], W, y[a:b], ref["n_valid"], (rt, R, r),
                             mode=kw.get("mode", L.BWD_CE), temperature=kw.get("tau"),
                             grad=kw["grad"][a:b].contiguous() if weighted else None)
           for r, (a, b) in enumerate(_bounds(split))]
    start = 0
    for j in range(R):
        ops.reduce_rows_to(recv[j][: R * sizes[j] * d].view(R, sizes[j], d), ot, R, start)
        start += sizes[j]
    torch.cuda.synchronize()
    for k in range(R):
        assert torch.equal(outs[k], ref["dW"]), k
    assert torch.equal(torch.cat([g["dH"] for g in got]), ref["dH"])
    assert torch.equal(torch.cat([g["lse"] for g in got]), ref["lse"])
    assert torch.equal(ops.sum_ranks(torch.stack([g["loss_mean"] for g in got])),
                       ref["loss_mean"])
    # the scatter runs the rank's rows as one chunk
    sh = L.make_shape(N, d, V, 0, N // 2, L.F_FUSED_BWD | L.F_MEAN)
    with pytest.raises(L.LmhError):
        L.lmh_dp_loss_fwd_bwd(sh, L.BWD_CE, H, W, y, None, torch.empty(N, device="cuda"),
                              torch.empty(N, device="cuda"), dest=(rt, R, 0),
                              workspace=L.workspace(sh, L.ENTRY_LOSS_FWD_BWD, "cuda"))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_data_parallel_class_on_one_rank():
    # the class over one NCCL rank: the one-device fused step's results
    import torch.distributed as dist
    N, d, V = 300, 128, 2100
    x, xc = device_inputs(ragged(N, d, V, n_ignored=6, seed=4400))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        out = DataParallelCE().forward_backward(x["H"], x["W"], x["labels"])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    check_ce_fused(out, O.ce_fused(xc["H"], xc["W"], xc["labels"]))
    one = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True)
    assert torch.equal(out["dH"], one["dH"]) and torch.equal(out["dW"], one["dW"])
    assert torch.equal(out["loss_mean"], one["loss_mean"])
    # one rank's direct bf16 dW: the bits of the rank-ordered sum of its one fp32 part
    ops = CudaOps()
    n = ops.count_valid(x["labels"], V)
    p = ops.fused(x["H"], x["W"], x["labels"], n)
    q = ops.fused(x["H"], x["W"], x["labels"], n, bf16_dW=True)
    assert torch.equal(ops.reduce_rows(p["dW_part"][None]), q["dW"])
    assert torch.equal(p["dH"], q["dH"]) and torch.equal(p["loss_mean"], q["loss_mean"])


def test_peer_memory_exchange_runs_on_one_rank():
    # The peer-memory dW exchange end to end on one NCCL rank, with p2p forced on (a single rank
    # normally skips the exchange): torch symmetric memory for the receive buffer, the dW
    # outputs and the barrier's signal words; the library's barrier kernel; the dW GEMM's row
    # scatter; the rank-order reduce into the symmetric output. Two steps, so the second one
    # checks the first one's barrier record and reuses the buffers. The dW must be the bits of
    # the one-device fused step (the reduce of one fp32 part is its bf16 cast).
    import torch.distributed as dist
    N, d, V = 300, 128, 2100
    x, xc = device_inputs(ragged(N, d, V, n_ignored=6, seed=4410))
    one = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        dp = DataParallelCE()
        dp.p2p = True
        outs = [dp.forward_backward(x["H"], x["W"], x["labels"]) for _ in range(2)]
        torch.cuda.synchronize()
        dp.check_exchange()                        # no barrier gave up
        assert dp._sym["epoch"] == 6               # three barriers per step
        dp._sym = None
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    for out in outs:
        assert torch.equal(out["dW"], one["dW"])
        assert torch.equal(out["dH"], one["dH"]) and torch.equal(out["lse"], one["lse"])
        assert torch.equal(out["loss_mean"], one["loss_mean"])
    check_ce_fused(outs[0], O.ce_fused(xc["H"], xc["W"], xc["labels"]))
