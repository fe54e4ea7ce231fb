"""CUDA-graph capture of the library's entries. They enqueue work on the caller's stream
without allocating memory or synchronising the host, so a captured step replays as the same
kernels with the same bits. Only the first call per kernel variant and device does one-time
host work (function attributes, occupancy query), so it must come before the capture."""
from __future__ import annotations

import pytest
import torch

import lm_head_cross_tcgen05_b200 as L
from tests.gpu_common import O, check_ce_fused, device_inputs
from workloads import make_inputs, ragged

pytestmark = pytest.mark.gpu


def _fused_step(N, d, V, chunk):
    shape = L.make_shape(N, d, V, 0, chunk, L.F_MEAN | L.F_FUSED_BWD)
    ws = L.workspace(shape, L.ENTRY_LOSS_FWD, "cuda")
    f32, dev = torch.float32, "cuda"
    out = dict(loss_rows=torch.empty(N, dtype=f32, device=dev),
               lse=torch.empty(N, dtype=f32, device=dev),
               logprob=torch.empty(N, dtype=f32, device=dev),
               argmax=torch.empty(N, dtype=torch.int32, device=dev),
               loss_mean=torch.empty(1, dtype=f32, device=dev),
               n_valid=torch.empty(1, dtype=torch.int32, device=dev),
               dH=torch.empty(N, d, dtype=torch.bfloat16, device=dev),
               dW=torch.empty(V, d, dtype=torch.bfloat16, device=dev))

    def run(H, W, y):
        L.lmh_loss_fwd(shape, H, W, y, out["loss_rows"], out["lse"], out["logprob"],
                       out["argmax"], out["loss_mean"], out["n_valid"], None, out["dH"],
                       out["dW"], None, workspace=ws)
    return run, out


def _snapshot(out):
    return {k: v.clone() for k, v in out.items()}


@pytest.mark.parametrize("chunk", [0, 128])
def test_fused_step_graph_replays_same_bits(chunk):
    N, d, V = 300, 192, 1000
    x, xc = device_inputs(ragged(N, d, V, n_ignored=5, seed=4600))
    H, W, y = x["H"].clone(), x["W"].clone(), x["labels"].clone()   # the graph's input buffers
    run, out = _fused_step(N, d, V, chunk)
    run(H, W, y)                          # first call: one-time host setup, outside the capture
    torch.cuda.synchronize()
    eager = _snapshot(out)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run(H, W, y)
    torch.cuda.current_stream().wait_stream(s)
    with torch.cuda.graph(g):
        run(H, W, y)
    for v in out.values():
        v.zero_()
    g.replay()
    torch.cuda.synchronize()
    for k in eager:
        assert torch.equal(out[k], eager[k]), k
    check_ce_fused(out, O.ce_fused(xc["H"], xc["W"], xc["labels"]))
    # new inputs copied into the captured buffers: the replay computes the new step
    x2 = make_inputs(ragged(N, d, V, n_ignored=9, seed=4601), device="cuda")
    H.copy_(x2["H"]); W.copy_(x2["W"]); y.copy_(x2["labels"])
    g.replay()
    torch.cuda.synchronize()
    replayed = _snapshot(out)
    run(H, W, y)
    torch.cuda.synchronize()
    for k in replayed:
        assert torch.equal(out[k], replayed[k]), k


def test_support_kl_and_backward_graph():
    N, d, V, K = 96, 128, 2500, 16
    x, xc = device_inputs(ragged(N, d, V, seed=4700, K=K))
    shape = L.make_shape(N, d, V, K, 0, L.F_MEAN)
    ws_f = L.workspace(shape, L.ENTRY_SUPPORT_KL, "cuda")
    ws_b = L.workspace(shape, L.ENTRY_LOSS_BWD, "cuda")
    f32 = torch.float32
    kl, klm = torch.empty(N, dtype=f32, device="cuda"), torch.empty(1, dtype=f32, device="cuda")
    lp, lse = torch.empty(N, K, dtype=f32, device="cuda"), torch.empty(N, dtype=f32, device="cuda")
    dH = torch.empty(N, d, dtype=torch.bfloat16, device="cuda")
    dW = torch.empty(V, d, dtype=torch.bfloat16, device="cuda")

    def step():
        L.lmh_support_kl(shape, x["H"], x["W"], x["ids"], x["ref_logp"], kl, klm, lp, lse,
                         workspace=ws_f)
        L.lmh_loss_bwd(shape, L.BWD_SUPPORT_KL, x["H"], x["W"], x["ids"], lse, None,
                       x["ref_logp"], dH, dW, workspace=ws_b)
    step()
    torch.cuda.synchronize()
    eager = [t.clone() for t in (kl, klm, lp, lse, dH, dW)]
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream().wait_stream(s)
    with torch.cuda.graph(g):
        step()
    for t in (kl, klm, lp, lse, dH, dW):
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    for a, b in zip((kl, klm, lp, lse, dH, dW), eager):
        assert torch.equal(a, b)
