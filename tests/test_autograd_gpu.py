"""The torch.autograd entry points (lm_head_cross_tcgen05_b200.autograd) against the fp64
oracle: forward values, and H.grad / W.grad after backward() with per-row and scalar upstream
gradients."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import lm_head_cross_tcgen05_b200 as L
from lm_head_cross_tcgen05_b200 import autograd as A
from tests.gpu_common import O, check_grad, check_rows, device_inputs
from workloads import ragged

pytestmark = pytest.mark.gpu


def _leaf(x):
    H = x["H"].clone().requires_grad_(True)
    W = x["W"].clone().requires_grad_(True)
    return H, W


def test_log_probs_backward_per_row_grad():
    x, xc = device_inputs(ragged(200, 192, 3000, n_ignored=7, seed=4100))
    H, W = _leaf(x)
    lp = A.log_probs(H, W, x["labels"], chunk_rows=96)
    c = torch.linspace(-2.0, 2.0, 200, dtype=torch.float32)
    (lp * c.cuda()).sum().backward()
    ref_f = O.logprob_forward(xc["H"], xc["W"], xc["labels"])
    check_rows(lp.detach(), ref_f["logprob"], what="logprob")
    ref = O.backward(O.BWD_LOGPROB, xc["H"], xc["W"], xc["labels"], c.numpy())
    check_grad(H.grad, ref["dH"], "dH")
    check_grad(W.grad, ref["dW"], "dW")


@pytest.mark.parametrize("reduction,scale", [("mean", 3.0), ("sum", -0.5), ("none", None)])
def test_cross_entropy_reductions(reduction, scale):
    x, xc = device_inputs(ragged(160, 128, 2100, n_ignored=9, seed=4200))
    H, W = _leaf(x)
    loss = A.cross_entropy(H, W, x["labels"], reduction=reduction, chunk_rows=64)
    f = O.ce_forward(xc["H"], xc["W"], xc["labels"])
    if reduction == "none":
        c = torch.linspace(0.5, 1.5, 160, dtype=torch.float32)
        (loss * c.cuda()).sum().backward()
        check_rows(loss.detach(), f["loss_rows"], what="loss_rows")
        g = c.numpy()
    else:
        (loss * scale).backward()
        s = f["loss_rows"].sum()
        want = s / f["n_valid"] if reduction == "mean" else s
        assert abs(loss.item() - want) < 2e-3 * max(1.0, abs(want))
        g = np.full(160, scale / (f["n_valid"] if reduction == "mean" else 1.0))
    ref = O.backward(O.BWD_CE, xc["H"], xc["W"], xc["labels"], g)
    check_grad(H.grad, ref["dH"], "dH")
    check_grad(W.grad, ref["dW"], "dW")


@pytest.mark.parametrize("renorm", [False, True])
def test_support_kl_mean_and_log_probs(renorm):
    wl = ragged(96, 128, 2500, seed=4300, K=16)
    x, xc = device_inputs(wl)
    H, W = _leaf(x)
    kl = A.support_kl(H, W, x["ids"], x["ref_logp"], renorm=renorm)
    (2.0 * kl).backward()
    if renorm:
        rk = O.support_renorm_kl(xc["H"], xc["W"], xc["ids"], xc["ref_logp"])
        ref = O.backward_renorm(O.BWD_SUPPORT_KL, xc["H"], xc["W"], xc["ids"],
                                np.full(96, 2.0 / 96), xc["ref_logp"])
    else:
        rk = O.support_kl(xc["H"], xc["W"], xc["ids"], xc["ref_logp"])
        ref = O.backward(O.BWD_SUPPORT_KL, xc["H"], xc["W"], xc["ids"], np.full(96, 2.0 / 96),
                         xc["ref_logp"])
    assert abs(kl.item() - rk["kl_mean"]) < 2e-3
    check_grad(H.grad, ref["dH"], "dH")
    check_grad(W.grad, ref["dW"], "dW")
    # per-candidate log-probs with a per-element upstream gradient, only H requiring grad
    H2 = x["H"].clone().requires_grad_(True)
    lp = A.support_log_probs(H2, x["W"], x["ids"], renorm=renorm)
    gam = torch.linspace(-1.0, 1.0, 96 * 16, dtype=torch.float32).view(96, 16)
    (lp * gam.cuda()).sum().backward()
    if renorm:
        r2 = O.backward_renorm(O.BWD_SUPPORT_LOGPROB, xc["H"], xc["W"], xc["ids"], gam.numpy())
    else:
        r2 = O.backward(O.BWD_SUPPORT_LOGPROB, xc["H"], xc["W"], xc["ids"], gam.numpy())
    check_grad(H2.grad, r2["dH"], "dH support lp")


def test_scalar_grad_requires_a_pointer():
    x, _ = device_inputs(ragged(32, 64, 300, seed=4400))
    shape = L.make_shape(32, 64, 300, 0, 0, L.F_GRAD_SCALAR)
    ws = L.workspace(shape, L.ENTRY_LOSS_BWD, "cuda")
    lse = torch.zeros(32, dtype=torch.float32, device="cuda")
    dH = torch.empty(32, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.LmhError):
        L.lmh_loss_bwd(shape, L.BWD_CE, x["H"], x["W"], x["labels"], lse, None, None, dH,
                       workspace=ws)


def test_reduced_cross_entropy_uses_the_one_pass_gradient():
    # loss.backward() with g = 1 returns exactly lmh_loss_fwd's fused dH / dW (the scale by
    # g = 1 changes no bit), and the step launches no recomputing logits GEMM
    from tests.test_parity_gpu import _kernels_launched
    x, _ = device_inputs(ragged(150, 128, 1800, n_ignored=4, seed=4250))
    H, W = _leaf(x)
    res = {}

    def step():
        loss = A.cross_entropy(H, W, x["labels"], chunk_rows=64)
        loss.backward()
        res["loss"] = loss
    names = _kernels_launched(step)
    assert "gemm_logits_grad" not in names and names.count("scale_bf16") == 2
    ref = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=64, grads=True)
    assert torch.equal(H.grad, ref["dH"]) and torch.equal(W.grad, ref["dW"])
    assert torch.equal(res["loss"].detach().view(1), ref["loss_mean"])
