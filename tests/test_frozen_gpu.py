"""Frozen inputs: backward calls that produce only dH (W frozen) or only dW (H frozen), the
case the test plan of miles-ext-kernels PR #14 (tests/cake/lm_head commit, "frozen inputs")
runs. Every entry that forms a gradient takes a null dH or dW to mean "not wanted" and skips
that GEMM. Each case checks the gradient it asked for against the fp64 oracle, checks that it
has the same bits as the call that asks for both, and checks from the library's own launch
record that the other contraction did not run. Two shapes: three row chunks (the dW
accumulator walks the chunk order) and one chunk whose dH is summed over vocabulary ranges
(split-K)."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import lm_head_cross_tcgen05_b200 as L
from lm_head_cross_tcgen05_b200._abi import lib
from tests.gpu_common import O, check_grad, check_rows, device_inputs
from workloads import ragged

pytestmark = pytest.mark.gpu

# (N, d, V, ignored rows, chunk_rows, dH split over vocabulary ranges)
CASES = [
    (520, 192, 3000, 9, 200, False),   # chunks of 200, 200, 120 rows
    (300, 320, 70000, 5, 0, True),     # 4 dH tiles: V split in 2 ranges + split_sum
]
IDS = ["chunked", "split_k"]


def launched(fn):
    """(result of fn(), names of the library kernels it launched)."""
    lib().lmh_profile_read(0, None, None)
    lib().lmh_profile_enable(1)
    try:
        r = fn()
        torch.cuda.synchronize()
    finally:
        lib().lmh_profile_enable(0)
    cap = 4096
    kid, ms = (ctypes.c_int32 * cap)(), (ctypes.c_float * cap)()
    n = lib().lmh_profile_read(cap, kid, ms)
    return r, [lib().lmh_kernel_name(kid[i]).decode() for i in range(n)]


def check_frozen(both, only, names, want: str, ref: dict, split: bool):
    """`only` computed just `want` ("dH" or "dW"): oracle parity, the bits of the call that
    computed both, and the other GEMM absent from the launch record."""
    other = "dW" if want == "dH" else "dH"
    assert only.get(other) is None
    check_grad(only[want], ref[want], f"{want} only")
    assert torch.equal(only[want], both[want]), f"{want} only vs both"
    assert f"gemm_{other}" not in names, names
    assert f"gemm_{want}" in names, names
    if want == "dW":
        assert "split_sum" not in names
    elif split:
        assert "split_sum" in names


def _inputs(N, d, V, ign, K=0):
    return device_inputs(ragged(N, d, V, n_ignored=ign, K=K, seed=7100 + N + V))


@pytest.mark.parametrize("N,d,V,ign,chunk,split", CASES, ids=IDS)
@pytest.mark.parametrize("want", ["dH", "dW"])
def test_fused_ce_frozen(N, d, V, ign, chunk, split, want):
    x, xc = _inputs(N, d, V, ign)
    both = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=chunk, grads=True)
    only, names = launched(lambda: L.loss_fwd(
        x["H"], x["W"], x["labels"], chunk_rows=chunk, grads=True, want_dH=want == "dH",
        want_dW=want == "dW"))
    assert L.lmh_read_errors(only["workspace"]) == 0
    for k in ("loss_rows", "lse", "logprob", "argmax", "loss_mean", "n_valid"):
        assert torch.equal(only[k], both[k]), k
    ref = O.ce_fused(xc["H"], xc["W"], xc["labels"])
    check_rows(only["lse"], ref["lse"], what="lse")
    check_frozen(both, only, names, want, ref, split)


@pytest.mark.parametrize("N,d,V,ign,chunk,split", CASES, ids=IDS)
@pytest.mark.parametrize("want", ["dH", "dW"])
@pytest.mark.parametrize("mode", [L.BWD_CE, L.BWD_LOGPROB])
def test_recompute_backward_frozen(N, d, V, ign, chunk, split, want, mode):
    x, xc = _inputs(N, d, V, ign)
    lse = L.logprob(x["H"], x["W"], x["labels"])["lse"]
    g = torch.linspace(-1.0, 1.5, N, dtype=torch.float32) / N
    both = L.loss_bwd(mode, x["H"], x["W"], x["labels"], lse, g.cuda(), chunk_rows=chunk)
    only, names = launched(lambda: L.loss_bwd(
        mode, x["H"], x["W"], x["labels"], lse, g.cuda(), chunk_rows=chunk,
        want_dH=want == "dH", want_dW=want == "dW"))
    assert L.lmh_read_errors(only["workspace"]) == 0
    ref = O.backward(mode, xc["H"], xc["W"], xc["labels"], g.numpy())
    check_frozen(both, only, names, want, ref, split)


@pytest.mark.parametrize("N,d,V,ign,chunk,split", CASES, ids=IDS)
@pytest.mark.parametrize("want", ["dH", "dW"])
def test_weighted_one_pass_frozen(N, d, V, ign, chunk, split, want):
    # a policy-gradient-like objective, weights known before the forward
    x, xc = _inputs(N, d, V, ign)
    g = torch.linspace(-1.5, 1.0, N, dtype=torch.float32)
    both = L.loss_fwd_bwd(L.BWD_LOGPROB, x["H"], x["W"], x["labels"], g.cuda(),
                          chunk_rows=chunk)
    only, names = launched(lambda: L.loss_fwd_bwd(
        L.BWD_LOGPROB, x["H"], x["W"], x["labels"], g.cuda(), chunk_rows=chunk,
        want_dH=want == "dH", want_dW=want == "dW"))
    assert torch.equal(only["lse"], both["lse"])
    ref = O.backward(O.BWD_LOGPROB, xc["H"], xc["W"], xc["labels"], g.numpy())
    check_frozen(both, only, names, want, ref, split)


@pytest.mark.parametrize("N,d,V,ign,chunk,split", CASES, ids=IDS)
@pytest.mark.parametrize("want", ["dH", "dW"])
def test_support_kl_frozen(N, d, V, ign, chunk, split, want):
    # the mean support KL: one pass (forward + backward) and the recomputing backward
    K = 16
    x, xc = _inputs(N, d, V, ign, K=K)
    ids, ref_lp = x["ids"], x["ref_logp"]
    both = L.support_kl(x["H"], x["W"], ids, ref_lp, chunk_rows=chunk, grads=True)
    only, names = launched(lambda: L.support_kl(
        x["H"], x["W"], ids, ref_lp, chunk_rows=chunk, grads=True, want_dH=want == "dH",
        want_dW=want == "dW"))
    assert L.lmh_read_errors(only["workspace"]) == 0
    assert torch.equal(only["kl_rows"], both["kl_rows"]) and torch.equal(only["lp"], both["lp"])
    ref = O.backward(O.BWD_SUPPORT_KL, xc["H"], xc["W"], xc["ids"], np.full(N, 1.0 / N),
                     xc["ref_logp"])
    check_frozen(both, only, names, want, ref, split)
    # the recomputing backward of the same objective
    b2 = L.loss_bwd(L.BWD_SUPPORT_KL, x["H"], x["W"], ids, both["lse"], None, ref_lp,
                    chunk_rows=chunk, mean=True)
    o2, names2 = launched(lambda: L.loss_bwd(
        L.BWD_SUPPORT_KL, x["H"], x["W"], ids, both["lse"], None, ref_lp, chunk_rows=chunk,
        mean=True, want_dH=want == "dH", want_dW=want == "dW"))
    check_frozen(b2, o2, names2, want, ref, split)


@pytest.mark.parametrize("want", ["dH", "dW"])
def test_support_logprob_one_pass_frozen(want):
    # weighted support log-probs, one chunk of several tiles
    N, d, V, K = 200, 128, 5000, 12
    x, xc = _inputs(N, d, V, 0, K=K)
    g = torch.linspace(-1.0, 2.0, N * K, dtype=torch.float32).view(N, K)
    both = L.support_fwd_bwd(L.BWD_SUPPORT_LOGPROB, x["H"], x["W"], x["ids"], g.cuda())
    only, names = launched(lambda: L.support_fwd_bwd(
        L.BWD_SUPPORT_LOGPROB, x["H"], x["W"], x["ids"], g.cuda(), want_dH=want == "dH",
        want_dW=want == "dW"))
    assert torch.equal(only["lp"], both["lp"])
    ref = O.backward(O.BWD_SUPPORT_LOGPROB, xc["H"], xc["W"], xc["ids"], g.numpy())
    check_frozen(both, only, names, want, ref, False)


def test_no_gradient_at_all_runs_no_backward_gemm():
    # both inputs frozen: the one-pass entry is then a forward
    x, _ = _inputs(300, 192, 3000, 4)
    out, names = launched(lambda: L.loss_fwd_bwd(
        L.BWD_CE, x["H"], x["W"], x["labels"], None, mean=True, want_dH=False, want_dW=False))
    assert not any(n in names for n in ("gemm_dH", "gemm_dW", "split_sum", "gbuild"))
    fwd = L.loss_fwd(x["H"], x["W"], x["labels"])
    assert torch.equal(out["lse"], fwd["lse"]) and torch.equal(out["loss_rows"], fwd["loss_rows"])


@pytest.mark.parametrize("want", ["dH", "dW"])
@pytest.mark.parametrize("mode", [L.BWD_SUPPORT_LOGPROB, L.BWD_SUPPORT_KL])
def test_renormalised_support_backward_frozen(mode, want):
    # the other reading of the support set (log-probs normalised over each row's candidates):
    # its backward has no GEMM, dH is a gather of W rows and dW a scatter per vocabulary row,
    # so a frozen input skips the gather's output or the whole scatter
    N, d, V, K = 200, 128, 3000, 12
    x, xc = _inputs(N, d, V, 0, K=K)
    ids, ref_lp = x["ids"], x["ref_logp"]
    kl = mode == L.BWD_SUPPORT_KL
    lse = L.support_logprob(x["H"], x["W"], ids, renorm=True)["lse"]
    g = (torch.linspace(0.5, 1.5, N, dtype=torch.float32) / N if kl else
         torch.linspace(-1.0, 2.0, N * K, dtype=torch.float32).view(N, K) / N)
    args = (mode, x["H"], x["W"], ids, lse, g.cuda(), ref_lp if kl else None)
    both = L.loss_bwd(*args, renorm=True)
    only, names = launched(lambda: L.loss_bwd(*args, renorm=True, want_dH=want == "dH",
                                              want_dW=want == "dW"))
    ref = O.backward_renorm(mode, xc["H"], xc["W"], xc["ids"], g.numpy(),
                            xc["ref_logp"] if kl else None)
    other = "dW" if want == "dH" else "dH"
    assert only.get(other) is None
    check_grad(only[want], ref[want], f"{want} only (renormalised)")
    assert torch.equal(only[want], both[want])
    assert ("support_dw" in names) == (want == "dW"), names
