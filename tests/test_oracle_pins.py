"""Pins of the fp64 oracle to things other than itself (CPU only).

Each test checks the oracle against brute force on tiny inputs, a closed form, a
finite-difference derivative, an invariant or a library routine, chosen so that a dropped
term, a wrong sign or index, or a transposed operand in the oracle fails at least one.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import lmh_oracle as O
from tests.parity import ATOL_ROW, check_grad, check_rows, rejects

HERE = os.path.dirname(os.path.abspath(__file__))


def rand_problem(N, d, V, seed, scale=0.5):
    rng = np.random.default_rng(seed)
    H = rng.normal(size=(N, d))
    W = rng.normal(size=(V, d)) * scale
    return H, W


# ---------------------------------------------------------------- brute force (pure Python)

def bf_logits(H, W):
    return [[sum(H[i][j] * W[v][j] for j in range(len(H[i]))) for v in range(len(W))]
            for i in range(len(H))]


def bf_lse_row(zr):
    # no max shift: the brute force uses the textbook formula on small logits
    return math.log(sum(math.exp(t) for t in zr))


def bf_ce_mean(H, W, y):
    z = bf_logits(H, W)
    tot, cnt = 0.0, 0
    for i, zr in enumerate(z):
        if 0 <= y[i] < len(W):
            tot += bf_lse_row(zr) - zr[y[i]]
            cnt += 1
    return tot / cnt if cnt else 0.0


def test_brute_force_forward():
    H, W = rand_problem(4, 3, 6, 1)
    y = [5, -100, 0, 2]
    f = O.ce_forward(H, W, np.array(y))
    z = bf_logits(H.tolist(), W.tolist())
    for i in range(4):
        lse = bf_lse_row(z[i])
        assert abs(f["lse"][i] - lse) < 1e-12
        if y[i] >= 0:
            assert abs(f["loss_rows"][i] - (lse - z[i][y[i]])) < 1e-12
            assert abs(f["logprob"][i] - (z[i][y[i]] - lse)) < 1e-12
        else:
            assert f["loss_rows"][i] == 0.0 and f["logprob"][i] == 0.0
        best = max(range(6), key=lambda v: (z[i][v], -v))
        assert f["argmax"][i] == best
    assert f["n_valid"] == 3
    assert abs(f["loss_mean"] - bf_ce_mean(H.tolist(), W.tolist(), y)) < 1e-12


def test_brute_force_exact_rational_sum():
    # logits ln(1), ln(2), ln(3), ln(4) for one row -> softmax exactly (1,2,3,4)/10
    V = 4
    H = np.array([[1.0]])
    W = np.log(np.arange(1, V + 1, dtype=np.float64))[:, None]
    f = O.ce_fused(H, W, np.array([2]))
    assert abs(f["lse"][0] - math.log(10.0)) < 1e-14
    assert abs(f["loss_rows"][0] - (math.log(10.0) - math.log(3.0))) < 1e-14
    # G = P - e_y with P = k/10
    np.testing.assert_allclose(f["G"][0], [0.1, 0.2, 0.3 - 1.0, 0.4], atol=1e-15)


# ---------------------------------------------------------------- finite differences

def fd_grad(fun, X, h=1e-6):
    g = np.zeros_like(X)
    it = np.nditer(X, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        old = X[idx]
        X[idx] = old + h
        fp = fun()
        X[idx] = old - h
        fm = fun()
        X[idx] = old
        g[idx] = (fp - fm) / (2 * h)
    return g


def assert_fd(analytic, numeric, rtol=1e-6):
    scale = max(1.0, float(np.max(np.abs(numeric))))
    err = float(np.max(np.abs(analytic - numeric)))
    assert err <= rtol * scale * 10, (err, scale)


@pytest.mark.parametrize("mean", [True, False])
def test_fd_ce(mean):
    H, W = rand_problem(5, 4, 7, 2)
    y = np.array([0, 6, -100, 3, 3])
    f = O.ce_fused(H, W, y, mean=mean)

    def L():
        r = O.ce_forward(H, W, y)
        return r["loss_mean"] if mean else r["loss_rows"].sum()

    assert_fd(f["dH"], fd_grad(L, H))
    assert_fd(f["dW"], fd_grad(L, W))


def test_fd_logprob():
    H, W = rand_problem(4, 3, 5, 3)
    y = np.array([1, 4, -1, 0])
    g = np.array([0.3, -1.2, 5.0, 0.7])
    b = O.backward(O.BWD_LOGPROB, H, W, y, g)

    def L():
        return float((O.logprob_forward(H, W, y)["logprob"] * g).sum())

    assert_fd(b["dH"], fd_grad(L, H))
    assert_fd(b["dW"], fd_grad(L, W))


def test_fd_ce_rows_weighted():
    H, W = rand_problem(4, 3, 5, 4)
    y = np.array([1, 4, 2, 0])
    g = np.array([0.3, -1.2, 2.0, 0.7])
    b = O.backward(O.BWD_CE, H, W, y, g)

    def L():
        return float((O.ce_forward(H, W, y)["loss_rows"] * g).sum())

    assert_fd(b["dH"], fd_grad(L, H))
    assert_fd(b["dW"], fd_grad(L, W))


def test_fd_support_logprob():
    H, W = rand_problem(3, 4, 9, 5)
    ids = np.array([[0, 8, 3], [2, 2, -1], [7, 1, 5]])   # a repeated id and a padding id
    gam = np.array([[0.5, -0.25, 1.0], [1.5, 0.5, 9.0], [-1.0, 0.2, 0.3]])
    b = O.backward(O.BWD_SUPPORT_LOGPROB, H, W, ids, gam)

    def L():
        lp = O.support_logprob(H, W, ids)["lp"]
        return float((lp * gam * (ids >= 0)).sum())

    assert_fd(b["dH"], fd_grad(L, H))
    assert_fd(b["dW"], fd_grad(L, W))


def test_fd_support_kl():
    H, W = rand_problem(3, 4, 9, 6)
    ids = np.array([[0, 8, 3], [2, 4, 6], [7, 1, 5]])
    rng = np.random.default_rng(7)
    r = rng.normal(size=ids.shape)
    r = r - np.log(np.exp(r).sum(axis=1, keepdims=True))
    g = np.array([0.5, 1.0, -2.0])
    b = O.backward(O.BWD_SUPPORT_KL, H, W, ids, g, r)

    def L():
        return float((O.support_kl(H, W, ids, r)["kl_rows"] * g).sum())

    assert_fd(b["dH"], fd_grad(L, H))
    assert_fd(b["dW"], fd_grad(L, W))


# ---------------------------------------------------------------- closed forms

def test_zero_weight_closed_form():
    N, d, V = 6, 5, 11
    rng = np.random.default_rng(8)
    H = rng.normal(size=(N, d))
    W = np.zeros((V, d))
    y = np.array([3, 3, 10, -100, 0, 7])
    f = O.ce_fused(H, W, y)
    np.testing.assert_allclose(f["lse"], math.log(V), atol=1e-14)
    np.testing.assert_allclose(f["loss_rows"][y >= 0], math.log(V), atol=1e-14)
    assert abs(f["loss_mean"] - math.log(V)) < 1e-14
    np.testing.assert_allclose(f["dH"], 0.0, atol=1e-15)
    # dW_v = (1/V) sum_i g_i H_i - sum_{i: y_i = v} g_i H_i with g_i = 1/n_valid
    valid = y >= 0
    g = 1.0 / valid.sum()
    expect = np.tile(H[valid].sum(axis=0) * g / V, (V, 1))
    for i in np.nonzero(valid)[0]:
        expect[y[i]] -= g * H[i]
    np.testing.assert_allclose(f["dW"], expect, atol=1e-14)


def test_logistic_d1_v2():
    # d = 1, V = 2: cross-entropy is the logistic loss softplus(z_other - z_label)
    H = np.array([[0.7], [-1.3], [2.0]])
    W = np.array([[0.4], [-0.9]])
    y = np.array([0, 1, 1])
    f = O.ce_forward(H, W, y)
    for i in range(3):
        z0, z1 = H[i, 0] * W[0, 0], H[i, 0] * W[1, 0]
        margin = (z0 - z1) if y[i] == 0 else (z1 - z0)
        assert abs(f["loss_rows"][i] - math.log1p(math.exp(-margin))) < 1e-14


def test_logprob_normalises_over_vocab():
    H, W = rand_problem(3, 4, 13, 9)
    tot = np.zeros(3)
    for v in range(13):
        tot += np.exp(O.logprob_forward(H, W, np.full(3, v))["logprob"])
    np.testing.assert_allclose(tot, 1.0, atol=1e-13)


def test_kl_zero_for_identical_and_nonnegative():
    N, d, V = 4, 3, 7
    H, W = rand_problem(N, d, V, 10)
    rng = np.random.default_rng(11)
    ids = np.stack([rng.permutation(V) for _ in range(N)])
    lp = O.support_logprob(H, W, ids)["lp"]
    kl = O.support_kl(H, W, ids, lp)["kl_rows"]
    np.testing.assert_allclose(kl, 0.0, atol=1e-14)
    # K < V and an arbitrary normalised reference: Gibbs' inequality gives KL >= 0
    for s in range(20):
        ids3 = np.stack([rng.choice(V, size=3, replace=False) for _ in range(N)])
        r = rng.normal(size=(N, 3)) * 2
        r -= np.log(np.exp(r).sum(axis=1, keepdims=True))
        assert np.all(O.support_kl(H, W, ids3, r)["kl_rows"] >= -1e-14)


def test_shift_invariance():
    N, d, V = 5, 4, 9
    H, W = rand_problem(N, d, V, 12)
    y = np.array([1, 2, 8, -100, 0])
    a = np.random.default_rng(13).normal(size=(N, 1)) * 3
    H2 = np.hstack([H, a])
    W2 = np.hstack([W, np.ones((V, 1))])      # every logit of row i moves by a_i
    f1, f2 = O.ce_fused(H, W, y), O.ce_fused(H2, W2, y)
    np.testing.assert_allclose(f2["loss_rows"], f1["loss_rows"], atol=1e-13)
    np.testing.assert_allclose(f2["G"], f1["G"], atol=1e-15)
    np.testing.assert_allclose(f2["dH"][:, :d], f1["dH"], atol=1e-13)
    np.testing.assert_allclose(f2["dW"][:, :d], f1["dW"], atol=1e-13)
    np.testing.assert_allclose(f2["lse"] - f1["lse"], a[:, 0], atol=1e-12)


def test_masked_rows_contribute_nothing():
    N, d, V = 8, 4, 10
    H, W = rand_problem(N, d, V, 14)
    y = np.array([1, -100, 3, -7, 9, 0, -100, 4])
    keep = y >= 0
    f = O.ce_fused(H, W, y)
    s = O.ce_fused(H[keep], W, y[keep])
    np.testing.assert_allclose(f["loss_rows"][keep], s["loss_rows"], atol=1e-14)
    assert np.all(f["loss_rows"][~keep] == 0) and np.all(f["dH"][~keep] == 0)
    assert abs(f["loss_mean"] - s["loss_mean"]) < 1e-14
    np.testing.assert_allclose(f["dW"], s["dW"], atol=1e-14)
    np.testing.assert_allclose(f["dH"][keep], s["dH"], atol=1e-14)


def test_label_out_of_range_is_ignored_and_flagged():
    H, W = rand_problem(3, 2, 4, 15)
    f = O.ce_fused(H, W, np.array([4, 1, 2]))
    assert f["label_out_of_range"] and f["n_valid"] == 2 and f["loss_rows"][0] == 0.0
    assert np.all(f["dH"][0] == 0)


def test_no_valid_rows():
    H, W = rand_problem(3, 2, 4, 16)
    f = O.ce_fused(H, W, np.array([-100, -1, -100]))
    assert f["n_valid"] == 0 and f["loss_mean"] == 0.0
    assert np.all(f["dH"] == 0) and np.all(f["dW"] == 0)


def test_argmax_takes_first_of_equal_maxima():
    H = np.array([[1.0], [1.0]])
    W = np.array([[0.5], [2.0], [2.0], [-1.0]])
    assert list(O.ce_forward(H, W, np.array([0, 0]))["argmax"]) == [1, 1]


def test_transposition_pins():
    # a non-square problem where G W and G^T H have distinct shapes and entries
    H, W = rand_problem(2, 3, 5, 17)
    f = O.ce_fused(H, W, np.array([4, 1]), mean=False)
    assert f["dH"].shape == (2, 3) and f["dW"].shape == (5, 3)
    # dH_i = sum_v G_iv W_v, spelt out
    for i in range(2):
        exp = sum(f["G"][i, v] * W[v] for v in range(5))
        np.testing.assert_allclose(f["dH"][i], exp, atol=1e-14)
    for v in range(5):
        exp = sum(f["G"][i, v] * H[i] for i in range(2))
        np.testing.assert_allclose(f["dW"][v], exp, atol=1e-14)


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(18)
    x = np.concatenate([rng.normal(size=4000) * 10.0 ** rng.integers(-30, 30, 4000),
                        [0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 65504.0, 3.4e38]])
    want = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(O.bf16_round(x), want)


def test_chunk_plan():
    assert O.chunk_plan(10, 4) == [(0, 4), (4, 8), (8, 10)]
    assert O.chunk_plan(8192, 0) == [(0, 4096), (4096, 8192)]
    assert O.chunk_plan(0, 4) == []
    for N, c in [(1, 1), (100, 7), (16384, 2048)]:
        p = O.chunk_plan(N, c)
        assert p[0][0] == 0 and p[-1][1] == N
        assert all(a[1] == b[0] for a, b in zip(p, p[1:]))


# ---------------------------------------------------------------- golden fixtures

def test_hand_worked_example():
    with open(os.path.join(HERE, "golden", "hand_example.json")) as fh:
        g = json.load(fh)
    f = O.ce_fused(np.array(g["H"]), np.array(g["W"]), np.array(g["labels"]))
    np.testing.assert_allclose(f["lse"], g["lse"], atol=1e-15)
    np.testing.assert_allclose(f["loss_rows"], g["loss_rows"], atol=1e-15)
    assert abs(f["loss_mean"] - g["loss_mean"]) < 1e-15
    np.testing.assert_allclose(f["dH"], g["dH"], atol=1e-15)
    np.testing.assert_allclose(f["dW"], g["dW"], atol=1e-15)


def test_tiny_workload_summary_reproduces():
    """The oracle still gives the stored summary of the 64 x 256 x 2048 workload."""
    from workloads import WORKLOADS, make_inputs
    with open(os.path.join(HERE, "golden", "tiny_oracle_summary.json")) as fh:
        g = json.load(fh)
    x = make_inputs(WORKLOADS["tiny"])
    f = O.ce_fused(x["H"], x["W"], x["labels"])
    np.testing.assert_allclose(f["loss_rows"], g["loss_rows"], atol=1e-12)
    np.testing.assert_allclose(f["lse"], g["lse"], atol=1e-12)
    assert f["n_valid"] == g["n_valid"]
    np.testing.assert_allclose(np.linalg.norm(f["dH"]), g["dH_norm"], rtol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(f["dW"]), g["dW_norm"], rtol=1e-12)
    np.testing.assert_allclose(f["dW"][:4, :4], g["dW_corner"], atol=1e-14)


# ---------------------------------------------------------------- the gates themselves

def test_gates_reject_two_percent_scale():
    H, W = rand_problem(16, 8, 40, 19)
    y = np.arange(16) % 40
    f = O.ce_fused(H, W, y)
    noise = np.random.default_rng(20)
    dW = f["dW"] * (1 + 1e-3 * noise.normal(size=f["dW"].shape))
    check_grad(dW, f["dW"])                        # realistic rounding noise passes
    assert rejects(check_grad, f["dW"] * 1.02, f["dW"])
    assert rejects(check_grad, f["dH"] * 1.02, f["dH"])
    assert rejects(check_rows, f["loss_rows"] * 1.02, f["loss_rows"])
    assert rejects(check_grad, f["dW"].T.copy().T[::-1], f["dW"])
    check_rows(f["lse"] + 0.5 * ATOL_ROW, f["lse"])


# ---------------------------------------------------------------- temperature

def test_fd_with_temperature_scalar_and_rows():
    H, W = rand_problem(4, 3, 6, 21)
    y = np.array([0, 5, -100, 2])
    for tau in (0.7, np.array([0.5, 1.0, 2.0, 1.3])):
        f = O.ce_fused(H, W, y, mean=True, tau=tau)

        def L():
            return O.ce_forward(H, W, y, tau)["loss_mean"]

        assert_fd(f["dH"], fd_grad(L, H))
        assert_fd(f["dW"], fd_grad(L, W))
    ids = np.array([[0, 5, 3], [2, 2, -1], [1, 4, 0], [5, 3, 1]])
    r = np.log(np.full((4, 3), 1.0 / 3.0))
    tau = np.array([0.8, 1.5, 1.0, 0.6])
    b = O.backward(O.BWD_SUPPORT_KL, H, W, ids, np.ones(4), r, tau=tau)

    def Lk():
        return float(O.support_kl(H, W, ids, r, tau)["kl_rows"].sum())

    assert_fd(b["dH"], fd_grad(Lk, H))
    assert_fd(b["dW"], fd_grad(Lk, W))


def test_scalar_temperature_equals_scaled_weights():
    H, W = rand_problem(5, 4, 9, 22)
    y = np.array([1, 8, 0, -100, 3])
    tau = 0.37
    a = O.ce_fused(H, W, y, tau=tau)
    b = O.ce_fused(H, W / tau, y)
    np.testing.assert_allclose(a["loss_rows"], b["loss_rows"], atol=1e-13)
    np.testing.assert_allclose(a["lse"], b["lse"], atol=1e-13)
    np.testing.assert_allclose(a["dH"], b["dH"], atol=1e-13)
    # d/dW of L(H (W/tau)^T) = (1/tau) dL/dW' at W' = W / tau
    np.testing.assert_allclose(a["dW"], b["dW"] / tau, atol=1e-13)


def test_temperature_one_is_off():
    H, W = rand_problem(3, 4, 7, 23)
    y = np.array([1, 2, 6])
    a, b = O.ce_fused(H, W, y), O.ce_fused(H, W, y, tau=np.ones(3))
    np.testing.assert_array_equal(a["dW"], b["dW"])
    np.testing.assert_array_equal(a["loss_rows"], b["loss_rows"])


# ---------------------------------------------------------------- renormalised support set

def test_renorm_support_normalises_and_kl_identities():
    H, W = rand_problem(3, 4, 10, 31)
    ids = np.array([[1, 7, 3, 7], [0, 9, -1, 4], [2, 5, 6, 8]])   # a repeat and a padding slot
    s = O.support_renorm_logprob(H, W, ids)
    for i in range(3):
        S = sorted({v for v in ids[i] if v >= 0})
        tot = sum(np.exp(s["lp"][i, list(ids[i]).index(v)]) for v in S)
        assert abs(tot - 1.0) < 1e-13
    # against a brute-force softmax over the support, row 2
    z = O.logits(H, W)[2, [2, 5, 6, 8]]
    np.testing.assert_allclose(s["lp"][2], z - np.log(np.exp(z).sum()), atol=1e-13)
    # KL = 0 against the model's own renormalised log-probs (distinct ids), >= 0 otherwise
    ids_u = np.array([[1, 7, 3], [0, 9, 4], [2, 5, 6]])
    lp = O.support_renorm_logprob(H, W, ids_u)["lp"]
    np.testing.assert_allclose(O.support_renorm_kl(H, W, ids_u, lp)["kl_rows"], 0.0, atol=1e-14)
    rng = np.random.default_rng(32)
    r = rng.normal(size=ids_u.shape)
    r -= np.log(np.exp(r).sum(axis=1, keepdims=True))
    assert np.all(O.support_renorm_kl(H, W, ids_u, r)["kl_rows"] >= -1e-14)


@pytest.mark.parametrize("tau", [None, np.array([0.6, 1.4, 1.0])])
def test_fd_renorm_support(tau):
    H, W = rand_problem(3, 4, 10, 33)
    ids = np.array([[1, 7, 3, 7], [0, 9, -1, 4], [2, 5, 6, 8]])
    gam = np.random.default_rng(34).normal(size=ids.shape)
    b = O.backward_renorm(O.BWD_SUPPORT_LOGPROB, H, W, ids, gam, tau=tau)

    def L():
        lp = O.support_renorm_logprob(H, W, ids, tau)["lp"]
        return float((lp * gam * (ids >= 0)).sum())

    assert_fd(b["dH"], fd_grad(L, H))
    assert_fd(b["dW"], fd_grad(L, W))
    r = np.log(np.full(ids.shape, 0.25))
    g = np.array([1.0, -0.5, 2.0])
    b = O.backward_renorm(O.BWD_SUPPORT_KL, H, W, ids, g, r, tau=tau)

    def Lk():
        return float((O.support_renorm_kl(H, W, ids, r, tau)["kl_rows"] * g).sum())

    assert_fd(b["dH"], fd_grad(Lk, H))
    assert_fd(b["dW"], fd_grad(Lk, W))
