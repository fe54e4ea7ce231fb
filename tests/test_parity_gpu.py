"""GPU parity of every entry against the fp64 oracle, element by element, at sizes that span
several tiles with ragged row, vocabulary and hidden tails. Calls go through the C ABI."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import lm_head_cross_tcgen05_b200 as L
from tests.gpu_common import O, check_argmax, check_ce_fused, check_grad, check_rows, device_inputs, digest
from tests.parity import rejects
from workloads import WORKLOADS, ragged

pytestmark = pytest.mark.gpu

# (N, d, V, ignored rows): tiles of 128 rows x 256 words, K blocks of 64
SHAPES = [
    (64, 256, 2048, 8),     # the tiny workload's shape
    (300, 192, 1000, 5),    # ragged rows (128+128+44), d not a multiple of 256, V tail of 232
    (129, 64, 257, 3),      # one K block, V one past a tile, padded row stride
    (200, 512, 4100, 20),   # V = 4100: row stride 4104, 17 vocabulary tiles
    (1, 128, 300, 0),       # a single row
    (130, 128, 100, 0),     # V smaller than one tile
]


def _wl(N, d, V, ign, **kw):
    return ragged(N, d, V, n_ignored=ign, seed=1000 + N + d + V, **kw)


@pytest.mark.parametrize("N,d,V,ign", SHAPES)
@pytest.mark.parametrize("chunk", [0, 128, 100])
def test_fused_ce(N, d, V, ign, chunk):
    x, xc = device_inputs(_wl(N, d, V, ign))
    out = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=chunk, grads=True)
    torch.cuda.synchronize()
    assert L.lmh_read_errors(out["workspace"]) == 0
    ref = O.ce_fused(xc["H"], xc["W"], xc["labels"])
    check_ce_fused(out, ref)


def test_tiny_workload_and_gates_reject_scaled_output():
    x, xc = device_inputs(WORKLOADS["tiny"])
    out = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True)
    ref = O.ce_fused(xc["H"], xc["W"], xc["labels"])
    check_ce_fused(out, ref)
    assert int(out["n_valid"].item()) == 56
    # the gates fail an output 2 % off
    assert rejects(check_grad, out["dW"].float() * 1.02, ref["dW"])
    assert rejects(check_grad, out["dH"].float() * 1.02, ref["dH"])
    assert rejects(check_rows, out["loss_rows"] * 1.02, ref["loss_rows"])


@pytest.mark.parametrize("N,d,V,ign", SHAPES[:4])
def test_forward_only_matches_fused_bits(N, d, V, ign):
    x, _ = device_inputs(_wl(N, d, V, ign))
    a = L.loss_fwd(x["H"], x["W"], x["labels"], grads=False)
    b = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True)
    for k in ("loss_rows", "lse", "logprob", "argmax", "loss_mean", "n_valid"):
        assert torch.equal(a[k], b[k]), k


@pytest.mark.parametrize("N,d,V,ign", SHAPES[:4])
def test_logprob_entry(N, d, V, ign):
    x, xc = device_inputs(_wl(N, d, V, ign))
    out = L.logprob(x["H"], x["W"], x["labels"], chunk_rows=100)
    ref = O.logprob_forward(xc["H"], xc["W"], xc["labels"])
    check_rows(out["logprob"], ref["logprob"], what="logprob")
    check_rows(out["lse"], ref["lse"], what="lse")


def _support_inputs(N, d, V, K, seed):
    wl = ragged(N, d, V, K=K, seed=seed)
    x, xc = device_inputs(wl)
    ids = xc["ids"].clone()
    if K >= 4:
        # a repeated id and padding slots exercise de-duplication and skipping
        ids[0, 1] = ids[0, 0]
        ids[1, -1] = -1
        ids[2, 3] = -7
    x["ids"] = ids.cuda()
    xc["ids"] = ids
    return x, xc


@pytest.mark.parametrize("N,d,V,K", [(200, 128, 3000, 16), (130, 64, 700, 64), (64, 256, 2048, 1)])
def test_support_logprob_and_kl(N, d, V, K):
    x, xc = _support_inputs(N, d, V, K, 77 + K)
    ref = O.support_kl(xc["H"], xc["W"], xc["ids"], xc["ref_logp"])
    a = L.support_logprob(x["H"], x["W"], x["ids"], chunk_rows=128)
    check_rows(a["lp"], ref["lp"], what="lp")
    check_rows(a["lse"], ref["lse"], what="lse")
    b = L.support_kl(x["H"], x["W"], x["ids"], x["ref_logp"], chunk_rows=0)
    check_rows(b["kl_rows"], ref["kl_rows"], what="kl_rows")
    check_rows(b["kl_mean"], np.array([ref["kl_mean"]]), what="kl_mean")
    check_rows(b["lp"], ref["lp"], what="lp(kl)")
    assert torch.equal(a["lp"], b["lp"])


@pytest.mark.parametrize("mode", [L.BWD_CE, L.BWD_LOGPROB, L.BWD_SUPPORT_LOGPROB, L.BWD_SUPPORT_KL])
@pytest.mark.parametrize("chunk", [0, 96])
def test_loss_bwd_modes(mode, chunk):
    N, d, V, K = 260, 192, 1500, 12
    x, xc = _support_inputs(N, d, V, K, 300 + mode)
    g = torch.Generator().manual_seed(5 + mode)
    if mode in (L.BWD_CE, L.BWD_LOGPROB):
        targets, tc = x["labels"], xc["labels"]
        grad = torch.randn(N, generator=g) / N
        lse = L.logprob(x["H"], x["W"], x["labels"])["lse"]
    else:
        targets, tc = x["ids"], xc["ids"]
        grad = (torch.randn(N, K, generator=g) / N) if mode == L.BWD_SUPPORT_LOGPROB else (
            torch.rand(N, generator=g) / N)
        lse = L.support_logprob(x["H"], x["W"], x["ids"])["lse"]
    ref_lp = x["ref_logp"] if mode == L.BWD_SUPPORT_KL else None
    out = L.loss_bwd(mode, x["H"], x["W"], targets, lse, grad.cuda(), ref_lp, chunk_rows=chunk)
    ref = O.backward(mode, xc["H"], xc["W"], tc, grad,
                     xc["ref_logp"] if mode == L.BWD_SUPPORT_KL else None)
    check_grad(out["dH"], ref["dH"], "dH")
    check_grad(out["dW"], ref["dW"], "dW")


def test_fused_equals_standalone_backward_within_tolerance():
    x, xc = device_inputs(_wl(300, 192, 1000, 5))
    f = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True)
    n = int(f["n_valid"].item())
    grad = torch.full((300,), 1.0 / n, device="cuda")
    b = L.loss_bwd(L.BWD_CE, x["H"], x["W"], x["labels"], f["lse"], grad)
    check_grad(b["dH"], f["dH"].float().cpu().double().numpy(), "dH")
    check_grad(b["dW"], f["dW"].float().cpu().double().numpy(), "dW")


def test_determinism_ten_runs():
    x, _ = device_inputs(_wl(520, 256, 5000, 9))
    ref = None
    for _ in range(10):
        o = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=200, grads=True)
        h = digest(o["loss_rows"], o["lse"], o["logprob"], o["argmax"], o["loss_mean"], o["dH"],
                   o["dW"])
        ref = ref or h
        assert h == ref


def test_chunk_plan_changes_only_dW_bits():
    x, xc = device_inputs(_wl(300, 128, 1000, 4))
    base = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True)
    ref = O.ce_fused(xc["H"], xc["W"], xc["labels"])
    for c in (128, 100, 37, 1):
        o = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=c, grads=True)
        for k in ("loss_rows", "lse", "logprob", "argmax", "dH"):
            assert torch.equal(o[k], base[k]), (c, k)
        check_grad(o["dW"], ref["dW"], f"dW chunk {c}")


def test_dW_is_bf16_cast_of_fp32_accumulator():
    x, xc = device_inputs(_wl(300, 128, 1000, 4))
    acc = torch.zeros(1000, 128, dtype=torch.float32, device="cuda")
    o = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=128, grads=True, dW_acc=acc)
    assert torch.equal(o["dW"], acc.to(torch.bfloat16))
    ref = O.ce_fused(xc["H"], xc["W"], xc["labels"])
    check_grad(acc, ref["dW"], "dW_acc")
    # a second call accumulates on top, in the same fixed order
    acc2 = acc.clone()
    o2 = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=128, grads=True, dW_acc=acc2)
    check_grad(acc2, 2 * ref["dW"], "dW_acc twice")
    assert torch.equal(o2["dW"], acc2.to(torch.bfloat16))
    # internal accumulator (no dW_acc given) gives the same bits as a zeroed external one
    o3 = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=128, grads=True)
    assert torch.equal(o3["dW"], o["dW"])


@pytest.mark.parametrize("chunk", [0, 16])
def test_dW_accumulate_is_ieee_add(chunk):
    # H = 0 makes every dW contribution zero, so the accumulator must come back unchanged:
    # subnormal values are neither flushed by the add nor by the cast's input
    x, _ = device_inputs(_wl(64, 128, 700, 0))
    H = torch.zeros_like(x["H"])
    acc = torch.full((700, 128), 1e-39, dtype=torch.float32, device="cuda")
    acc[::2] = -3.5e-40
    acc[1::7] = 1.25
    before = acc.clone()
    o = L.loss_fwd(H, x["W"], x["labels"], chunk_rows=chunk, grads=True, dW_acc=acc)
    assert torch.equal(acc, before)
    assert torch.equal(o["dW"], before.to(torch.bfloat16))
    assert torch.count_nonzero(o["dH"]) > 0  # dH = G W does not vanish


def test_no_valid_rows_and_empty_call():
    x, xc = device_inputs(_wl(140, 64, 500, 0))
    y = torch.full_like(x["labels"], -100)
    y[3] = -1
    o = L.loss_fwd(x["H"], x["W"], y, grads=True)
    assert int(o["n_valid"].item()) == 0 and float(o["loss_mean"].item()) == 0.0
    assert torch.count_nonzero(o["dH"]) == 0 and torch.count_nonzero(o["dW"]) == 0
    assert torch.count_nonzero(o["loss_rows"]) == 0
    ref = O.ce_forward(xc["H"], xc["W"], y.cpu())
    check_rows(o["lse"], ref["lse"], what="lse")
    e = L.loss_fwd(x["H"][:0], x["W"], y[:0], grads=True)
    assert int(e["n_valid"].item()) == 0 and torch.count_nonzero(e["dW"]) == 0


def test_label_out_of_range_sets_error_word():
    x, xc = device_inputs(_wl(100, 64, 300, 0))
    y = x["labels"].clone()
    y[7] = 300
    y[9] = 10 ** 6
    o = L.loss_fwd(x["H"], x["W"], y, grads=True)
    assert L.lmh_read_errors(o["workspace"]) & L.DEVERR_LABEL_RANGE
    ref = O.ce_fused(xc["H"], xc["W"], y.cpu())
    check_ce_fused(o, ref)
    ok = L.loss_fwd(x["H"], x["W"], x["labels"], ws=o["workspace"])
    assert L.lmh_read_errors(ok["workspace"]) == 0


def test_side_stream_same_bits():
    x, _ = device_inputs(_wl(300, 192, 1000, 5))
    a = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        b = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True, stream=s)
    s.synchronize()
    assert digest(a["dW"], a["dH"], a["lse"]) == digest(b["dW"], b["dH"], b["lse"])


def test_host_rejections():
    x, _ = device_inputs(_wl(64, 64, 300, 0))
    shape = L.make_shape(64, 64, 300)
    ws = L.workspace(shape, L.ENTRY_LOSS_FWD, "cuda")
    lr, lse = torch.empty(64, device="cuda"), torch.empty(64, device="cuda")
    with pytest.raises(L.LmhError, match="WORKSPACE_TOO_SMALL"):
        L.lmh_loss_fwd(shape, x["H"], x["W"], x["labels"], lr, lse, workspace=ws[:100])
    bad = L.make_shape(64, 96, 300)     # d not a multiple of 64: refused by the library
    H96 = torch.zeros(64, 96, dtype=torch.bfloat16, device="cuda")
    W96 = torch.zeros(300, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.LmhError, match="INVALID_ARG"):
        L.lmh_loss_fwd(bad, H96, W96, x["labels"], lr, lse, workspace=ws)
    with pytest.raises(ValueError, match="W has"):  # too small for the shape: the binding
        L.lmh_loss_fwd(shape, x["H"], x["W"][:200], x["labels"], lr, lse, workspace=ws)
    with pytest.raises(L.LmhError, match="ALIGNMENT"):
        L.lmh_loss_fwd(shape, x["H"], x["W"], x["labels"], lr, lse, workspace=ws[8:])


def _temps(kind, N, seed=3):
    if kind == "scalar":
        return 0.7, 0.7
    if kind == "rows":
        g = torch.Generator().manual_seed(seed)
        t = torch.rand(N, generator=g, dtype=torch.float32) * 1.5 + 0.5
        return t.cuda(), t.double().numpy()
    return 1.0, None


@pytest.mark.parametrize("kind", ["scalar", "rows", "one"])
def test_temperature_ce_logprob_and_backward(kind):
    N, d, V = 300, 192, 1000
    x, xc = device_inputs(_wl(N, d, V, 5))
    t_dev, t_ref = _temps(kind, N)
    out = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=128, grads=True, temperature=t_dev)
    ref = O.ce_fused(xc["H"], xc["W"], xc["labels"], tau=t_ref)
    check_ce_fused(out, ref)
    lp = L.logprob(x["H"], x["W"], x["labels"], temperature=t_dev)
    check_rows(lp["logprob"], ref["logprob"], what="logprob")
    n = int(out["n_valid"].item())
    grad = torch.full((N,), 1.0 / n, device="cuda")
    b = L.loss_bwd(L.BWD_CE, x["H"], x["W"], x["labels"], out["lse"], grad, chunk_rows=100,
                   temperature=t_dev)
    check_grad(b["dH"], ref["dH"], "dH (recompute, tempered)")
    check_grad(b["dW"], ref["dW"], "dW (recompute, tempered)")
    if kind == "one":
        plain = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=128, grads=True)
        assert digest(plain["dW"], plain["dH"], plain["lse"]) == digest(out["dW"], out["dH"], out["lse"])


@pytest.mark.parametrize("kind", ["scalar", "rows"])
def test_temperature_support_kl(kind):
    N, d, V, K = 200, 128, 3000, 16
    x, xc = _support_inputs(N, d, V, K, 91)
    t_dev, t_ref = _temps(kind, N, seed=8)
    kl = L.support_kl(x["H"], x["W"], x["ids"], x["ref_logp"], temperature=t_dev)
    ref = O.support_kl(xc["H"], xc["W"], xc["ids"], xc["ref_logp"], tau=t_ref)
    check_rows(kl["kl_rows"], ref["kl_rows"], what="kl_rows")
    check_rows(kl["lp"], ref["lp"], what="lp")
    grad = torch.full((N,), 1.0 / N, device="cuda")
    b = L.loss_bwd(L.BWD_SUPPORT_KL, x["H"], x["W"], x["ids"], kl["lse"], grad, x["ref_logp"],
                   temperature=t_dev)
    rb = O.backward(O.BWD_SUPPORT_KL, xc["H"], xc["W"], xc["ids"], np.full(N, 1.0 / N),
                    xc["ref_logp"], tau=t_ref)
    check_grad(b["dH"], rb["dH"], "dH")
    check_grad(b["dW"], rb["dW"], "dW")


def test_invalid_row_temperature_is_flagged_and_used_as_one():
    N = 130
    x, xc = device_inputs(_wl(N, 64, 300, 0))
    t = torch.ones(N, device="cuda")
    t[5] = 0.0
    t[9] = float("nan")
    out = L.loss_fwd(x["H"], x["W"], x["labels"], temperature=t)
    assert L.lmh_read_errors(out["workspace"]) & L.DEVERR_TEMPERATURE
    ref = O.ce_forward(xc["H"], xc["W"], xc["labels"])
    check_rows(out["loss_rows"], ref["loss_rows"], what="loss_rows")


def test_backward_without_grad_uses_device_count():
    N, d, V = 300, 192, 1000
    x, xc = device_inputs(_wl(N, d, V, 5))
    f = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True)
    n = int(f["n_valid"].item())
    explicit = L.loss_bwd(L.BWD_CE, x["H"], x["W"], x["labels"], f["lse"],
                          torch.full((N,), 1.0 / n, device="cuda"))
    implicit = L.loss_bwd(L.BWD_CE, x["H"], x["W"], x["labels"], f["lse"], None, mean=True)
    assert torch.equal(explicit["dW"], implicit["dW"]) and torch.equal(explicit["dH"], implicit["dH"])
    ref = O.ce_fused(xc["H"], xc["W"], xc["labels"])
    check_grad(implicit["dW"], ref["dW"], "dW mean, no grad")
    # the sum objective: unit weights
    s = L.loss_bwd(L.BWD_CE, x["H"], x["W"], x["labels"], f["lse"], None, mean=False)
    rs = O.ce_fused(xc["H"], xc["W"], xc["labels"], mean=False)
    check_grad(s["dH"], rs["dH"], "dH sum, no grad")
    # support KL, mean over N rows
    xs, xsc = _support_inputs(N, d, V, 8, 55)
    kl = L.support_kl(xs["H"], xs["W"], xs["ids"], xs["ref_logp"])
    a = L.loss_bwd(L.BWD_SUPPORT_KL, xs["H"], xs["W"], xs["ids"], kl["lse"],
                   torch.full((N,), 1.0 / N, device="cuda"), xs["ref_logp"])
    b = L.loss_bwd(L.BWD_SUPPORT_KL, xs["H"], xs["W"], xs["ids"], kl["lse"], None, xs["ref_logp"],
                   mean=True)
    assert torch.equal(a["dW"], b["dW"]) and torch.equal(a["dH"], b["dH"])


@pytest.mark.parametrize("tau_kind", ["off", "rows"])
def test_renorm_support_forward_and_backward(tau_kind):
    N, d, V, K = 260, 192, 3000, 16
    x, xc = _support_inputs(N, d, V, K, 123)
    t_dev, t_ref = (None, None) if tau_kind == "off" else _temps("rows", N, seed=12)
    lp = L.support_logprob(x["H"], x["W"], x["ids"], renorm=True, temperature=t_dev)
    kl = L.support_kl(x["H"], x["W"], x["ids"], x["ref_logp"], renorm=True, temperature=t_dev)
    ref = O.support_renorm_kl(xc["H"], xc["W"], xc["ids"], xc["ref_logp"], tau=t_ref)
    check_rows(lp["lp"], ref["lp"], what="lp renorm")
    check_rows(lp["lse"], ref["lse"], what="lse over the support")
    check_rows(kl["kl_rows"], ref["kl_rows"], what="kl renorm")
    assert torch.equal(kl["lp"], lp["lp"])
    g = torch.Generator().manual_seed(4)
    gam = torch.randn(N, K, generator=g) / N
    b = L.loss_bwd(L.BWD_SUPPORT_LOGPROB, x["H"], x["W"], x["ids"], lp["lse"], gam.cuda(),
                   renorm=True, temperature=t_dev)
    rb = O.backward_renorm(O.BWD_SUPPORT_LOGPROB, xc["H"], xc["W"], xc["ids"], gam, tau=t_ref)
    check_grad(b["dH"], rb["dH"], "dH renorm logprob")
    check_grad(b["dW"], rb["dW"], "dW renorm logprob")
    acc = torch.zeros(V, d, device="cuda")
    bk = L.loss_bwd(L.BWD_SUPPORT_KL, x["H"], x["W"], x["ids"], kl["lse"], None, x["ref_logp"],
                    mean=True, renorm=True, temperature=t_dev, dW_acc=acc)
    rk = O.backward_renorm(O.BWD_SUPPORT_KL, xc["H"], xc["W"], xc["ids"], np.full(N, 1.0 / N),
                           xc["ref_logp"], tau=t_ref)
    check_grad(bk["dH"], rk["dH"], "dH renorm KL")
    check_grad(acc, rk["dW"], "dW_acc renorm KL")
    assert torch.equal(bk["dW"], acc.to(torch.bfloat16))
    # bitwise repeats (the scatter is summed in a fixed row order)
    b2 = L.loss_bwd(L.BWD_SUPPORT_LOGPROB, x["H"], x["W"], x["ids"], lp["lse"], gam.cuda(),
                    renorm=True, temperature=t_dev)
    assert torch.equal(b2["dW"], b["dW"]) and torch.equal(b2["dH"], b["dH"])


def test_single_word_vocabulary():
    # V = 1: every valid row has loss 0, lse = its only logit, and zero gradients
    N, d = 50, 64
    x, xc = device_inputs(_wl(N, d, 1, 0))
    y = torch.zeros(N, dtype=torch.int32, device="cuda")
    y[3] = -100
    out = L.loss_fwd(x["H"], x["W"], y, grads=True, chunk_rows=16)
    ref = O.ce_fused(xc["H"], xc["W"], y.cpu())
    check_ce_fused(out, ref)
    assert torch.count_nonzero(out["argmax"]) == 0
    assert torch.count_nonzero(out["dW"]) == 0 and torch.count_nonzero(out["dH"]) == 0


def test_maximum_candidate_count():
    N, d, V, K = 40, 64, 5000, L.MAX_K
    x, xc = _support_inputs(N, d, V, K, 31)
    kl = L.support_kl(x["H"], x["W"], x["ids"], x["ref_logp"])
    ref = O.support_kl(xc["H"], xc["W"], xc["ids"], xc["ref_logp"])
    check_rows(kl["kl_rows"], ref["kl_rows"], what="kl_rows K=1024")
    check_rows(kl["lp"], ref["lp"], what="lp K=1024")
    b = L.loss_bwd(L.BWD_SUPPORT_KL, x["H"], x["W"], x["ids"], kl["lse"], None, x["ref_logp"],
                   mean=True)
    rb = O.backward(O.BWD_SUPPORT_KL, xc["H"], xc["W"], xc["ids"], np.full(N, 1.0 / N),
                    xc["ref_logp"])
    check_grad(b["dW"], rb["dW"], "dW K=1024")
    r = L.support_logprob(x["H"], x["W"], x["ids"], renorm=True)
    rr = O.support_renorm_logprob(xc["H"], xc["W"], xc["ids"])
    check_rows(r["lp"], rr["lp"], what="renorm lp K=1024")
    with pytest.raises((ValueError, L.LmhError)):
        ids = torch.zeros(N, K + 1, dtype=torch.int32, device="cuda")
        L.support_logprob(x["H"], x["W"], ids)


def _kernels_launched(fn):
    """Names of the library kernels that fn() launched (the library's own launch record)."""
    import ctypes
    from lm_head_cross_tcgen05_b200._abi import lib
    lib().lmh_profile_read(0, None, None)  # drop any earlier records
    lib().lmh_profile_enable(1)
    try:
        fn()
        torch.cuda.synchronize()
    finally:
        lib().lmh_profile_enable(0)
    cap = 4096
    kid, ms = (ctypes.c_int32 * cap)(), (ctypes.c_float * cap)()
    n = lib().lmh_profile_read(cap, kid, ms)
    return [lib().lmh_kernel_name(kid[i]).decode() for i in range(n)]


@pytest.mark.parametrize("N,d,V,ign,splits", [
    (300, 320, 70000, 5, 2),     # 4 dH tiles: V split in 2 ranges, the last K block ragged
    (130, 128, 132072, 0, 4),    # 1 dH tile: V split in 4 ranges
])
def test_dh_split_over_vocabulary(N, d, V, ign, splits):
    # chunks with few dH tiles and a large V sum dH over vocabulary ranges in a fixed order
    x, xc = device_inputs(_wl(N, d, V, ign))
    res = {}

    def run():
        res["o"] = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True)
    names = _kernels_launched(run)
    assert names.count("split_sum") == 1 and names.count("gemm_dH") == 1
    out = res["o"]
    assert L.lmh_read_errors(out["workspace"]) == 0
    check_ce_fused(out, O.ce_fused(xc["H"], xc["W"], xc["labels"]))
    again = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True)
    assert torch.equal(again["dH"], out["dH"]) and torch.equal(again["dW"], out["dW"])
    # the same problem split across row chunks sums dW in chunk order: same values to rounding
    ch = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=128, grads=True)
    assert torch.equal(ch["lse"], out["lse"])
    check_grad(ch["dH"], out["dH"], "dH chunked vs split")


@pytest.mark.parametrize("N,d,V,ign,splits", [
    (1000, 4096, 65536, 17, 2),  # 4 x 8 wide tiles, the vocabulary in 2 ranges, ragged rows
    (1000, 4352, 65536, 0, 2),   # the last wide tile's second half lies past d
    (600, 1024, 262144, 9, 8),   # 6 wide tiles, 8 ranges of 32768 words
])
def test_wide_dh_tiles(N, d, V, ign, splits):
    # 256 x 512 pair tiles for dH (two MMAs per K step share the staged G), summed over the
    # vocabulary ranges in a fixed order
    assert L.lmh_dh_plan(N, d, V) == (True, splits)
    x, xc = device_inputs(_wl(N, d, V, ign))
    res = {}

    def run():
        res["o"] = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True)
    names = _kernels_launched(run)
    assert names.count("split_sum") == 1 and names.count("gemm_dH") == 1
    out = res["o"]
    assert L.lmh_read_errors(out["workspace"]) == 0
    check_ce_fused(out, O.ce_fused(xc["H"], xc["W"], xc["labels"]))
    again = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True)
    assert torch.equal(again["dH"], out["dH"]) and torch.equal(again["dW"], out["dW"])


def test_unsplit_wide_dh_has_the_narrow_bits():
    # one 4096-row chunk runs dH in 64 wide tiles, 1024-row chunks in 32 narrow ones, neither
    # split: the tensor core adds the same K steps in the same order, so dH has the same bits
    N, d, V = 4096, 2048, 32000
    assert L.lmh_dh_plan(N, d, V) == (True, 1) and L.lmh_dh_plan(1024, d, V) == (False, 1)
    x, _ = device_inputs(_wl(N, d, V, 40))
    wide = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True)
    narrow = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=1024, grads=True)
    assert torch.equal(wide["lse"], narrow["lse"])
    assert torch.equal(wide["dH"], narrow["dH"])


def test_wide_dw_tiles_and_bits():
    # one chunk of 8192 rows: dW's bf16 output in 256 x 512 pair tiles (and dH's too), with a
    # ragged vocabulary (12 row tiles of dW, the last partial) and d = 8.5 wide tiles
    N, d, V = 8192, 4352, 3000
    assert L.lmh_dh_plan(N, d, V) == (True, 1)
    x, xc = device_inputs(_wl(N, d, V, 61))
    out = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True)
    assert L.lmh_read_errors(out["workspace"]) == 0
    check_ce_fused(out, O.ce_fused(xc["H"], xc["W"], xc["labels"]))
    # a caller accumulator makes the same chunk's dW run 256 x 256 tiles (load, add to the
    # zeros, store the sum, cast): 0 + s is s, so the bits agree up to the sign of zero
    acc = torch.zeros(V, d, dtype=torch.float32, device="cuda")
    narrow = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True, dW_acc=acc)
    assert torch.equal(out["dW"].float() + 0.0, narrow["dW"].float() + 0.0)
    assert torch.equal(narrow["dW"], acc.to(torch.bfloat16))
    assert torch.equal(out["dH"], narrow["dH"])


def test_no_split_when_vocabulary_is_small():
    # V = 32000: the fp32 partials would cost more than the fuller waves give back
    x, _ = device_inputs(_wl(256, 256, 32000, 0))
    names = _kernels_launched(lambda: L.loss_fwd(x["H"], x["W"], x["labels"], grads=True))
    assert "split_sum" not in names and names.count("gemm_dH") == 1


@pytest.mark.parametrize("N,d,V,ign,chunk", [
    (256, 8192, 3000, 4, 0),      # 64 K blocks per logits tile, 32 dH column tiles
    (8, 128, 200000, 1, 0),       # 782 vocabulary tiles, dH split into 6 ranges, dW K = 8 rows
    (520, 64, 70001, 0, 200),     # minimum d, V one past a multiple of 8, 3 chunks
])
def test_extreme_aspect_ratios(N, d, V, ign, chunk):
    x, xc = device_inputs(_wl(N, d, V, ign))
    out = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=chunk, grads=True)
    torch.cuda.synchronize()
    assert L.lmh_read_errors(out["workspace"]) == 0
    check_ce_fused(out, O.ce_fused(xc["H"], xc["W"], xc["labels"]))
    lse = out["lse"]
    b = L.loss_bwd(L.BWD_CE, x["H"], x["W"], x["labels"], lse, None, chunk_rows=chunk, mean=True)
    check_grad(b["dH"], out["dH"], "dH recompute vs fused")
    check_grad(b["dW"], out["dW"], "dW recompute vs fused")


_DIGEST_SCRIPT = r"""
import sys
sys.path.insert(0, {root!r})
import torch
import lm_head_cross_tcgen05_b200 as L
from tests.gpu_common import digest
from workloads import make_inputs, ragged
x = {{k: v.cuda() for k, v in
      make_inputs(ragged(520, 256, 5000, n_ignored=9, seed=1000 + 520 + 256 + 5000)).items()}}
o = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=200, grads=True)
s = L.support_kl(x["H"], x["W"], torch.stack([x["labels"].clamp(min=0), x["labels"].clamp(min=0) + 1], 1),
                 torch.full((520, 2), -0.7, device="cuda"))
print(digest(o["loss_rows"], o["lse"], o["argmax"], o["dH"], o["dW"], s["kl_rows"], s["lp"]))
"""


def test_same_bits_in_a_new_process():
    # the pages' determinism contract: a fresh process (new context, new allocations,
    # first-call setup) gives the same bits as this one
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    script = _DIGEST_SCRIPT.format(root=root)
    here = subprocess.run([sys.executable, "-c", script], capture_output=True, text=True,
                          timeout=300, cwd=root)
    assert here.returncode == 0, here.stderr[-2000:]
    again = subprocess.run([sys.executable, "-c", script], capture_output=True, text=True,
                           timeout=300, cwd=root)
    assert again.returncode == 0, again.stderr[-2000:]
    x = device_inputs(_wl(520, 256, 5000, 9))[0]
    o = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=200, grads=True)
    ids = torch.stack([x["labels"].clamp(min=0), x["labels"].clamp(min=0) + 1], 1)
    s = L.support_kl(x["H"], x["W"], ids, torch.full((520, 2), -0.7, device="cuda"))
    mine = digest(o["loss_rows"], o["lse"], o["argmax"], o["dH"], o["dW"], s["kl_rows"], s["lp"])
    assert here.stdout.strip().splitlines()[-1] == again.stdout.strip().splitlines()[-1] == mine


@pytest.mark.parametrize("N,d,V,K,chunk,tau", [
    (200, 192, 3000, 16, 0, None),
    (300, 128, 5000, 8, 128, "rows"),   # three chunks: the internal dW accumulator
    (64, 256, 2048, 64, 0, "scalar"),
])
def test_support_kl_fused_backward(N, d, V, K, chunk, tau):
    x, xc = device_inputs(ragged(N, d, V, seed=4800 + N, K=K))
    ids = x["ids"].clone()
    ids[0, -1] = -1                      # padding
    ids[1, 1] = ids[1, 0]                # a repeated id counts once per slot
    ids_c = ids.cpu()
    t_dev, t_ref = _temps(tau, N) if tau else (None, None)
    out = L.support_kl(x["H"], x["W"], ids, x["ref_logp"], chunk_rows=chunk, temperature=t_dev,
                       grads=True)
    torch.cuda.synchronize()
    assert L.lmh_read_errors(out["workspace"]) == 0
    rk = O.support_kl(xc["H"], xc["W"], ids_c, xc["ref_logp"], tau=t_ref)
    check_rows(out["kl_rows"], rk["kl_rows"], what="kl_rows")
    check_rows(out["kl_mean"], np.array([rk["kl_mean"]]), what="kl_mean")
    check_rows(out["lp"], rk["lp"], what="lp")
    check_rows(out["lse"], rk["lse"], what="lse")
    ref = O.backward(O.BWD_SUPPORT_KL, xc["H"], xc["W"], ids_c, np.full(N, 1.0 / N),
                     xc["ref_logp"], tau=t_ref)
    check_grad(out["dH"], ref["dH"], "dH")
    check_grad(out["dW"], ref["dW"], "dW")
    # the two-call path: the same forward bits, the same gradients to rounding
    f = L.support_kl(x["H"], x["W"], ids, x["ref_logp"], chunk_rows=chunk, temperature=t_dev)
    assert torch.equal(f["kl_rows"], out["kl_rows"]) and torch.equal(f["lse"], out["lse"])
    b = L.loss_bwd(L.BWD_SUPPORT_KL, x["H"], x["W"], ids, f["lse"], None, x["ref_logp"],
                   chunk_rows=chunk, temperature=t_dev, mean=True)
    check_grad(out["dH"], b["dH"], "dH fused vs two calls")
    check_grad(out["dW"], b["dW"], "dW fused vs two calls")
    again = L.support_kl(x["H"], x["W"], ids, x["ref_logp"], chunk_rows=chunk,
                         temperature=t_dev, grads=True)
    assert torch.equal(again["dH"], out["dH"]) and torch.equal(again["dW"], out["dW"])


def test_support_kl_fused_sum_caller_accumulator_and_renorm_refused():
    N, d, V, K = 120, 128, 1500, 8
    x, xc = device_inputs(ragged(N, d, V, seed=4900, K=K))
    acc = torch.zeros(V, d, dtype=torch.float32, device="cuda")
    out = L.support_kl(x["H"], x["W"], x["ids"], x["ref_logp"], chunk_rows=50, grads=True,
                       mean=False, dW_acc=acc)
    ref = O.backward(O.BWD_SUPPORT_KL, xc["H"], xc["W"], xc["ids"], np.ones(N), xc["ref_logp"])
    check_grad(acc, ref["dW"], "dW_acc")
    assert torch.equal(out["dW"], acc.to(torch.bfloat16))
    check_grad(out["dH"], ref["dH"], "dH")
    with pytest.raises(L.LmhError, match="INVALID_ARG"):
        L.support_kl(x["H"], x["W"], x["ids"], x["ref_logp"], grads=True, renorm=True)


@pytest.mark.parametrize("mode", [L.BWD_CE, L.BWD_LOGPROB])
@pytest.mark.parametrize("chunk", [0, 100])
def test_weighted_fused_objective(mode, chunk):
    # a policy-gradient-like objective: per-row weights known before the forward
    N, d, V = 300, 192, 2000
    x, xc = device_inputs(_wl(N, d, V, 7))
    g = torch.linspace(-1.5, 1.0, N, dtype=torch.float32)
    out = L.loss_fwd_bwd(mode, x["H"], x["W"], x["labels"], g.cuda(), chunk_rows=chunk)
    torch.cuda.synchronize()
    assert L.lmh_read_errors(out["workspace"]) == 0
    f = O.ce_forward(xc["H"], xc["W"], xc["labels"])
    check_rows(out["loss_rows"], f["loss_rows"], what="loss_rows")
    check_rows(out["lse"], f["lse"], what="lse")
    ref = O.backward(mode, xc["H"], xc["W"], xc["labels"], g.numpy())
    check_grad(out["dH"], ref["dH"], "dH")
    check_grad(out["dW"], ref["dW"], "dW")
    fwd = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=chunk)
    assert torch.equal(fwd["lse"], out["lse"]) and torch.equal(fwd["loss_rows"], out["loss_rows"])
    b = L.loss_bwd(mode, x["H"], x["W"], x["labels"], out["lse"], g.cuda(), chunk_rows=chunk)
    check_grad(out["dH"], b["dH"], "dH fused vs standalone")
    check_grad(out["dW"], b["dW"], "dW fused vs standalone")


def test_weighted_fused_scalar_mean_count_and_temperature():
    N, d, V = 260, 128, 1500
    x, xc = device_inputs(_wl(N, d, V, 11))
    t_dev, t_ref = _temps("rows", N)
    n = torch.tensor([77], dtype=torch.int32, device="cuda")
    g = torch.tensor([2.5], dtype=torch.float32, device="cuda")
    out = L.loss_fwd_bwd(L.BWD_CE, x["H"], x["W"], x["labels"], g, mean=True, scalar_grad=True,
                         n_valid_given=n, temperature=t_dev, chunk_rows=128)
    valid = xc["labels"].numpy() >= 0
    w = np.where(valid, 2.5 / 77, 0.0)
    ref = O.backward(O.BWD_CE, xc["H"], xc["W"], xc["labels"], w, tau=t_ref)
    check_grad(out["dH"], ref["dH"], "dH")
    check_grad(out["dW"], ref["dW"], "dW")
    # without weights and with the mean: the same bits as lmh_loss_fwd's fused path
    a = L.loss_fwd_bwd(L.BWD_CE, x["H"], x["W"], x["labels"], None, mean=True, chunk_rows=128)
    b = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=128, grads=True)
    assert torch.equal(a["dH"], b["dH"]) and torch.equal(a["dW"], b["dW"])


@pytest.mark.parametrize("mode", [L.BWD_SUPPORT_LOGPROB, L.BWD_SUPPORT_KL])
def test_support_fwd_bwd_weighted(mode):
    N, d, V, K = 120, 128, 3000, 12
    x, xc = device_inputs(ragged(N, d, V, seed=5200, K=K))
    kl = mode == L.BWD_SUPPORT_KL
    shape_g = (N,) if kl else (N, K)
    g = torch.linspace(-1.0, 2.0, int(np.prod(shape_g)), dtype=torch.float32).view(shape_g)
    ref_lp = x["ref_logp"] if kl else None
    out = L.support_fwd_bwd(mode, x["H"], x["W"], x["ids"], g.cuda(), ref_lp, chunk_rows=50)
    torch.cuda.synchronize()
    assert L.lmh_read_errors(out["workspace"]) == 0
    if kl:
        rf = O.support_kl(xc["H"], xc["W"], xc["ids"], xc["ref_logp"])
        check_rows(out["kl_rows"], rf["kl_rows"], what="kl_rows")
    else:
        rf = O.support_logprob(xc["H"], xc["W"], xc["ids"])
    check_rows(out["lp"], rf["lp"], what="lp")
    check_rows(out["lse"], rf["lse"], what="lse")
    ref = O.backward(mode, xc["H"], xc["W"], xc["ids"], g.numpy(),
                     xc["ref_logp"] if kl else None)
    check_grad(out["dH"], ref["dH"], "dH")
    check_grad(out["dW"], ref["dW"], "dW")
    b = L.loss_bwd(mode, x["H"], x["W"], x["ids"], out["lse"], g.cuda(), ref_lp, chunk_rows=50)
    check_grad(out["dH"], b["dH"], "dH one pass vs standalone")
    check_grad(out["dW"], b["dW"], "dW one pass vs standalone")
