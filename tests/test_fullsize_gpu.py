"""Parity at the full sizes of the four large workloads, in the launch configuration bench.py
uses (one chunk of all rows for large_vocab and support, 2048-row chunks into a caller-owned
fp32 accumulator for budgeted).

Every output of those steps is compared with the fp64 oracle element by element: per-row
outputs for all rows, dH for all rows and dW in full. The oracle runs over 1024-row blocks
(its logits, softmax gradient and both contractions per block, dW summed over the blocks in
fp64), and the gradient gates are accumulated block by block (``GradStats``), so a full-size
dW never needs two fp64 copies. That is about 3.3e13, 9.8e13 and 4.1e13 fp64 flops for the
three workloads: minutes of host CPU. Properties that hold at any size (columns of dW summing
to zero, bitwise repeats, one chunk against many) are checked as well."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import lm_head_cross_tcgen05_b200 as L
from tests.gpu_common import O, check_argmax, check_grad, check_rows, digest, f64
from tests.parity import GradStats
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def sample_rows(y: torch.Tensor, n: int = 12, seed: int = 0) -> np.ndarray:
    """n rows spread over the batch, with at least one ignored row when there is one."""
    N = y.shape[0]
    g = np.random.default_rng(seed)
    rows = set(g.choice(N, size=n, replace=False).tolist()) | {0, N - 1}
    ign = torch.nonzero(y < 0).flatten().tolist()
    if ign:
        rows.add(ign[0])
    return np.array(sorted(rows))


def dev_inputs(name):
    wl = WORKLOADS[name]
    return wl, make_inputs(wl, device="cuda")


def check_sampled_ce(out, x, rows, n_valid_total):
    Hs, ys = x["H"][rows].cpu(), x["labels"][rows].cpu()
    Wc = x["W"].cpu()
    f = O.ce_forward(Hs, Wc, ys)
    check_rows(out["loss_rows"][rows], f["loss_rows"], what="loss_rows")
    check_rows(out["lse"][rows], f["lse"], what="lse")
    check_rows(out["logprob"][rows], f["logprob"], what="logprob")
    check_argmax(out["argmax"][rows], f["z"])
    if out.get("dH") is not None:
        valid = (ys.numpy() >= 0)
        g = np.where(valid, 1.0 / n_valid_total, 0.0)
        b = O.backward(O.BWD_CE, Hs, Wc, ys, g)
        check_grad(out["dH"][rows], b["dH"], "dH rows")


def check_dw_properties(dW: torch.Tensor):
    s = dW.float().sum(0).double()                     # sum over the vocabulary
    a = dW.float().abs().sum(0).double()
    assert torch.all(s.abs() <= 2e-3 * a + 1e-6), float((s.abs() / (a + 1e-30)).max())
    assert torch.isfinite(dW.float()).all()


@pytest.fixture(scope="module")
def large_vocab():
    wl, x = dev_inputs("large_vocab")
    out = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=wl.N, grads=True)
    torch.cuda.synchronize()
    return wl, x, out


def test_large_vocab_sampled_rows(large_vocab):
    wl, x, out = large_vocab
    y = x["labels"]
    n_valid = int(((y >= 0) & (y < wl.V)).sum())
    assert int(out["n_valid"].item()) == n_valid == wl.N - wl.num_ignored
    assert L.lmh_read_errors(out["workspace"]) == 0
    check_sampled_ce(out, x, sample_rows(y), n_valid)
    # the mean is the fixed-order mean of the per-row losses over valid rows
    lr = out["loss_rows"].double()
    assert abs(float(out["loss_mean"]) - float(lr.sum() / n_valid)) < 1e-4


def test_large_vocab_dw_properties_and_repeats(large_vocab):
    wl, x, out = large_vocab
    check_dw_properties(out["dW"])
    h = digest(out["dW"], out["dH"], out["lse"], out["loss_rows"])
    ws = out["workspace"]
    for _ in range(9):
        o = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=wl.N, grads=True, ws=ws)
        assert digest(o["dW"], o["dH"], o["lse"], o["loss_rows"]) == h


def test_large_vocab_fused_matches_recompute_and_chunking(large_vocab):
    wl, x, out = large_vocab
    n = int(out["n_valid"].item())
    grad = torch.where(x["labels"] >= 0, 1.0 / n, 0.0).float()
    b = L.loss_bwd(L.BWD_CE, x["H"], x["W"], x["labels"], out["lse"], grad, chunk_rows=wl.N)
    ref_dw = f64(out["dW"])
    check_grad(b["dW"], ref_dw, "dW recompute vs fused")
    check_grad(b["dH"], f64(out["dH"]), "dH recompute vs fused")
    del b
    c = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=3000, grads=True)
    # the forward outputs never depend on the chunk plan; dH of 3000-row chunks is summed over
    # vocabulary ranges (too few tiles to fill the GPU) and dW over chunks: same values to
    # rounding
    assert torch.equal(c["lse"], out["lse"]) and torch.equal(c["loss_rows"], out["loss_rows"])
    check_grad(c["dH"], f64(out["dH"]), "dH 3 chunks vs 1")
    check_grad(c["dW"], ref_dw, "dW 3 chunks vs 1")


def test_full_vocab_and_hidden_dw_slice():
    """dW element by element at V = 128256, d = 4096 on a 128-row slice."""
    wl = WORKLOADS["large_vocab"].scaled(N=128)
    x = make_inputs(wl, device="cuda")
    out = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True)
    ref = O.ce_fused(x["H"].cpu(), x["W"].cpu(), x["labels"].cpu())
    check_grad(out["dW"], ref["dW"], "dW")
    check_grad(out["dH"], ref["dH"], "dH")
    check_rows(out["lse"], ref["lse"], what="lse")


BLOCK = 1024


def full_oracle(x, out, kind, n_valid=None, acc=None):
    """Every row's outputs, all of dH and all of dW (and acc, a caller's fp32 accumulator)
    against the fp64 oracle, over blocks of BLOCK rows. kind "ce": the mean cross entropy
    over n_valid rows (loss_rows, lse, logprob, argmax, loss_mean); "support_kl": the mean KL
    over all rows (kl_rows, kl_mean, lp, lse)."""
    Hc = x["H"].cpu()
    W64 = O.as_f64(x["W"].cpu())
    N, d = Hc.shape
    V = W64.shape[0]
    got = {k: v.cpu() for k, v in out.items()
           if isinstance(v, torch.Tensor) and k not in ("workspace", "dW")}
    dW = np.zeros((V, d))
    sH = GradStats("dH (all rows)")
    total = 0.0
    for r0 in range(0, N, BLOCK):
        r1 = min(N, r0 + BLOCK)
        Hb = O.as_f64(Hc[r0:r1])
        if kind == "ce":
            y = x["labels"][r0:r1].cpu()
            f = O.ce_forward(Hb, W64, y)
            for k in ("loss_rows", "lse", "logprob"):
                check_rows(got[k][r0:r1], f[k], what=f"{k} rows {r0}..{r1}")
            check_argmax(got["argmax"][r0:r1], f["z"])
            total += float(f["loss_rows"].sum())
            g = np.where(O.valid_rows(y, V)[0], 1.0 / n_valid, 0.0)
            G = O.grad_logits(O.BWD_CE, f["z"], f["lse"], y, g)
        else:
            ids, ref = x["ids"][r0:r1].cpu(), x["ref_logp"][r0:r1].cpu()
            f = O.support_kl(Hb, W64, ids, ref)
            for k in ("kl_rows", "lp", "lse"):
                check_rows(got[k][r0:r1], f[k], what=f"{k} rows {r0}..{r1}")
            total += float(f["kl_rows"].sum())
            G = O.grad_logits(O.BWD_SUPPORT_KL, f["z"], f["lse"], ids, np.full(r1 - r0, 1.0 / N),
                              ref)
        del f
        dHb, dWb = O.lm_head_backward(Hb, W64, G)
        del G
        sH.add(got["dH"][r0:r1], dHb)
        dW += dWb
        del dWb
    sH.check()
    mean = "loss_mean" if kind == "ce" else "kl_mean"
    check_rows(got[mean], np.array([total / (n_valid if kind == "ce" else N)]), what=mean)
    sW, sA = GradStats("dW (full)"), GradStats("fp32 dW accumulator (full)")
    dW_got = out["dW"].cpu()
    acc_got = acc.cpu() if acc is not None else None
    for v0 in range(0, V, 8192):
        sW.add(dW_got[v0:v0 + 8192], dW[v0:v0 + 8192])
        if acc_got is not None:
            sA.add(acc_got[v0:v0 + 8192], dW[v0:v0 + 8192])
    sW.check()
    if acc_got is not None:
        sA.check()


def test_large_vocab_full_oracle(large_vocab):
    """The headline step (8192 x 128256 x 4096, one chunk): every output against the oracle."""
    wl, x, out = large_vocab
    n = int(O.valid_rows(x["labels"].cpu(), wl.V)[0].sum())
    assert int(out["n_valid"].item()) == n
    full_oracle(x, out, "ce", n_valid=n)


def test_small_workload_full_oracle():
    wl, x = dev_inputs("small")
    out = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=wl.N, grads=True)
    ref = O.ce_fused(x["H"].cpu(), x["W"].cpu(), x["labels"].cpu())
    check_rows(out["loss_rows"], ref["loss_rows"], what="loss_rows")
    check_rows(out["lse"], ref["lse"], what="lse")
    check_rows(out["logprob"], ref["logprob"], what="logprob")
    check_rows(out["loss_mean"], np.array([ref["loss_mean"]]), what="loss_mean")
    assert int(out["n_valid"].item()) == ref["n_valid"]
    check_argmax(out["argmax"], ref["z"])
    check_grad(out["dH"], ref["dH"], "dH")
    check_grad(out["dW"], ref["dW"], "dW")


def test_budgeted_workload_chunked_with_caller_accumulator():
    """16384 x 151936 x 5120 in 8 chunks of 2048 rows, dW accumulated in chunk order into a
    caller-owned fp32 buffer: every output, the accumulator and the log-prob entry against
    the oracle."""
    wl, x = dev_inputs("budgeted")
    shape = L.make_shape(wl.N, wl.d, wl.V, 0, wl.chunk_rows,
                         L.F_MEAN | L.F_FUSED_BWD | L.F_DW_ACC_GIVEN)
    assert L.lmh_workspace_size(shape, L.ENTRY_LOSS_FWD) <= 2 * 1024 ** 3
    acc = torch.zeros(wl.V, wl.d, dtype=torch.float32, device="cuda")
    out = L.loss_fwd(x["H"], x["W"], x["labels"], chunk_rows=wl.chunk_rows, grads=True,
                     dW_acc=acc)
    torch.cuda.synchronize()
    assert L.lmh_read_errors(out["workspace"]) == 0
    assert torch.equal(out["dW"], acc.to(torch.bfloat16))
    check_dw_properties(out["dW"])
    y = x["labels"]
    lp = L.logprob(x["H"], x["W"], y, chunk_rows=wl.chunk_rows)
    assert torch.equal(lp["logprob"], out["logprob"]) and torch.equal(lp["lse"], out["lse"])
    n = int(O.valid_rows(y.cpu(), wl.V)[0].sum())
    assert int(out["n_valid"].item()) == n == wl.N
    full_oracle(x, out, "ce", n_valid=n, acc=acc)


def test_support_workload_sampled_rows():
    wl, x = dev_inputs("support")
    ids, ref = x["ids"], x["ref_logp"]
    kl = L.support_kl(x["H"], x["W"], ids, ref, chunk_rows=wl.N)
    lp = L.support_logprob(x["H"], x["W"], ids, chunk_rows=wl.N)
    assert torch.equal(kl["lp"], lp["lp"])
    rows = sample_rows(x["labels"], seed=5)
    Hs, Wc = x["H"][rows].cpu(), x["W"].cpu()
    r = O.support_kl(Hs, Wc, ids[rows].cpu(), ref[rows].cpu())
    check_rows(kl["lp"][rows], r["lp"], what="lp")
    check_rows(kl["kl_rows"][rows], r["kl_rows"], what="kl_rows")
    check_rows(kl["lse"][rows], r["lse"], what="lse")
    assert abs(float(kl["kl_mean"]) - float(kl["kl_rows"].double().mean())) < 1e-4
    # backward of the mean KL
    grad = torch.full((wl.N,), 1.0 / wl.N, device="cuda")
    b = L.loss_bwd(L.BWD_SUPPORT_KL, x["H"], x["W"], ids, kl["lse"], grad, ref,
                   chunk_rows=wl.N)
    rb = O.backward(O.BWD_SUPPORT_KL, Hs, Wc, ids[rows].cpu(), np.full(len(rows), 1.0 / wl.N),
                    ref[rows].cpu())
    check_grad(b["dH"][rows], rb["dH"], "dH rows (KL)")
    check_dw_properties(b["dW"])
    # the one-pass entry bench.py times for this workload: same forward bits, same gradients
    f = L.support_kl(x["H"], x["W"], ids, ref, chunk_rows=wl.N, grads=True)
    assert torch.equal(f["kl_rows"], kl["kl_rows"]) and torch.equal(f["lse"], kl["lse"])
    check_grad(f["dH"][rows], rb["dH"], "dH rows (KL, one pass)")
    check_grad(f["dH"], b["dH"], "dH one pass vs two calls")
    check_grad(f["dW"], b["dW"], "dW one pass vs two calls")
    check_dw_properties(f["dW"])


def test_large_vocab_vocabulary_parallel_step(large_vocab):
    # bench.py's vocab_parallel step at one rank (the full workload): the records' combine
    # gives the one-device lse to fp32 rounding and the same argmax; gradients agree
    from lm_head_cross_tcgen05_b200.vocab_parallel import VocabParallelCE
    wl, x, out = large_vocab
    vp = VocabParallelCE(wl.V, chunk_rows=wl.N)
    f = vp.forward_backward(x["H"], x["W"], x["labels"])
    torch.cuda.synchronize()
    assert (f["lse"] - out["lse"]).abs().max().item() < 1e-4
    assert torch.equal(f["argmax"], out["argmax"])
    check_grad(f["dH"], f64(out["dH"]), "dH vocabulary-parallel vs one device")
    check_grad(f["dW"], f64(out["dW"]), "dW vocabulary-parallel vs one device")


def test_large_vocab_data_parallel_two_ranks(large_vocab):
    # the large_vocab batch split over two data-parallel ranks on this GPU, through both dW
    # exchanges: per-row results are the one-device bits, the dW sums agree with the
    # one-device dW, and the row scatter from the dW GEMM gives the collective route's bits
    from lm_head_cross_tcgen05_b200._ranks import row_slices
    from lm_head_cross_tcgen05_b200.data_parallel import CudaOps
    wl, x, out = large_vocab
    H, W, y = x["H"], x["W"], x["labels"]
    V, d = W.shape
    bounds = [(0, 5000), (5000, wl.N)]
    ops = CudaOps()
    n = (ops.count_valid(y[:5000], V) + ops.count_valid(y[5000:], V)).to(torch.int32)
    parts = [ops.fused(H[a:b], W, y[a:b], n, chunk_rows=b - a) for a, b in bounds]
    for k in ("loss_rows", "lse", "argmax"):
        assert torch.equal(torch.cat([p[k] for p in parts]), out[k]), k
    dW = ops.reduce_rows(torch.stack([p.pop("dW_part") for p in parts]))
    check_grad(torch.cat([p["dH"] for p in parts]), f64(out["dH"]), "dH two ranks")
    check_grad(dW, f64(out["dW"]), "dW two ranks vs one device")
    check_dw_properties(dW)
    sizes = [b - a for a, b in row_slices(V, 2)]
    recv = [torch.full((2 * max(sizes) * d,), float("nan"), device="cuda") for _ in range(2)]
    outs = [torch.zeros(V, d, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    rt = torch.tensor([t.data_ptr() for t in recv], dtype=torch.int64, device="cuda")
    ot = torch.tensor([t.data_ptr() for t in outs], dtype=torch.int64, device="cuda")
    for r, (a, b) in enumerate(bounds):
        g = ops.fused_scatter(H[a:b], W, y[a:b], n, (rt, 2, r))
        assert torch.equal(g["dH"], parts[r]["dH"])
    ops.reduce_rows_to(recv[0][: 2 * sizes[0] * d].view(2, sizes[0], d), ot, 2, 0)
    ops.reduce_rows_to(recv[1][: 2 * sizes[1] * d].view(2, sizes[1], d), ot, 2, sizes[0])
    torch.cuda.synchronize()
    assert torch.equal(outs[0], dW) and torch.equal(outs[1], dW)


def test_many_chunks_and_large_row_indices():
    # 131149 rows in 33 default-size chunks (32 x 4096 + 77): the dW accumulator is stored,
    # added 31 times and finally added and cast in the epilogue; row indices pass 2^17 and
    # per-row partial offsets pass 2^20. The full fp64 oracle still fits (V = 300).
    from workloads import ragged
    wl = ragged(131149, 64, 300, n_ignored=1000, seed=4500)
    x = make_inputs(wl, device="cuda")
    out = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True)
    torch.cuda.synchronize()
    assert L.lmh_read_errors(out["workspace"]) == 0
    xc = {k: v.cpu() for k, v in x.items()}
    ref = O.ce_fused(xc["H"], xc["W"], xc["labels"])
    check_rows(out["loss_rows"], ref["loss_rows"], what="loss_rows")
    check_rows(out["lse"], ref["lse"], what="lse")
    check_rows(out["loss_mean"], np.array([ref["loss_mean"]]), what="loss_mean")
    assert int(out["n_valid"].item()) == ref["n_valid"]
    check_argmax(out["argmax"], ref["z"])
    check_grad(out["dH"], ref["dH"], "dH")
    check_grad(out["dW"], ref["dW"], "dW")
    again = L.loss_fwd(x["H"], x["W"], x["labels"], grads=True)
    assert torch.equal(again["dW"], out["dW"]) and torch.equal(again["dH"], out["dH"])


def test_support_workload_one_pass_full_oracle():
    """The support step bench.py times (8192 x 151936 x 4096, K = 64, the mean KL's forward
    and backward in one pass): every output against the oracle."""
    wl, x = dev_inputs("support")
    out = L.support_kl(x["H"], x["W"], x["ids"], x["ref_logp"], chunk_rows=wl.N, grads=True)
    torch.cuda.synchronize()
    assert L.lmh_read_errors(out["workspace"]) == 0
    lp = L.support_logprob(x["H"], x["W"], x["ids"], chunk_rows=wl.N)
    assert torch.equal(lp["lp"], out["lp"]) and torch.equal(lp["lse"], out["lse"])
    full_oracle(x, out, "support_kl")
