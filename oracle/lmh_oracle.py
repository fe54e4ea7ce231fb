"""fp64 CPU oracle for the deterministic chunked LM-head + loss.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this module.
The library (``lm_head_cross_tcgen05_b200``) never imports it, and it imports nothing
from the library: the two share no code.

What it states, in plain fp64 (inputs are the exact bf16 values widened to fp64):

* FlashInfer PR #8059 "feat(cake_lm_head_det_loss): det names for the chunked LM-head +
  loss backend", description: the backend computes the CE (and policy) losses, a
  log-probability entry, and "candidate-restricted" log-probabilities and a forward KL over
  a support set, in BF16, forward and backward.
* miles-ext-kernels PR #14 "[Cake 13/13]", the commit declaring
  ``miles_ext_kernels/cake/lm_head.py`` (its "Review items"): every negative label marks an
  ignored row; dW is the BF16 cast of an FP32 [V, H] accumulator.

The method reaches these results exactly up to rounding order, so each function is the
plain definition, with library matmuls as steps. Chunking only reorders rounding and has no
place here; ``chunk_plan`` states the row partition the library walks, for host-side tests.

Readings taken where the pages are silent:

* "candidate-restricted log-probabilities" are full-vocabulary log-probs evaluated at the
  candidate ids: lp_ik = z_i,c_ik - lse_i.
* "forward KL" is KL(ref || model) over the K candidates:
  KL_i = sum_k exp(r_ik) (r_ik - lp_ik).
* a label >= V is out of range: the row is ignored (and flagged).
* argmax takes the smallest index among equal maxima.
* the mean divides by the count of valid rows; with no valid row the loss is 0 and every
  gradient is 0.
* a candidate id < 0 is padding: it has lp = 0 and takes no part in the KL or gradients.
* temperature (the lm_head op commit's temperature stages: off, scalar, per row): every
  quantity is computed on the tempered logits z_iv / tau_i, and the gradients carry the chain
  rule factor 1 / tau_i. tau_i is a scalar, a per-row array, or None (off, the same as 1).

Parity status: every function here is pinned by the tests in
``tests/test_oracle_pins.py`` (brute force, closed forms, finite differences, invariants).
The pages print no numeric example, so no value is pinned to the pages themselves.
"""
from __future__ import annotations

import numpy as np

IGNORE_INDEX = -100

# Backward modes, same meaning as the library's LMH_BWD_* constants.
BWD_CE = 0
BWD_LOGPROB = 1
BWD_SUPPORT_LOGPROB = 2
BWD_SUPPORT_KL = 3


def as_f64(x) -> np.ndarray:
    """Widen a tensor/array (bf16 values included) to a float64 numpy array."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def as_i64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.asarray(x).astype(np.int64)


def chunk_plan(N: int, chunk_rows: int, default_chunk: int = 4096):
    """Row chunks [r0, r1) in the fixed order the library processes them.

    The chunk size defaults to 4096 rows (miles-ext-kernels PR #14, lm_head op commit:
    "--cake-lm-head-chunk-size (default 4096)"); the plan is part of the determinism key
    (FlashInfer PR #8059, description: "fixed inputs, hardware, chunk plan and initial
    accumulation buffers").
    """
    c = chunk_rows if chunk_rows > 0 else default_chunk
    return [(r0, min(N, r0 + c)) for r0 in range(0, N, c)]


def tau_rows(tau, N: int) -> np.ndarray:
    """Per-row temperatures as an [N] fp64 array (None: all ones)."""
    if tau is None:
        return np.ones(N)
    t = as_f64(tau)
    return np.full(N, float(t)) if t.ndim == 0 else t.reshape(N)


def logits(H, W, tau=None) -> np.ndarray:
    """z = H W^T, the LM-head logits, in fp64 ([N, V]); with a temperature, z_iv / tau_i."""
    z = as_f64(H) @ as_f64(W).T
    if tau is not None:
        z = z / tau_rows(tau, z.shape[0])[:, None]
    return z


def logsumexp_rows(z: np.ndarray) -> np.ndarray:
    """lse_i = m_i + log sum_v exp(z_iv - m_i), m_i = max_v z_iv."""
    m = z.max(axis=1)
    return m + np.log(np.exp(z - m[:, None]).sum(axis=1))


def valid_rows(labels, V: int):
    """(valid mask, out-of-range mask). Negative labels are ignored rows."""
    y = as_i64(labels)
    return (y >= 0) & (y < V), y >= V


def ce_forward(H, W, labels, tau=None) -> dict:
    """Cross-entropy forward: per-row loss, lse, target log-prob, argmax, count and mean.

    loss_i = lse_i - z_i,y_i and logprob_i = z_i,y_i - lse_i for valid rows, 0 for ignored
    rows; lse_i and argmax_i are reported for every row; mean = sum_valid loss / n_valid
    (0 when n_valid = 0).
    """
    z = logits(H, W, tau)
    N, V = z.shape
    y = as_i64(labels)
    valid, oob = valid_rows(y, V)
    lse = logsumexp_rows(z) if N else np.zeros(0)
    zy = np.zeros(N)
    zy[valid] = z[np.nonzero(valid)[0], y[valid]]
    loss = np.where(valid, lse - zy, 0.0)
    n_valid = int(valid.sum())
    mean = float(loss.sum() / n_valid) if n_valid else 0.0
    argmax = z.argmax(axis=1) if N else np.zeros(0, dtype=np.int64)  # first maximum
    return dict(z=z, lse=lse, loss_rows=loss, logprob=np.where(valid, -loss, 0.0),
                argmax=argmax, n_valid=n_valid, loss_mean=mean, label_out_of_range=bool(oob.any()))


def softmax_from(z: np.ndarray, lse: np.ndarray) -> np.ndarray:
    return np.exp(z - lse[:, None])


def grad_logits(mode: int, z: np.ndarray, lse: np.ndarray, targets, grad, ref_logp=None):
    """dL/dz for the four row objectives, as G [N, V].

    * BWD_CE: L = sum_i g_i loss_i -> G = g_i (P_i - e_{y_i}), valid rows only.
    * BWD_LOGPROB: L = sum_i g_i logprob_i -> G = g_i (e_{y_i} - P_i), valid rows only.
    * BWD_SUPPORT_LOGPROB: L = sum_ik g_ik lp_ik -> G = sum_k g_ik (e_{c_ik} - P_i).
    * BWD_SUPPORT_KL: L = sum_i g_i KL_i with KL_i = sum_k p_ik (r_ik - lp_ik), p = exp(r)
      -> G = g_i sum_k p_ik (P_i - e_{c_ik}).
    Candidate ids < 0 (padding) and >= V are skipped.
    """
    N, V = z.shape
    P = softmax_from(z, lse)
    if mode in (BWD_CE, BWD_LOGPROB):
        G = np.zeros_like(z)
        y = as_i64(targets)
        g = as_f64(grad).reshape(N)
        sign = 1.0 if mode == BWD_CE else -1.0
        for i in range(N):
            if 0 <= y[i] < V:
                G[i] = sign * g[i] * P[i]
                G[i, y[i]] -= sign * g[i]
        return G
    # Support objectives: each valid slot (i, k) adds w_ik (e_{c_ik} - P_i) to row i, with
    # w = g for the log-probs and w = -g_i exp(r_ik) for the KL. The P_i parts of a row are
    # one multiple of P_i (the sum of its slots' w), the one-hot parts a scatter-add of the
    # slots' w at their ids (repeated ids add once per slot).
    ids = as_i64(targets)
    K = ids.shape[1]
    ok = (ids >= 0) & (ids < V)
    if mode == BWD_SUPPORT_LOGPROB:
        w = as_f64(grad).reshape(N, K)
    elif mode == BWD_SUPPORT_KL:
        w = -as_f64(grad).reshape(N)[:, None] * np.exp(as_f64(ref_logp).reshape(N, K))
    else:
        raise ValueError(f"unknown backward mode {mode}")
    w = np.where(ok, w, 0.0)
    G = -w.sum(axis=1)[:, None] * P
    rr, kk = np.nonzero(ok)
    np.add.at(G, (rr, ids[rr, kk]), w[rr, kk])
    return G


def lm_head_backward(H, W, G: np.ndarray):
    """dH = G W and dW = G^T H (fp64), the two backward contractions of z = H W^T."""
    return G @ as_f64(W), G.T @ as_f64(H)


def ce_fused(H, W, labels, mean: bool = True, tau=None) -> dict:
    """Forward CE plus dH, dW of the reduced loss (mean over valid rows, or sum)."""
    f = ce_forward(H, W, labels, tau)
    N = f["z"].shape[0]
    if mean:
        g = np.full(N, 1.0 / f["n_valid"]) if f["n_valid"] else np.zeros(N)
    else:
        g = np.ones(N)
    G = grad_logits(BWD_CE, f["z"], f["lse"], labels, g) / tau_rows(tau, N)[:, None]
    dH, dW = lm_head_backward(H, W, G)
    f.update(G=G, dH=dH, dW=dW, grad_rows=g)
    return f


def logprob_forward(H, W, labels, tau=None) -> dict:
    """Per-row target log-prob z_i,y_i - lse_i (0 for ignored rows) and lse."""
    f = ce_forward(H, W, labels, tau)
    return dict(logprob=f["logprob"], lse=f["lse"], z=f["z"])


def support_logprob(H, W, ids, tau=None) -> dict:
    """lp_ik = z_i,c_ik - lse_i: full-vocabulary log-probs at K candidate ids per row."""
    z = logits(H, W, tau)
    N, V = z.shape
    c = as_i64(ids)
    lse = logsumexp_rows(z) if N else np.zeros(0)
    ok = (c >= 0) & (c < V)
    lp = np.zeros(c.shape)
    rr, kk = np.nonzero(ok)
    lp[rr, kk] = z[rr, c[rr, kk]] - lse[rr]
    return dict(lp=lp, lse=lse, z=z, out_of_range=bool((c >= V).any()))


def support_kl(H, W, ids, ref_logp, tau=None) -> dict:
    """KL_i = sum_k exp(r_ik) (r_ik - lp_ik) over valid candidates; mean over all N rows."""
    s = support_logprob(H, W, ids, tau)
    c = as_i64(ids)
    V = s["z"].shape[1]
    r = as_f64(ref_logp).reshape(c.shape)
    ok = (c >= 0) & (c < V)
    terms = np.where(ok, np.exp(r) * (r - s["lp"]), 0.0)
    kl = terms.sum(axis=1)
    N = c.shape[0]
    s.update(kl_rows=kl, kl_mean=float(kl.sum() / N) if N else 0.0)
    return s


def backward(mode: int, H, W, targets, grad, ref_logp=None, tau=None) -> dict:
    """Standalone backward of one of the four row objectives: recompute z and lse, form G,
    contract. The library's backward takes lse from its forward; here it is recomputed,
    which is the same value. With a temperature, G carries the factor 1 / tau_i."""
    z = logits(H, W, tau)
    lse = logsumexp_rows(z) if z.shape[0] else np.zeros(0)
    G = grad_logits(mode, z, lse, targets, grad, ref_logp) / tau_rows(tau, z.shape[0])[:, None]
    dH, dW = lm_head_backward(H, W, G)
    return dict(G=G, dH=dH, dW=dW, lse=lse)


# ---------------------------------------------------------------- renormalised support set
# The other reading of "candidate-restricted log-probabilities": log-probs normalised over the
# row's distinct valid candidate ids (the support) instead of the whole vocabulary.

def support_renorm_logprob(H, W, ids, tau=None) -> dict:
    """lpK_ik = z_i,c_ik - log sum_{c in S_i} exp z_ic, S_i the distinct valid ids of row i;
    lseK_i is that log-normaliser (0 for a row without candidates); padding slots get 0."""
    z = logits(H, W, tau)
    N, V = z.shape
    c = as_i64(ids)
    lp = np.zeros(c.shape)
    lse = np.zeros(N)
    for i in range(N):
        S = sorted({int(v) for v in c[i] if 0 <= v < V})
        if not S:
            continue
        zs = z[i, S]
        m = zs.max()
        lse[i] = m + np.log(np.exp(zs - m).sum())
        for k in range(c.shape[1]):
            if 0 <= c[i, k] < V:
                lp[i, k] = z[i, c[i, k]] - lse[i]
    return dict(lp=lp, lse=lse, z=z)


def support_renorm_kl(H, W, ids, ref_logp, tau=None) -> dict:
    """KL_i = sum_k exp(r_ik) (r_ik - lpK_ik) over valid slots; mean over all N rows."""
    s = support_renorm_logprob(H, W, ids, tau)
    c = as_i64(ids)
    V = s["z"].shape[1]
    r = as_f64(ref_logp).reshape(c.shape)
    ok = (c >= 0) & (c < V)
    kl = np.where(ok, np.exp(r) * (r - s["lp"]), 0.0).sum(axis=1)
    N = c.shape[0]
    s.update(kl_rows=kl, kl_mean=float(kl.sum() / N) if N else 0.0)
    return s


def backward_renorm(mode: int, H, W, ids, grad, ref_logp=None, tau=None) -> dict:
    """Backward of sum_ik g_ik lpK_ik (BWD_SUPPORT_LOGPROB) or sum_i g_i KL_i (BWD_SUPPORT_KL)
    over the renormalised support: with q = softmax of z over S_i,
    dL/dz_ic = sum_{k: c_ik = c} w_ik - q_ic sum_k w_ik for c in S_i (w = g for log-probs,
    w = -g_i exp(r_ik) for the KL), 0 outside S_i; times 1 / tau_i."""
    s = support_renorm_logprob(H, W, ids, tau)
    z, lse = s["z"], s["lse"]
    N, V = z.shape
    c = as_i64(ids)
    K = c.shape[1]
    if mode == BWD_SUPPORT_LOGPROB:
        w = as_f64(grad).reshape(N, K)
    elif mode == BWD_SUPPORT_KL:
        w = -as_f64(grad).reshape(N)[:, None] * np.exp(as_f64(ref_logp).reshape(N, K))
    else:
        raise ValueError("renormalised backward exists for the support objectives only")
    G = np.zeros_like(z)
    for i in range(N):
        S = sorted({int(v) for v in c[i] if 0 <= v < V})
        if not S:
            continue
        q = np.exp(z[i, S] - lse[i])
        wsum = sum(w[i, k] for k in range(K) if 0 <= c[i, k] < V)
        for j, v in enumerate(S):
            G[i, v] = sum(w[i, k] for k in range(K) if c[i, k] == v) - q[j] * wsum
    G = G / tau_rows(tau, N)[:, None]
    dH, dW = lm_head_backward(H, W, G)
    return dict(G=G, dH=dH, dW=dW, lse=lse)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round fp64 -> fp32 -> bf16 (round to nearest even), returned as fp64 values."""
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    nan = np.isnan(f)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    out = (r & 0xFFFFFFFF).astype(np.uint32).view(np.float32).astype(np.float64)
    out[nan] = np.nan
    return out
