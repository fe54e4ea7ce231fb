"""Parity gates shared by the tests.

Tolerances (the targets stated for this path):
* loss, lse, log-prob, KL: absolute error <= 2e-3;
* dH, dW: max-abs error <= 1e-2 * max|ref| and cosine >= 0.9999, plus a relative-RMS
  budget of 1e-2 so that a 2 % scale error is rejected (the test plan of miles-ext-kernels
  PR #14, lm_head tests commit: an accuracy gate "checked to fail a 2 % error");
* integers (argmax, valid-row counts): exact.
"""
from __future__ import annotations

import numpy as np

ATOL_ROW = 2e-3
GRAD_MAXABS_FRAC = 1e-2
GRAD_COSINE = 0.9999
GRAD_REL_RMS = 1e-2


def f64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().float().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def check_rows(got, ref, atol: float = ATOL_ROW, what: str = "rows"):
    g, r = f64(got), f64(ref)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    if g.size == 0:
        return 0.0
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    err = float(np.max(np.abs(g - r)))
    assert err <= atol, f"{what}: max abs err {err:.3e} > {atol:.1e}"
    return err


def grad_metrics(got, ref):
    g, r = f64(got).ravel(), f64(ref).ravel()
    maxref = float(np.max(np.abs(r))) if r.size else 0.0
    maxerr = float(np.max(np.abs(g - r))) if r.size else 0.0
    nr, ng = float(np.linalg.norm(r)), float(np.linalg.norm(g))
    if nr == 0.0 and ng == 0.0:
        cos, rel = 1.0, 0.0
    elif nr == 0.0 or ng == 0.0:
        cos, rel = 0.0, float("inf")
    else:
        cos = float(np.dot(g, r) / (ng * nr))
        rel = float(np.linalg.norm(g - r) / nr)
    return dict(maxerr=maxerr, maxref=maxref, cos=cos, rel_rms=rel)


def check_grad(got, ref, what: str = "grad"):
    g, r = f64(got), f64(ref)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    return assert_grad_metrics(grad_metrics(g, r), what)


class GradStats:
    """check_grad over an array compared one block at a time, for arrays too large to hold
    twice in fp64 (a full-size dW): the same maximum errors, norms and inner product,
    accumulated over the blocks, then the same gates."""

    def __init__(self, what: str):
        self.what = what
        self.maxerr = self.maxref = 0.0
        self.dot = self.gg = self.rr = self.dd = 0.0

    def add(self, got, ref):
        g, r = f64(got), f64(ref)
        assert g.shape == r.shape, (self.what, g.shape, r.shape)
        assert np.all(np.isfinite(g)), f"{self.what}: non-finite values"
        if not r.size:
            return
        d = g - r
        self.maxerr = max(self.maxerr, float(np.max(np.abs(d))))
        self.maxref = max(self.maxref, float(np.max(np.abs(r))))
        gv, rv, dv = g.ravel(), r.ravel(), d.ravel()
        self.dot += float(np.dot(gv, rv))
        self.gg += float(np.dot(gv, gv))
        self.rr += float(np.dot(rv, rv))
        self.dd += float(np.dot(dv, dv))

    def check(self):
        nr, ng = self.rr ** 0.5, self.gg ** 0.5
        if nr == 0.0 and ng == 0.0:
            cos, rel = 1.0, 0.0
        elif nr == 0.0 or ng == 0.0:
            cos, rel = 0.0, float("inf")
        else:
            cos, rel = self.dot / (ng * nr), self.dd ** 0.5 / nr
        return assert_grad_metrics(dict(maxerr=self.maxerr, maxref=self.maxref, cos=cos,
                                        rel_rms=rel), self.what)


def assert_grad_metrics(m: dict, what: str):
    if m["maxref"] == 0.0:
        assert m["maxerr"] == 0.0, f"{what}: reference is zero, got max {m['maxerr']:.3e}"
        return m
    assert m["maxerr"] <= GRAD_MAXABS_FRAC * m["maxref"], f"{what}: {m}"
    assert m["cos"] >= GRAD_COSINE, f"{what}: {m}"
    assert m["rel_rms"] <= GRAD_REL_RMS, f"{what}: {m}"
    return m


def rejects(fn, *args) -> bool:
    """True when the gate ``fn`` raises on the given arguments."""
    try:
        fn(*args)
    except AssertionError:
        return True
    return False
