"""Shared pieces of the GPU parity tests: inputs on the device, oracle results on the host."""
from __future__ import annotations

import hashlib

import numpy as np
import torch

from oracle import lmh_oracle as O
from tests.parity import check_grad, check_rows, f64
from workloads import Workload, make_inputs, ragged


def device_inputs(wl: Workload, seed=None):
    x = make_inputs(wl, device="cpu", seed=seed)
    return {k: v.cuda() for k, v in x.items()}, x


def digest(*ts) -> str:
    h = hashlib.sha256()
    for t in ts:
        if t is None:
            continue
        h.update(t.detach().contiguous().cpu().view(torch.uint8).numpy().tobytes()
                 if t.dtype != torch.bfloat16 else
                 t.detach().contiguous().cpu().view(torch.int16).numpy().tobytes())
    return h.hexdigest()


def check_argmax(got, z: np.ndarray, gap: float = 1e-3):
    """argmax exact where the oracle's top-2 gap exceeds `gap`; elsewhere the chosen id must
    attain the maximum within `gap`."""
    g = got.cpu().numpy().astype(np.int64)
    srt = np.sort(z, axis=1)
    top2gap = srt[:, -1] - srt[:, -2] if z.shape[1] > 1 else np.full(z.shape[0], np.inf)
    ref = z.argmax(axis=1)
    clear = top2gap > gap
    assert np.array_equal(g[clear], ref[clear]), np.nonzero(g[clear] != ref[clear])
    rows = np.arange(z.shape[0])
    assert np.all(z[rows, g] >= z.max(axis=1) - gap)


def check_ce_fused(out: dict, ref: dict, grads: bool = True):
    check_rows(out["loss_rows"], ref["loss_rows"], what="loss_rows")
    check_rows(out["lse"], ref["lse"], what="lse")
    check_rows(out["logprob"], ref["logprob"], what="logprob")
    check_rows(out["loss_mean"], np.array([ref["loss_mean"]]), what="loss_mean")
    assert int(out["n_valid"].item()) == ref["n_valid"]
    check_argmax(out["argmax"], ref["z"])
    if grads:
        if out.get("dH") is not None:
            check_grad(out["dH"], ref["dH"], "dH")
        if out.get("dW") is not None:
            check_grad(out["dW"], ref["dW"], "dW")


__all__ = ["device_inputs", "digest", "check_argmax", "check_ce_fused", "O", "f64", "ragged",
           "check_rows", "check_grad"]
