"""Seeded synthetic inputs for the chunked LM-head + loss.

This module only draws random inputs. It holds none of the method's arithmetic
(no logits, no softmax of the model, no gradients) and imports neither the CUDA
package nor the oracle; both the GPU path and the oracle are fed from here.

Shapes and value distributions follow the five workloads the path is measured on:

=============  =====  ====  ======  ==========================================
name           N      d     V       extras
=============  =====  ====  ======  ==========================================
tiny           64     256   2048    uniform labels, exactly 8 rows ignored
small          4096   2048  32000   Zipf(1.1) labels, 5 % rows ignored
large_vocab    8192   4096  128256  Zipf(1.1) labels, 3 % rows ignored
budgeted       16384  5120  151936  W ~ N(0, 0.015^2), uniform labels,
                                    chunk_rows = 2048
support        8192   4096  151936  K = 64 candidate ids per row (label
                                    included, no repeats) and reference
                                    log-probs over them
=============  =====  ====  ======  ==========================================

H ~ N(0, 1) and W ~ N(0, sigma_W^2) are rounded to bf16. Ignored rows carry the
label -100. The seed of workload k (0-based, in the order above) is 1234 + k.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

IGNORE_INDEX = -100


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    N: int
    d: int
    V: int
    w_std: float = 0.02
    labels: str = "uniform"          # "uniform" | "zipf"
    n_ignored: Optional[int] = None  # exact count of ignored rows
    ignore_frac: float = 0.0         # else round(ignore_frac * N)
    chunk_rows: int = 0              # 0: one chunk holds every row
    K: int = 0                       # candidate ids per row (support entries)
    ref_eps_std: float = 0.0         # std of the W perturbation behind ref log-probs
    index: int = 0

    @property
    def seed(self) -> int:
        return 1234 + self.index

    @property
    def num_ignored(self) -> int:
        if self.n_ignored is not None:
            return self.n_ignored
        return int(round(self.ignore_frac * self.N))

    def flops_fwd_bwd(self) -> int:
        """6 N V d: 2NVd for the logits, 4NVd for dH and dW."""
        return 6 * self.N * self.V * self.d

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 64, 256, 2048, n_ignored=8, index=0),
    "small": Workload("small", 4096, 2048, 32000, labels="zipf", ignore_frac=0.05, index=1),
    "large_vocab": Workload("large_vocab", 8192, 4096, 128256, labels="zipf",
                            ignore_frac=0.03, index=2),
    "budgeted": Workload("budgeted", 16384, 5120, 151936, w_std=0.015, chunk_rows=2048,
                         index=3),
    "support": Workload("support", 8192, 4096, 151936, K=64, ref_eps_std=0.002, index=4),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def zipf_labels(n: int, V: int, s: float, gen: torch.Generator, device) -> torch.Tensor:
    """Labels with P(k) proportional to (k+1)^-s over 0..V-1, by inverse-CDF sampling."""
    k = torch.arange(1, V + 1, dtype=torch.float64, device=device)
    cdf = torch.cumsum(k.pow(-s), 0)
    cdf = cdf / cdf[-1]
    u = torch.rand(n, generator=gen, dtype=torch.float64, device=device)
    return torch.searchsorted(cdf, u).clamp_(max=V - 1).to(torch.int32)


def make_hw(N: int, d: int, V: int, w_std: float, seed: int, device="cpu"):
    """H [N,d] ~ N(0,1) and W [V,d] ~ N(0, w_std^2), both rounded to bf16."""
    g = _gen(seed, device)
    H = torch.randn(N, d, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    W = (torch.randn(V, d, generator=g, device=device, dtype=torch.float32) * w_std).to(
        torch.bfloat16)
    return H, W


def make_labels(wl: Workload, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed + 7919, device)
    if wl.labels == "zipf":
        y = zipf_labels(wl.N, wl.V, 1.1, g, device)
    else:
        y = torch.randint(0, wl.V, (wl.N,), generator=g, device=device, dtype=torch.int64).to(
            torch.int32)
    n_ign = wl.num_ignored
    if n_ign:
        rows = torch.randperm(wl.N, generator=g, device=device)[:n_ign]
        y[rows] = IGNORE_INDEX
    return y


def make_candidates(labels: torch.Tensor, V: int, K: int, seed: int) -> torch.Tensor:
    """K distinct ids per row, the row's label among them at a random position.

    Rows whose label is negative get K distinct random ids. Drawn on the host with
    numpy (without replacement per row), returned as int32 [N, K] on the CPU.
    """
    rng = np.random.default_rng(seed + 104729)
    y = labels.cpu().numpy().astype(np.int64)
    N = y.shape[0]
    out = np.empty((N, K), dtype=np.int32)
    for i in range(N):
        if y[i] >= 0:
            others = rng.choice(V - 1, size=K - 1, replace=False)
            others = others + (others >= y[i])          # skip the label itself
            row = np.concatenate([[y[i]], others])
        else:
            row = rng.choice(V, size=K, replace=False)
        rng.shuffle(row)
        out[i] = row
    return torch.from_numpy(out)


def make_ref_logprobs(H: torch.Tensor, W: torch.Tensor, ids: torch.Tensor, eps_std: float,
                      seed: int, block_rows: int = 256) -> torch.Tensor:
    """Reference log-probs over each row's K candidates.

    A perturbed weight W' = W + eps (eps ~ N(0, eps_std^2), one draw per element of W)
    scores the candidates, z'_ik = <H_i, W'_{ids_ik}>, and the scores are renormalised over
    the K candidates of the row: ref_ik = z'_ik - log sum_k exp z'_ik. Computed in fp32 on
    the tensors' device. This is how the reference distribution is built; it is an input
    of the KL entry, not part of the method.
    """
    dev = H.device
    g = _gen(seed + 15485863, dev)
    eps = torch.randn(W.shape, generator=g, device=dev, dtype=torch.float32) * eps_std
    Wp = W.float() + eps
    ids_d = ids.to(dev).long()
    out = torch.empty(ids.shape, dtype=torch.float32, device=dev)
    Hf = H.float()
    for r0 in range(0, H.shape[0], block_rows):
        r1 = min(H.shape[0], r0 + block_rows)
        Wc = Wp[ids_d[r0:r1]]                                  # [b, K, d]
        zp = torch.einsum("bkd,bd->bk", Wc, Hf[r0:r1])
        out[r0:r1] = zp - torch.logsumexp(zp, dim=1, keepdim=True)
    return out


def make_inputs(wl: Workload, device="cpu", seed: Optional[int] = None) -> dict:
    """All inputs of a workload: H, W, labels (+ ids, ref_logp for support workloads)."""
    seed = wl.seed if seed is None else seed
    H, W = make_hw(wl.N, wl.d, wl.V, wl.w_std, seed, device)
    labels = make_labels(wl, seed, device)
    out = dict(H=H, W=W, labels=labels)
    if wl.K:
        ids = make_candidates(labels, wl.V, wl.K, seed).to(device)
        out["ids"] = ids
        out["ref_logp"] = make_ref_logprobs(H, W, ids, wl.ref_eps_std or 0.002, seed)
    return out


def ragged(N: int, d: int, V: int, *, seed: int = 99, n_ignored: int = 0, K: int = 0,
           w_std: float = 0.02, labels: str = "uniform") -> Workload:
    """A small ad-hoc workload (ragged tails, several tiles) for parity cases."""
    return Workload(f"adhoc_{N}x{d}x{V}", N, d, V, w_std=w_std, labels=labels,
                    n_ignored=n_ignored, K=K, ref_eps_std=0.002 if K else 0.0,
                    index=seed - 1234)
