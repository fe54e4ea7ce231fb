"""The compute steps of the row data-parallel path restated from the oracle's definitions on
CPU (fp64), with the interface of lm_head_cross_tcgen05_b200.data_parallel's CudaOps. Test
infrastructure: it lets DataParallelCE's exchange logic run on CPU ranks over gloo and be
checked against the one-device oracle on the concatenated batch."""
from __future__ import annotations

import numpy as np
import torch

from oracle import lmh_oracle as O


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))


class DataParallelOracleOps:
    def count_valid(self, labels, V):
        valid, _ = O.valid_rows(labels, V)
        return torch.tensor([int(valid.sum())], dtype=torch.int32)

    def fused(self, H, W, labels, n_given, *, mode=O.BWD_CE, grad=None, weighted=False,
              mean=True, scalar_grad=False, chunk_rows=0, temperature=None, want_dH=True,
              bf16_dW=False):
        f = O.ce_forward(H, W, labels, temperature)
        N = f["z"].shape[0]
        n = int(n_given[0])
        # per-row weights are taken as given; the mean divides the unit weight or the scalar
        g = O.as_f64(grad).reshape(-1) if weighted else np.ones(1)
        if weighted and not scalar_grad:
            g = g.reshape(N)
        else:
            g = np.full(N, g[0] / n if n else 0.0) if mean else np.full(N, g[0])
        b = O.backward(mode if weighted else O.BWD_CE, H, W, labels, g, tau=temperature)
        out = dict(loss_rows=_t(f["loss_rows"]), lse=_t(f["lse"]), logprob=_t(f["logprob"]),
                   argmax=torch.from_numpy(f["argmax"]),
                   loss_mean=_t([f["loss_rows"].sum() / n if n else 0.0]),
                   dH=_t(b["dH"]) if want_dH else None)
        out["dW" if bf16_dW else "dW_part"] = _t(b["dW"])
        return out

    def sum_ranks(self, parts):
        out = parts[0].clone()
        for r in range(1, parts.shape[0]):
            out += parts[r]
        return out

    def reduce_rows(self, parts):
        out = parts[0].clone()
        for r in range(1, parts.shape[0]):
            out += parts[r]
        return out
