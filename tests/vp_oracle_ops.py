"""The four compute steps of the vocabulary-parallel path restated from the oracle's
definitions on CPU (fp64), with the interface of lm_head_cross_tcgen05_b200.vocab_parallel's
CudaOps. Test infrastructure: it lets the exchange logic of VocabParallelCE run on CPU ranks
over gloo and be checked against the one-device oracle."""
from __future__ import annotations

import numpy as np
import torch

from oracle import lmh_oracle as O


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))


class OracleOps:
    def partials(self, H, W_shard, labels, v0, V_total, chunk_rows=0, temperature=None):
        z = O.logits(H, W_shard, temperature)                     # [N, V_r], tempered
        y = O.as_i64(labels)
        lse = O.logsumexp_rows(z)
        arg = z.argmax(axis=1)                                     # first maximum
        loc = y - v0
        inside = (loc >= 0) & (loc < z.shape[1])
        zy = np.where(inside, z[np.arange(len(y)), np.clip(loc, 0, z.shape[1] - 1)], -np.inf)
        return _t(np.stack([lse, z.max(axis=1), arg + v0, zy], axis=1))

    def combine(self, records, labels, V_total, d, n_valid_given=None):
        r = records.numpy()                                         # [R, N, 4]
        lse = np.logaddexp.reduce(r[:, :, 0], axis=0)
        best = r[:, :, 1].argmax(axis=0)                            # first rank on ties
        arg = r[best, np.arange(r.shape[1]), 2].astype(np.int64)
        zy = r[:, :, 3].max(axis=0)
        y = O.as_i64(labels)
        valid = (y >= 0) & (y < V_total)
        loss = np.where(valid, lse - zy, 0.0)
        n = int(valid.sum()) if n_valid_given is None else int(n_valid_given)
        return dict(loss_rows=_t(loss), lse=_t(lse), logprob=_t(-loss),
                    argmax=torch.from_numpy(arg), loss_mean=_t([loss.sum() / n if n else 0.0]),
                    n_valid=torch.tensor([int(valid.sum())]))

    def backward(self, mode, H, W_shard, labels, lse, grad, v0, V_total, chunk_rows=0,
                 mean=True, temperature=None, dW_acc=None, want_dW=True, dest=None):
        z = O.logits(H, W_shard, temperature)
        N, Vr = z.shape
        y = O.as_i64(labels)
        valid = (y >= 0) & (y < V_total)
        if grad is None:
            n = int(valid.sum())
            g = np.full(N, (1.0 / n if n else 0.0) if mean else 1.0)
        else:
            g = O.as_f64(grad).reshape(N)
        g = np.where(valid, g, 0.0) * (1.0 if mode == 0 else -1.0)
        G = g[:, None] * np.exp(z - O.as_f64(lse)[:, None])
        loc = y - v0
        hit = valid & (loc >= 0) & (loc < Vr)
        G[np.nonzero(hit)[0], loc[hit]] -= g[hit]
        G = G / O.tau_rows(temperature, N)[:, None]
        dH, dW = O.lm_head_backward(H, W_shard, G)
        return _t(dH), (_t(dW) if want_dW else None)

    def partials_fused(self, H, W_shard, labels, v0, V_total, mean=True, temperature=None):
        return self.partials(H, W_shard, labels, v0, V_total, 0, temperature), \
            dict(mean=mean, temperature=temperature)

    def fused_backward(self, state, H, W_shard, labels, lse, v0, V_total, n_valid_given=None,
                       dW_acc=None, want_dW=True, dest=None):
        grad = None
        if n_valid_given is not None:
            n = int(n_valid_given)
            grad = np.full(len(O.as_i64(labels)), (1.0 / n if n else 0.0) if state["mean"] else 1.0)
        return self.backward(0, H, W_shard, labels, lse, grad, v0, V_total, 0, state["mean"],
                             state["temperature"], dW_acc, want_dW)

    # support entries
    def support_partials(self, H, W_shard, ids, v0, V_total, chunk_rows=0, temperature=None):
        z = O.logits(H, W_shard, temperature)
        c = O.as_i64(ids)
        loc = c - v0
        inside = (loc >= 0) & (loc < z.shape[1])
        zc = np.where(inside, z[np.arange(z.shape[0])[:, None], np.clip(loc, 0, z.shape[1] - 1)],
                      -np.inf)
        return _t(np.concatenate([O.logsumexp_rows(z)[:, None], zc], axis=1))

    def support_combine(self, records, ids, ref_logp, V_total, d):
        r = records.numpy()
        lse = np.logaddexp.reduce(r[:, :, 0], axis=0)
        z = r[:, :, 1:].max(axis=0)
        c = O.as_i64(ids)
        ok = (c >= 0) & (c < V_total)
        lp = np.where(ok, z - lse[:, None], 0.0)
        out = dict(lp=_t(lp), lse=_t(lse))
        if ref_logp is not None:
            rr = O.as_f64(ref_logp).reshape(c.shape)
            kl = np.where(ok, np.exp(rr) * (rr - lp), 0.0).sum(axis=1)
            out.update(kl_rows=_t(kl), kl_mean=_t([kl.sum() / len(kl)]))
        return out

    def support_backward(self, mode, H, W_shard, ids, lse, grad, ref_logp, v0, V_total,
                         chunk_rows=0, mean=True, temperature=None, dW_acc=None, want_dW=True,
                         dest=None, scalar_grad=False):
        z = O.logits(H, W_shard, temperature)
        N, Vr = z.shape
        c = O.as_i64(ids)
        K = c.shape[1]
        ok = (c >= 0) & (c < V_total)
        unit = (1.0 / N if N else 0.0) if mean else 1.0
        if mode == 2:   # sum_ik g_ik lp_ik
            g = np.full((N, K), unit) if grad is None else O.as_f64(grad).reshape(N, K)
            w = -g
        else:           # sum_i g_i KL_i
            g = np.full(N, unit) if grad is None else O.as_f64(grad).reshape(N)
            w = g[:, None] * np.exp(O.as_f64(ref_logp).reshape(N, K))
        w = np.where(ok, w, 0.0)
        P = np.exp(z - O.as_f64(lse)[:, None])
        G = w.sum(axis=1)[:, None] * P
        loc = c - v0
        hit = ok & (loc >= 0) & (loc < Vr)
        for i, k in zip(*np.nonzero(hit)):
            G[i, loc[i, k]] -= w[i, k]
        G = G / O.tau_rows(temperature, N)[:, None]
        dH, dW = O.lm_head_backward(H, W_shard, G)
        return _t(dH), (_t(dW) if want_dW else None)

    def reduce_rows(self, parts):
        out = parts[0].clone()
        for r in range(1, parts.shape[0]):
            out += parts[r]
        return out
