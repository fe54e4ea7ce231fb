"""torch.autograd entry points over the library's entries, for training code that calls
``loss.backward()``.

The pages' training integration exposes the head as an autograd function whose entry point
returns per-row log-probabilities (miles-ext-kernels PR #14, lm_head op commit: ``log_probs``,
its backward run by the same package as the forward). These functions do the same with this
library: the forward runs a forward entry and keeps the per-row lse; the backward runs
``lmh_loss_bwd`` with the upstream gradient, recomputing the logits chunk by chunk. The
upstream gradient of a reduced loss stays on the device (``LMH_F_GRAD_SCALAR``), so no call
synchronises the host. All arithmetic runs in the library's kernels.

For a step whose loss is final (gradient 1), ``loss_fwd(..., grads=True)`` does forward and
backward in one pass and saves one of the four GEMMs; these functions suit graphs where the
head's output feeds further computation.
"""
from __future__ import annotations

import torch

from . import (BWD_CE, BWD_LOGPROB, BWD_SUPPORT_KL, BWD_SUPPORT_LOGPROB, logprob, loss_bwd,
               loss_fwd, support_kl as _support_kl, support_logprob as _support_logprob)

__all__ = ["log_probs", "cross_entropy", "support_log_probs", "support_kl"]


def _grads(ctx, mode, targets, g, ref=None, *, mean=False, scalar=False, renorm=False):
    H, W, lse = ctx.saved_tensors[:3]
    out = loss_bwd(mode, H, W, targets, lse, g.contiguous().float(), ref,
                   chunk_rows=ctx.chunk_rows, want_dH=ctx.needs_input_grad[0],
                   want_dW=ctx.needs_input_grad[1], temperature=ctx.temperature, mean=mean,
                   renorm=renorm, scalar_grad=scalar)
    return out["dH"], out["dW"]


class _LogProbs(torch.autograd.Function):
    @staticmethod
    def forward(ctx, H, W, labels, chunk_rows, temperature):
        out = logprob(H, W, labels, chunk_rows=chunk_rows, temperature=temperature)
        ctx.chunk_rows, ctx.temperature = chunk_rows, temperature
        ctx.save_for_backward(H, W, out["lse"], labels)
        return out["logprob"]

    @staticmethod
    def backward(ctx, g):
        labels = ctx.saved_tensors[3]
        dH, dW = _grads(ctx, BWD_LOGPROB, labels, g)
        return dH, dW, None, None, None


def log_probs(H, W, labels, *, chunk_rows: int = 0, temperature=None) -> torch.Tensor:
    """Per-row target log-probability [N] (0 for ignored rows), differentiable in H and W."""
    return _LogProbs.apply(H, W, labels, chunk_rows, temperature)


class _CrossEntropy(torch.autograd.Function):
    @staticmethod
    def forward(ctx, H, W, labels, reduction, chunk_rows, temperature):
        one = None
        if reduction == "sum":  # the entry's mean divides by a given count: give it 1
            one = torch.ones(1, dtype=torch.int32, device=H.device)
        out = loss_fwd(H, W, labels, chunk_rows=chunk_rows, n_valid_given=one,
                       temperature=temperature)
        ctx.chunk_rows, ctx.temperature, ctx.reduction = chunk_rows, temperature, reduction
        ctx.save_for_backward(H, W, out["lse"], labels)
        return out["loss_rows"] if reduction == "none" else out["loss_mean"].view(())

    @staticmethod
    def backward(ctx, g):
        labels = ctx.saved_tensors[3]
        if ctx.reduction == "none":
            dH, dW = _grads(ctx, BWD_CE, labels, g)
        else:
            dH, dW = _grads(ctx, BWD_CE, labels, g.reshape(1), mean=ctx.reduction == "mean",
                            scalar=True)
        return dH, dW, None, None, None, None


def cross_entropy(H, W, labels, *, reduction: str = "mean", chunk_rows: int = 0,
                  temperature=None) -> torch.Tensor:
    """Cross entropy of logits H W^T against labels (negative labels ignored): per row
    (reduction="none"), summed, or averaged over the valid rows, differentiable in H and W."""
    if reduction not in ("none", "mean", "sum"):
        raise ValueError(f"reduction must be none, mean or sum, got {reduction!r}")
    return _CrossEntropy.apply(H, W, labels, reduction, chunk_rows, temperature)


class _SupportLogProbs(torch.autograd.Function):
    @staticmethod
    def forward(ctx, H, W, ids, chunk_rows, temperature, renorm):
        out = _support_logprob(H, W, ids, chunk_rows=chunk_rows, temperature=temperature,
                               renorm=renorm)
        ctx.chunk_rows, ctx.temperature, ctx.renorm = chunk_rows, temperature, renorm
        ctx.save_for_backward(H, W, out["lse"], ids)
        return out["lp"]

    @staticmethod
    def backward(ctx, g):
        ids = ctx.saved_tensors[3]
        dH, dW = _grads(ctx, BWD_SUPPORT_LOGPROB, ids, g, renorm=ctx.renorm)
        return dH, dW, None, None, None, None


def support_log_probs(H, W, ids, *, chunk_rows: int = 0, temperature=None,
                      renorm: bool = False) -> torch.Tensor:
    """Log-probabilities [N, K] at K candidate ids per row (full-vocabulary normaliser, or the
    candidates' own with renorm=True), differentiable in H and W."""
    return _SupportLogProbs.apply(H, W, ids, chunk_rows, temperature, renorm)


class _SupportKL(torch.autograd.Function):
    @staticmethod
    def forward(ctx, H, W, ids, ref_logp, reduction, chunk_rows, temperature, renorm):
        out = _support_kl(H, W, ids, ref_logp, chunk_rows=chunk_rows, temperature=temperature,
                          renorm=renorm)
        ctx.chunk_rows, ctx.temperature, ctx.renorm = chunk_rows, temperature, renorm
        ctx.reduction = reduction
        ctx.save_for_backward(H, W, out["lse"], ids, ref_logp)
        return out["kl_rows"] if reduction == "none" else out["kl_mean"].view(())

    @staticmethod
    def backward(ctx, g):
        ids, ref = ctx.saved_tensors[3], ctx.saved_tensors[4]
        if ctx.reduction == "none":
            dH, dW = _grads(ctx, BWD_SUPPORT_KL, ids, g, ref, renorm=ctx.renorm)
        else:
            dH, dW = _grads(ctx, BWD_SUPPORT_KL, ids, g.reshape(1), ref, mean=True, scalar=True,
                            renorm=ctx.renorm)
        return dH, dW, None, None, None, None, None, None


def support_kl(H, W, ids, ref_logp, *, reduction: str = "mean", chunk_rows: int = 0,
               temperature=None, renorm: bool = False) -> torch.Tensor:
    """KL(ref || model) over each row's candidates: per row (reduction="none") or the mean
    over all rows, differentiable in H and W."""
    if reduction not in ("none", "mean"):
        raise ValueError(f"reduction must be none or mean, got {reduction!r}")
    return _SupportKL.apply(H, W, ids, ref_logp, reduction, chunk_rows, temperature, renorm)
