"""torch.autograd entry points over the library's entries, for training code that calls
``loss.backward()``.

The pages' training integration exposes the head as an autograd function whose entry point
returns per-row log-probabilities (miles-ext-kernels PR #14, lm_head op commit: ``log_probs``,
its backward run by the same package as the forward). These functions do the same with this
library, in one of two ways:

* per-row outputs (``log_probs``, ``cross_entropy(reduction="none")``, ``support_log_probs``,
  ``support_kl(reduction="none")``): the upstream gradient is a row vector known only in the
  backward, so the forward keeps lse and the backward runs ``lmh_loss_bwd``, recomputing the
  logits chunk by chunk (four GEMMs per step);
* reduced losses (``cross_entropy`` with "mean" or "sum", ``support_kl`` with "mean"): the
  gradient is the one for g = 1 times the scalar upstream g, so the forward already runs the
  one-pass entry (``lmh_loss_fwd`` with dH / dW, ``lmh_support_kl_fwd_bwd``: three GEMMs) and
  keeps dH and dW, and the backward scales them by g on the device (``lmh_scale_bf16``; g = 1
  changes no bit). They hold dH and dW from the forward to the backward, like activations.

No call synchronises the host, and all arithmetic runs in the library's kernels.
"""
from __future__ import annotations

import torch

from . import (BWD_CE, BWD_LOGPROB, BWD_SUPPORT_KL, BWD_SUPPORT_LOGPROB, lmh_scale_bf16,
               logprob, loss_bwd, loss_fwd, support_kl as _support_kl,
               support_logprob as _support_logprob)

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


def _scaled(ctx, g):
    """The one-pass gradients of the forward, times the scalar upstream gradient g."""
    g = g.reshape(1).contiguous().float()
    out = []
    for t in (ctx.dH, ctx.dW):
        if t is not None:
            lmh_scale_bf16(t, g)
        out.append(t)
    ctx.dH = ctx.dW = None
    return out


class _CrossEntropy(torch.autograd.Function):
    @staticmethod
    def forward(ctx, H, W, labels, reduction, chunk_rows, temperature):
        one = None
        if reduction == "sum":  # the entry's mean divides by a given count: give it 1
            one = torch.ones(1, dtype=torch.int32, device=H.device)
        ctx.chunk_rows, ctx.temperature, ctx.reduction = chunk_rows, temperature, reduction
        fused = reduction != "none" and (ctx.needs_input_grad[0] or ctx.needs_input_grad[1])
        out = loss_fwd(H, W, labels, chunk_rows=chunk_rows, n_valid_given=one,
                       temperature=temperature, grads=fused, mean=reduction == "mean",
                       want_dH=ctx.needs_input_grad[0], want_dW=ctx.needs_input_grad[1])
        ctx.dH, ctx.dW = (out.get("dH"), out.get("dW")) if fused else (None, None)
        if not fused:
            ctx.save_for_backward(H, W, out["lse"], labels)
        if reduction == "none":
            return out["loss_rows"]
        return out["loss_mean"].view(())

    @staticmethod
    def backward(ctx, g):
        if ctx.reduction == "none":
            dH, dW = _grads(ctx, BWD_CE, ctx.saved_tensors[3], g)
        else:
            dH, dW = _scaled(ctx, g)
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
        ctx.chunk_rows, ctx.temperature, ctx.renorm = chunk_rows, temperature, renorm
        ctx.reduction = reduction
        # the one-pass entry covers the full-vocabulary reading; the renormalised one's
        # backward is a sparse gather / scatter with no logits GEMM to save
        fused = (reduction == "mean" and not renorm
                 and (ctx.needs_input_grad[0] or ctx.needs_input_grad[1]))
        out = _support_kl(H, W, ids, ref_logp, chunk_rows=chunk_rows, temperature=temperature,
                          renorm=renorm, grads=fused)
        ctx.dH = out.get("dH") if fused and ctx.needs_input_grad[0] else None
        ctx.dW = out.get("dW") if fused and ctx.needs_input_grad[1] else None
        if not fused:
            ctx.save_for_backward(H, W, out["lse"], ids, ref_logp)
        return out["kl_rows"] if reduction == "none" else out["kl_mean"].view(())

    @staticmethod
    def backward(ctx, g):
        if ctx.reduction != "none" and (ctx.dH is not None or ctx.dW is not None):
            dH, dW = _scaled(ctx, g)
            return dH, dW, None, None, None, None, None, None
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
