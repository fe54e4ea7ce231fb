"""Vocabulary-parallel cross entropy over the ranks of a torch.distributed process group.

Each of the R ranks holds a contiguous row range of W (its shard, from ``shard_plan``) and the
whole batch (H, labels). The pages run the head at tensor-parallel size 1 only
(miles-ext-kernels PR #14, lm_head op commit: the validate hook's startup checks). This module
splits the same definitions over ranks, with one exchange per direction:

forward
    every rank reduces each row over its shard to a 4-word record (``lmh_vp_partials``); the
    records are all-gathered in rank order (N x 16 bytes per rank) and every rank combines them
    in ascending rank order (``lmh_vp_combine``), so all ranks hold the same lse, loss,
    log-prob, argmax and mean.
backward
    every rank forms G on its shard with the combined lse and contracts it: from recomputed
    logits (``lmh_vp_loss_bwd``), or, in ``forward_backward``, from the softmax numerators its
    forward kept (``lmh_vp_fused_bwd``, one GEMM fewer). This gives the shard's dW (no
    exchange) and an fp32 contribution to dH. The
    contributions are summed in a fixed order: an all-to-all hands rank j the rows of slice j
    from every rank, rank j adds them in ascending rank order (``lmh_vp_reduce_rows``), and an
    all-gather returns the bf16 slices to every rank.

With a fixed R every result is bitwise reproducible: no floating-point value is reduced by a
collective, only moved.

``p2p=True`` fuses the dH exchange into the kernels instead of NCCL: the receive buffers and
every rank's dH live in symmetric memory (peer-mapped over NVLink); the dH GEMM's epilogue
writes each fp32 row straight into the receive buffer of the rank that reduces it while the
GEMM runs, and ``lmh_vp_reduce_rows_to`` stores each reduced bf16 slice into every rank's dH.
Stream-ordered barriers of the library (``lmh_peer_barrier``: signal words in symmetric memory,
a bounded wait that records a time-out instead of spinning) order the steps; the next step
reads that record on the host first and raises if a barrier gave up. The same fixed order of
additions gives the same bits as the NCCL path. The compute steps run in the library's CUDA kernels through
``CudaOps``; ``VocabParallelCE`` takes any object with the same four methods, which is how its
exchange logic is tested on CPU ranks.
"""
from __future__ import annotations

from typing import List, Optional, Tuple

import torch
import torch.distributed as dist

from . import (BWD_CE, BWD_SUPPORT_KL, ENTRY_VP_BWD, ENTRY_VP_COMBINE, ENTRY_VP_PARTIALS,
               ENTRY_VP_SUPPORT_BWD, ENTRY_VP_SUPPORT_COMBINE, ENTRY_VP_SUPPORT_PARTIALS,
               F_DW_ACC_GIVEN, F_FUSED_BWD, F_GRAD_SCALAR, F_MEAN, lmh_vp_combine,
               lmh_vp_fused_bwd, lmh_vp_loss_bwd, lmh_vp_partials, lmh_vp_reduce_rows,
               lmh_vp_reduce_rows_to, lmh_vp_support_bwd, lmh_vp_support_combine,
               lmh_vp_support_partials, make_shape, workspace)
from ._ranks import RankGroup, row_slices

__all__ = ["shard_plan", "row_slices", "CudaOps", "VocabParallelCE", "VocabParallelSupport"]


def shard_plan(V: int, R: int) -> List[Tuple[int, int]]:
    """The R contiguous vocabulary ranges [v0, v1) that cover [0, V), in rank order. Sizes are
    equal up to the last range, rounded up to the 256-wide logits tile when a range holds at
    least one tile; every range is non-empty (so V >= R is required)."""
    if R < 1 or V < R:
        raise ValueError(f"cannot split V={V} into {R} non-empty ranges")
    per = -(-V // R)
    if per >= 256:
        tiled = -(-per // 256) * 256
        if (R - 1) * tiled < V:  # every range keeps at least one word
            per = tiled
    return [(min(r * per, V), min((r + 1) * per, V)) for r in range(R)]


class CudaOps:
    """The library's vocabulary-parallel entries on CUDA tensors (outputs allocated here)."""

    def partials(self, H, W_shard, labels, v0, V_total, chunk_rows=0, temperature=None):
        N, d = H.shape
        shard = make_shape(N, d, W_shard.shape[0], 0, chunk_rows, 0, temperature)
        ws = workspace(shard, ENTRY_VP_PARTIALS, H.device)
        rec = torch.empty(N, 4, dtype=torch.float32, device=H.device)
        lmh_vp_partials(shard, v0, V_total, H, W_shard, labels, rec, workspace=ws)
        return rec

    def partials_fused(self, H, W_shard, labels, v0, V_total, mean=True, temperature=None):
        """partials() that also keeps p~ for fused_backward; all rows form one chunk."""
        N, d = H.shape
        flags = F_FUSED_BWD | (F_MEAN if mean else 0)
        shard = make_shape(N, d, W_shard.shape[0], 0, max(N, 1), flags, temperature)
        ws = workspace(shard, ENTRY_VP_PARTIALS, H.device)
        rec = torch.empty(N, 4, dtype=torch.float32, device=H.device)
        lmh_vp_partials(shard, v0, V_total, H, W_shard, labels, rec, workspace=ws)
        return rec, (shard, ws)

    def fused_backward(self, state, H, W_shard, labels, lse, v0, V_total, n_valid_given=None,
                       dW_acc=None, want_dW=True, dest=None):
        shard, ws = state
        N, d = H.shape
        dH_part = None if dest else torch.empty(N, d, dtype=torch.float32, device=H.device)
        dW = (torch.empty(W_shard.shape[0], d, dtype=torch.bfloat16, device=H.device)
              if want_dW else None)
        lmh_vp_fused_bwd(shard, v0, V_total, H, W_shard, labels, lse, n_valid_given, dH_part,
                         dW, dW_acc, dest, workspace=ws)
        return dH_part, dW

    def reduce_rows_to(self, parts, out_table, n_out, row_offset):
        lmh_vp_reduce_rows_to(parts, out_table, n_out, row_offset)

    def combine(self, records, labels, V_total, d, n_valid_given=None):
        R, N, _ = records.shape
        shape = make_shape(N, d, V_total, 0, 0, 0)
        ws = workspace(shape, ENTRY_VP_COMBINE, records.device)
        f32, dev = torch.float32, records.device
        out = dict(loss_rows=torch.empty(N, dtype=f32, device=dev),
                   lse=torch.empty(N, dtype=f32, device=dev),
                   logprob=torch.empty(N, dtype=f32, device=dev),
                   argmax=torch.empty(N, dtype=torch.int32, device=dev),
                   loss_mean=torch.empty(1, dtype=f32, device=dev),
                   n_valid=torch.empty(1, dtype=torch.int32, device=dev))
        lmh_vp_combine(shape, R, records, labels, out["loss_rows"], out["lse"], out["logprob"],
                       out["argmax"], out["loss_mean"], out["n_valid"], n_valid_given,
                       workspace=ws)
        return out

    def backward(self, mode, H, W_shard, labels, lse, grad, v0, V_total, chunk_rows=0,
                 mean=True, temperature=None, dW_acc=None, want_dW=True, dest=None):
        """(dH_part, dW); with dest = (receive-buffer table, R, rank) the dH rows are scattered
        to the reducing ranks instead and dH_part is None."""
        N, d = H.shape
        Vr = W_shard.shape[0]
        flags = (F_MEAN if mean else 0) | (F_DW_ACC_GIVEN if dW_acc is not None else 0)
        shard = make_shape(N, d, Vr, 0, chunk_rows, flags, temperature)
        ws = workspace(shard, ENTRY_VP_BWD, H.device)
        dH_part = None if dest else torch.empty(N, d, dtype=torch.float32, device=H.device)
        dW = torch.empty(Vr, d, dtype=torch.bfloat16, device=H.device) if want_dW else None
        lmh_vp_loss_bwd(shard, mode, v0, V_total, H, W_shard, labels, lse, grad, dH_part, dW,
                        dW_acc, dest, workspace=ws)
        return dH_part, dW

    def reduce_rows(self, parts):
        out = torch.empty(parts.shape[1], parts.shape[2], dtype=torch.bfloat16,
                          device=parts.device)
        lmh_vp_reduce_rows(parts, out)
        return out

    # support entries: records [N, K + 1] (lse_r, then the candidates' logits or -inf)
    def support_partials(self, H, W_shard, ids, v0, V_total, chunk_rows=0, temperature=None):
        N, d = H.shape
        K = ids.shape[1]
        shard = make_shape(N, d, W_shard.shape[0], K, chunk_rows, 0, temperature)
        ws = workspace(shard, ENTRY_VP_SUPPORT_PARTIALS, H.device)
        rec = torch.empty(N, K + 1, dtype=torch.float32, device=H.device)
        lmh_vp_support_partials(shard, v0, V_total, H, W_shard, ids, rec, workspace=ws)
        return rec

    def support_combine(self, records, ids, ref_logp, V_total, d):
        R, N, _ = records.shape
        K = ids.shape[1]
        shape = make_shape(N, d, V_total, K, 0, 0)
        ws = workspace(shape, ENTRY_VP_SUPPORT_COMBINE, records.device)
        f32, dev = torch.float32, records.device
        out = dict(lp=torch.empty(N, K, dtype=f32, device=dev),
                   lse=torch.empty(N, dtype=f32, device=dev))
        if ref_logp is not None:
            out["kl_rows"] = torch.empty(N, dtype=f32, device=dev)
            out["kl_mean"] = torch.empty(1, dtype=f32, device=dev)
        lmh_vp_support_combine(shape, R, records, ids, ref_logp, out["lp"], out["lse"],
                               out.get("kl_rows"), out.get("kl_mean"), workspace=ws)
        return out

    def support_backward(self, mode, H, W_shard, ids, lse, grad, ref_logp, v0, V_total,
                         chunk_rows=0, mean=True, temperature=None, dW_acc=None, want_dW=True,
                         dest=None, scalar_grad=False):
        N, d = H.shape
        Vr, K = W_shard.shape[0], ids.shape[1]
        flags = ((F_MEAN if mean else 0) | (F_DW_ACC_GIVEN if dW_acc is not None else 0)
                 | (F_GRAD_SCALAR if scalar_grad else 0))
        shard = make_shape(N, d, Vr, K, chunk_rows, flags, temperature)
        ws = workspace(shard, ENTRY_VP_SUPPORT_BWD, H.device)
        dH_part = None if dest else torch.empty(N, d, dtype=torch.float32, device=H.device)
        dW = torch.empty(Vr, d, dtype=torch.bfloat16, device=H.device) if want_dW else None
        lmh_vp_support_bwd(shard, mode, v0, V_total, H, W_shard, ids, lse, grad, ref_logp,
                           dH_part, dW, dW_acc, dest, workspace=ws)
        return dH_part, dW


class _VocabParallel(RankGroup):
    """The shard plan of ``group``'s ranks and the exchange steps every vocabulary-parallel
    objective shares: gathering per-row records, and summing the ranks' dH contributions in
    a fixed order (collectives, or peer-memory stores with ``p2p``). Without an initialised
    process group it runs as the only rank (R = 1, no collective)."""

    def __init__(self, V_total: int, group=None, chunk_rows: int = 0, mean: bool = True,
                 temperature=None, ops=None, p2p: bool = False):
        super().__init__(group, ops if ops is not None else CudaOps())
        self.V_total = int(V_total)
        self.v0, self.v1 = shard_plan(self.V_total, self.R)[self.rank]
        self.chunk_rows = chunk_rows
        self.mean = mean
        self.temperature = temperature
        self.p2p = p2p and self.R > 1   # one rank has nothing to exchange

    def _check_shard(self, W_shard):
        if W_shard.shape[0] != self.v1 - self.v0:
            raise ValueError(f"rank {self.rank} holds rows [{self.v0}, {self.v1}) of W, "
                             f"got {W_shard.shape[0]} rows")

    def _dH(self, run, N, d, device):
        """dH summed over the ranks from run(dest) -> (dH_part or None, dW): collectives, or
        with p2p the rows scattered straight to their reducing ranks."""
        if self.p2p:
            sym = self._open_p2p(N, d, device)
            _, dW = run((sym["recv_tab"], self.R, self.rank))
            return self._reduce_p2p(sym), dW
        dH_part, dW = run(None)
        return self._sum_rows(dH_part), dW


class VocabParallelCE(_VocabParallel):
    """Cross entropy (and the per-row log-prob objective) with W split over the ranks of
    ``group``. Every rank calls ``forward`` and ``backward`` (or ``forward_backward``) with its
    own shard ``W[v0:v1]`` (``self.v0``, ``self.v1``) and the same H, labels and options."""

    def forward(self, H, W_shard, labels, n_valid_given=None) -> dict:
        """loss_rows, lse, logprob, argmax, loss_mean, n_valid: the same on every rank."""
        self._check_shard(W_shard)
        rec = self.ops.partials(H, W_shard, labels, self.v0, self.V_total, self.chunk_rows,
                                self.temperature)
        return self.ops.combine(self._gather(rec), labels, self.V_total, H.shape[1],
                                n_valid_given)

    def forward_backward(self, H, W_shard, labels, n_valid_given=None,
                         dW_acc: Optional[torch.Tensor] = None, want_dW: bool = True) -> dict:
        """forward() plus dH and this rank's dW of the loss (mean or sum), in one pass: the
        backward reuses the forward's softmax numerators instead of recomputing the logits.
        All rows form one chunk (chunk_rows is not used)."""
        self._check_shard(W_shard)
        N, d = H.shape
        rec, state = self.ops.partials_fused(H, W_shard, labels, self.v0, self.V_total,
                                             self.mean, self.temperature)
        out = self.ops.combine(self._gather(rec), labels, self.V_total, d, n_valid_given)
        out["dH"], out["dW"] = self._dH(
            lambda dest: self.ops.fused_backward(state, H, W_shard, labels, out["lse"], self.v0,
                                                 self.V_total, n_valid_given, dW_acc, want_dW,
                                                 dest=dest), N, d, H.device)
        return out

    def backward(self, H, W_shard, labels, lse, grad=None, mode: int = BWD_CE,
                 dW_acc: Optional[torch.Tensor] = None, want_dW: bool = True) -> dict:
        """dH [N, d] (the same on every rank) and this rank's dW shard [v1 - v0, d]."""
        self._check_shard(W_shard)
        N, d = H.shape
        dH, dW = self._dH(
            lambda dest: self.ops.backward(mode, H, W_shard, labels, lse, grad, self.v0,
                                           self.V_total, self.chunk_rows, self.mean,
                                           self.temperature, dW_acc, want_dW, dest=dest),
            N, d, H.device)
        return dict(dH=dH, dW=dW)


class VocabParallelSupport(_VocabParallel):
    """The support-set entries with W split over the ranks: log-probs at K candidate ids per
    row (full-vocabulary normaliser) and the KL against reference log-probs, and the backward of
    sum_ik g_ik lp_ik (BWD_SUPPORT_LOGPROB) or of the (mean) KL (BWD_SUPPORT_KL). Each rank
    reports its lse and the logits of the candidates in its shard (K + 1 floats per row)."""

    def forward(self, H, W_shard, ids, ref_logp=None) -> dict:
        """lp [N, K], lse [N] (and kl_rows, kl_mean with ref_logp): the same on every rank."""
        self._check_shard(W_shard)
        rec = self.ops.support_partials(H, W_shard, ids, self.v0, self.V_total, self.chunk_rows,
                                        self.temperature)
        return self.ops.support_combine(self._gather(rec), ids, ref_logp, self.V_total,
                                        H.shape[1])

    def backward(self, H, W_shard, ids, lse, mode: int = BWD_SUPPORT_KL, grad=None,
                 ref_logp=None, dW_acc: Optional[torch.Tensor] = None,
                 want_dW: bool = True, scalar_grad: bool = False) -> dict:
        """dH [N, d] (the same on every rank) and this rank's dW shard."""
        self._check_shard(W_shard)
        N, d = H.shape
        dH, dW = self._dH(
            lambda dest: self.ops.support_backward(mode, H, W_shard, ids, lse, grad, ref_logp,
                                                   self.v0, self.V_total, self.chunk_rows,
                                                   self.mean, self.temperature, dW_acc, want_dW,
                                                   dest=dest, scalar_grad=scalar_grad),
            N, d, H.device)
        return dict(dH=dH, dW=dW)
