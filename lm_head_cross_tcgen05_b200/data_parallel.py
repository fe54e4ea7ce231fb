"""Row data-parallel cross entropy over the ranks of a torch.distributed process group.

Every rank holds all of W and its own rows of the batch (H_r, labels_r; the row counts may
differ). The objective is the one a single device computes on the concatenated batch: the mean
loss divides by the valid rows of ALL ranks, and dW is the sum over the ranks. The pages' ops
sum a weight gradient over the rows of one call and leave its reduction across ranks to the
caller (miles-ext-kernels PR #14, gated RMSNorm commit notes); this module does that reduction
in a fixed order, so the result is bitwise reproducible for a given rank count and batch split:

1. ``lmh_count_valid`` counts the rank's valid rows; an integer all-reduce gives the global
   count (exact in any order).
2. The one-pass entry (``lmh_loss_fwd`` with dH and dW, or ``lmh_loss_fwd_bwd`` for weighted
   objectives) runs on the rank's rows with that count as ``n_valid_given`` and writes the
   rank's fp32 dW into a buffer it overwrites (``LMH_F_DW_ACC_STORE``). Its ``loss_mean`` is
   the rank's share of the global mean; dH is already final (each row's gradient depends on
   that row only, plus the global count).
3. The R shares of the mean are gathered and added in rank order (``lmh_reduce_ranks_f32``);
   the fp32 dW are summed in rank order by row slices: an all-to-all hands rank j the rows of
   slice j from every rank, ``lmh_vp_reduce_rows`` adds them, and an all-gather returns the
   bf16 slices to every rank.

With ``p2p=True`` the dW exchange runs over peer memory instead of NCCL: the receive buffers
and every rank's dW live in symmetric memory (peer-mapped over NVLink), the dW GEMM's epilogue
stores each fp32 row straight into the receive buffer of the rank that reduces it while the
GEMM runs (``lmh_dp_loss_fwd_bwd``), and ``lmh_vp_reduce_rows_to`` stores each reduced bf16
slice into every rank's dW. The library's bounded peer-memory barrier (``lmh_peer_barrier``)
orders the steps, and each step first checks on the host that the previous step's barriers
did not time out. The additions are the same, so the bits are the same. All rows of a rank
then form one chunk, so the workspace holds the softmax buffer of all of them
(rows x round_up(V, 8) x 2 bytes); ``chunk_rows`` cannot be combined with ``p2p``.

Against one device on the concatenated batch the values agree to fp32 rounding (the dW sum and
the mean are grouped by rank). The compute steps run in the library's CUDA kernels through
``CudaOps``; ``DataParallelCE`` takes any object with the same methods, which is how its
exchange logic is tested on CPU ranks.
"""
from __future__ import annotations

import torch

from . import (BWD_CE, ENTRY_LOSS_FWD, ENTRY_LOSS_FWD_BWD, F_DW_ACC_GIVEN, F_DW_ACC_STORE,
               F_FUSED_BWD, F_GRAD_SCALAR, F_MEAN, lmh_count_valid, lmh_dp_loss_fwd_bwd,
               lmh_loss_fwd, lmh_loss_fwd_bwd, lmh_reduce_ranks_f32, lmh_vp_reduce_rows,
               lmh_vp_reduce_rows_to, make_shape, workspace)
from ._ranks import RankGroup

__all__ = ["CudaOps", "DataParallelCE"]


class CudaOps:
    """The library's entries for the data-parallel step on CUDA tensors (outputs allocated
    here)."""

    def count_valid(self, labels, V):
        n = torch.empty(1, dtype=torch.int32, device=labels.device)
        lmh_count_valid(labels, V, n)
        return n

    def fused(self, H, W, labels, n_given, *, mode=BWD_CE, grad=None, weighted=False,
              mean=True, scalar_grad=False, chunk_rows=0, temperature=None, want_dH=True,
              bf16_dW=False):
        """Forward outputs, dH (nullable) and the rank's fp32 dW ``dW_part`` in one pass; with
        bf16_dW its bf16 cast ``dW`` instead (the same bits as casting dW_part)."""
        N, d = H.shape
        V = W.shape[0]
        dev = H.device
        acc = 0 if bf16_dW else F_DW_ACC_GIVEN | F_DW_ACC_STORE
        flags = (F_FUSED_BWD | acc | (F_MEAN if mean else 0)
                 | (F_GRAD_SCALAR if scalar_grad else 0))
        shape = make_shape(N, d, V, 0, chunk_rows, flags, temperature)
        f32 = torch.float32
        out = dict(loss_rows=torch.empty(N, dtype=f32, device=dev),
                   lse=torch.empty(N, dtype=f32, device=dev),
                   logprob=torch.empty(N, dtype=f32, device=dev),
                   argmax=torch.empty(N, dtype=torch.int32, device=dev),
                   loss_mean=torch.empty(1, dtype=f32, device=dev),
                   dH=torch.empty(N, d, dtype=torch.bfloat16, device=dev) if want_dH else None)
        if bf16_dW:
            out["dW"] = torch.empty(V, d, dtype=torch.bfloat16, device=dev)
        else:
            out["dW_part"] = torch.empty(V, d, dtype=f32, device=dev)
        dW, acc_t = out.get("dW"), out.get("dW_part")
        if weighted:
            ws = workspace(shape, ENTRY_LOSS_FWD_BWD, dev)
            lmh_loss_fwd_bwd(shape, mode, H, W, labels, grad, out["loss_rows"], out["lse"],
                             out["logprob"], out["argmax"], out["loss_mean"], None, n_given,
                             out["dH"], dW, acc_t, workspace=ws)
        else:
            ws = workspace(shape, ENTRY_LOSS_FWD, dev)
            lmh_loss_fwd(shape, H, W, labels, out["loss_rows"], out["lse"], out["logprob"],
                         out["argmax"], out["loss_mean"], None, n_given, out["dH"], dW, acc_t,
                         workspace=ws)
        out["workspace"] = ws
        return out

    def fused_scatter(self, H, W, labels, n_given, dest, *, mode=BWD_CE, grad=None,
                      mean=True, scalar_grad=False, temperature=None, want_dH=True):
        """fused() whose dW GEMM stores the rank's fp32 dW rows into the reducing ranks'
        receive buffers (dest = (address table, R, rank)); all rows form one chunk."""
        N, d = H.shape
        V = W.shape[0]
        dev = H.device
        flags = F_FUSED_BWD | (F_MEAN if mean else 0) | (F_GRAD_SCALAR if scalar_grad else 0)
        shape = make_shape(N, d, V, 0, max(N, 1), flags, temperature)
        f32 = torch.float32
        out = dict(loss_rows=torch.empty(N, dtype=f32, device=dev),
                   lse=torch.empty(N, dtype=f32, device=dev),
                   logprob=torch.empty(N, dtype=f32, device=dev),
                   argmax=torch.empty(N, dtype=torch.int32, device=dev),
                   loss_mean=torch.empty(1, dtype=f32, device=dev),
                   dH=torch.empty(N, d, dtype=torch.bfloat16, device=dev) if want_dH else None)
        ws = workspace(shape, ENTRY_LOSS_FWD_BWD, dev)
        lmh_dp_loss_fwd_bwd(shape, mode, H, W, labels, grad, out["loss_rows"], out["lse"],
                            out["logprob"], out["argmax"], out["loss_mean"], n_given, out["dH"],
                            dest, workspace=ws)
        out["workspace"] = ws
        return out

    def reduce_rows_to(self, parts, out_table, n_out, row_offset):
        lmh_vp_reduce_rows_to(parts, out_table, n_out, row_offset)

    def sum_ranks(self, parts):
        out = torch.empty(parts.shape[1], dtype=torch.float32, device=parts.device)
        lmh_reduce_ranks_f32(parts, out)
        return out

    def reduce_rows(self, parts):
        out = torch.empty(parts.shape[1], parts.shape[2], dtype=torch.bfloat16,
                          device=parts.device)
        lmh_vp_reduce_rows(parts, out)
        return out


class DataParallelCE(RankGroup):
    """Cross entropy of the concatenated batch with its rows split over the ranks of
    ``group``. Every rank calls ``forward_backward`` with its own rows and the full W.

    mean=True: the gradient is of the mean loss over the valid rows of all ranks; False: of
    the summed loss. ``loss_mean`` is the global mean in both cases, ``n_valid`` the global
    count. With ``grad`` (and ``mode``) the gradient is instead that of the weighted objective
    of ``lmh_loss_fwd_bwd``: sum_i w_i l_i over all ranks' rows, with w_i = this rank's
    ``grad[i]`` taken as given, or with ``scalar_grad`` one upstream gradient g for every
    row (divided by the global count with mean=True). ``count`` gives the global count
    before the step, for callers whose per-row weights depend on it. With ``p2p`` (and more
    than one rank) dW is exchanged over peer memory and each rank's rows form one chunk, so
    ``chunk_rows`` must stay 0 (a ValueError otherwise)."""

    def __init__(self, group=None, chunk_rows: int = 0, mean: bool = True, temperature=None,
                 ops=None, p2p: bool = False):
        super().__init__(group, ops if ops is not None else CudaOps())
        self.chunk_rows = chunk_rows
        self.mean = mean
        self.temperature = temperature
        self.p2p = p2p and self.R > 1   # one rank has nothing to exchange
        if self.p2p and chunk_rows:
            raise ValueError("p2p runs each rank's rows as one chunk: chunk_rows cannot be set "
                             "(the workspace holds rows x round_up(V, 8) x 2 bytes of softmax)")

    def count(self, labels, V: int):
        """The valid rows (0 <= label < V) of all ranks: a one-element int32 device tensor."""
        return self._count_sum(self.ops.count_valid(labels, V))

    def forward_backward(self, H, W, labels, grad=None, mode: int = BWD_CE,
                         scalar_grad: bool = False, want_dH: bool = True) -> dict:
        """loss_rows, lse, logprob, argmax, dH: this rank's rows; loss_mean, n_valid and dW
        [V, d] bf16: the same on every rank."""
        n = self.count(labels, W.shape[0])
        if self.p2p:
            V, d = W.shape
            sym = self._open_p2p(V, d, H.device)
            out = self.ops.fused_scatter(H, W, labels, n, (sym["recv_tab"], self.R, self.rank),
                                         mode=mode, grad=grad, mean=self.mean,
                                         scalar_grad=scalar_grad,
                                         temperature=self.temperature, want_dH=want_dH)
            out["dW"] = self._reduce_p2p(sym)
        else:
            # one rank has nothing to add: its bf16 dW comes straight from the GEMM's fp32
            # tile sums, the bits the rank-ordered sum of one fp32 part would give
            out = self.ops.fused(H, W, labels, n, mode=mode, grad=grad,
                                 weighted=grad is not None, mean=self.mean,
                                 scalar_grad=scalar_grad, chunk_rows=self.chunk_rows,
                                 temperature=self.temperature, want_dH=want_dH,
                                 bf16_dW=self.R == 1)
            if self.R > 1:
                out["dW"] = self._sum_rows(out.pop("dW_part"))
        if self.R > 1:
            shares = self._gather(out["loss_mean"].reshape(1, 1)).reshape(self.R, 1)
            out["loss_mean"] = self.ops.sum_ranks(shares)
        out["n_valid"] = n
        return out
