"""Deterministic chunked LM-head + loss on B200 (sm_100a): Python binding of liblmh.so.

The functions named ``lmh_*`` mirror the C ABI of ``include/lmh.h`` one to one: they take
torch CUDA tensors, check dtype / contiguity / device, and pass raw pointers and the
current stream through ctypes. Every step of the computation runs in the library's CUDA
kernels; there is no fallback path, and importing this package fails if ``liblmh.so`` has
not been built (``python lm_head_cross_tcgen05_b200/build.py``).

The lower-case helpers (``loss_fwd``, ``loss_bwd``, ``logprob``, ``support_logprob``,
``support_kl``) allocate the outputs and the workspace with torch and call the same entries.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from ._abi import (BWD_CE, BWD_LOGPROB, BWD_SUPPORT_KL, BWD_SUPPORT_LOGPROB, DEVERR_LABEL_RANGE,
                   DEVERR_NONFINITE, DEVERR_TEMPERATURE, DEVERR_TIMEOUT, ENTRY_LOGPROB, ENTRY_LOSS_BWD,
                   ENTRY_LOSS_FWD, ENTRY_SUPPORT_KL, ENTRY_SUPPORT_LOGPROB, ENTRY_VP_BWD,
                   ENTRY_LOSS_FWD_BWD, ENTRY_VP_COMBINE, ENTRY_VP_PARTIALS,
                   ENTRY_VP_SUPPORT_BWD, ENTRY_VP_SUPPORT_COMBINE, ENTRY_VP_SUPPORT_PARTIALS,
                   F_DW_ACC_GIVEN, F_DW_ACC_STORE,
                   F_GRAD_SCALAR, lmh_vp_dest,
                   F_FUSED_BWD, F_MEAN, F_SUPPORT_RENORM, IGNORE_INDEX, MAX_K, STATUS_NAMES, lib, lmh_shape)

__all__ = [
    "lmh_shape", "make_shape", "lmh_workspace_size", "lmh_dh_plan", "lmh_loss_fwd", "lmh_loss_bwd",
    "lmh_logprob", "lmh_support_logprob", "lmh_support_kl", "lmh_support_kl_fwd_bwd",
    "lmh_support_fwd_bwd", "support_fwd_bwd",
    "lmh_read_errors", "LmhError",
    "loss_fwd", "loss_bwd", "logprob", "support_logprob", "support_kl", "workspace",
    "IGNORE_INDEX", "BWD_CE", "BWD_LOGPROB", "BWD_SUPPORT_LOGPROB", "BWD_SUPPORT_KL",
    "F_MEAN", "F_FUSED_BWD", "F_DW_ACC_GIVEN", "F_SUPPORT_RENORM", "ENTRY_LOSS_FWD", "ENTRY_LOSS_BWD",
    "ENTRY_LOGPROB", "ENTRY_SUPPORT_LOGPROB", "ENTRY_SUPPORT_KL", "DEVERR_LABEL_RANGE",
    "DEVERR_TIMEOUT", "DEVERR_NONFINITE", "DEVERR_TEMPERATURE", "MAX_K",
    "lmh_vp_partials", "lmh_vp_combine", "lmh_vp_loss_bwd", "lmh_vp_fused_bwd",
    "lmh_vp_reduce_rows", "lmh_vp_reduce_rows_to", "lmh_scale_bf16",
    "ENTRY_VP_PARTIALS", "ENTRY_VP_COMBINE", "ENTRY_VP_BWD", "F_GRAD_SCALAR",
    "ENTRY_LOSS_FWD_BWD", "lmh_loss_fwd_bwd", "loss_fwd_bwd",
    "ENTRY_VP_SUPPORT_PARTIALS", "ENTRY_VP_SUPPORT_COMBINE", "ENTRY_VP_SUPPORT_BWD",
    "lmh_vp_support_partials", "lmh_vp_support_combine", "lmh_vp_support_bwd",
    "F_DW_ACC_STORE", "lmh_count_valid", "lmh_reduce_ranks_f32", "lmh_dp_loss_fwd_bwd",
    "lmh_peer_barrier",
]

lib()  # load now: a missing library is an import error, never a silent fallback


class LmhError(RuntimeError):
    def __init__(self, entry: str, status: int):
        super().__init__(f"{entry}: {STATUS_NAMES.get(status, status)}")
        self.status = status


def make_shape(N: int, d: int, V: int, K: int = 0, chunk_rows: int = 0, flags: int = 0,
               temperature=None) -> lmh_shape:
    """temperature: None (off), a float (one temperature for every row) or a CUDA float32
    tensor [N] of per-row temperatures (kept alive by the caller for the call)."""
    scalar, rows = 0.0, None
    if isinstance(temperature, torch.Tensor):
        if temperature.numel() != int(N):
            raise ValueError("per-row temperature must have N elements")
        rows = _p(temperature, _f32, "temperature")
    elif temperature is not None:
        scalar = float(temperature)
    return lmh_shape(int(N), int(d), int(V), int(K), int(chunk_rows), int(flags), scalar, rows)


def _p(t: Optional[torch.Tensor], dtype=None, what: str = "tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{what} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _fits(**named) -> None:
    """Each named (tensor, elements) pair: the tensor, when given, holds at least that many
    elements, so no kernel can index past its allocation for the shape the call declares."""
    for what, (t, n) in named.items():
        if t is not None and t.numel() < int(n):
            raise ValueError(f"{what} has {t.numel()} elements; the shape needs {int(n)}")


def _s(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ok(name: str, status: int):
    if status != 0:
        raise LmhError(name, status)


_bf, _f32, _i32, _u8 = torch.bfloat16, torch.float32, torch.int32, torch.uint8


# ----------------------------------------------------------------------------- C ABI mirror

def lmh_workspace_size(shape: lmh_shape, entry: int) -> int:
    return int(lib().lmh_workspace_size(ctypes.byref(shape), int(entry)))


def lmh_dh_plan(rows: int, d: int, V: int) -> tuple[bool, int]:
    """(wide 256 x 512 tiles?, vocabulary ranges) of one chunk's dH GEMM."""
    wide, splits = ctypes.c_int32(), ctypes.c_int32()
    _ok("lmh_dh_plan",
        lib().lmh_dh_plan(int(rows), int(d), int(V), ctypes.byref(wide), ctypes.byref(splits)))
    return bool(wide.value), int(splits.value)


def lmh_loss_fwd(shape, H, W, labels, loss_rows, lse, logprob=None, argmax=None, loss_mean=None,
                 n_valid=None, n_valid_given=None, dH=None, dW=None, dW_acc=None, *, workspace,
                 stream=None) -> None:
    N, d, V = shape.N, shape.d, shape.V
    _fits(H=(H, N * d), W=(W, V * d), labels=(labels, N), loss_rows=(loss_rows, N),
          lse=(lse, N), logprob=(logprob, N), argmax=(argmax, N), loss_mean=(loss_mean, 1),
          n_valid=(n_valid, 1), n_valid_given=(n_valid_given, 1), dH=(dH, N * d),
          dW=(dW, V * d), dW_acc=(dW_acc, V * d))
    st = lib().lmh_loss_fwd(
        ctypes.byref(shape), _p(H, _bf, "H"), _p(W, _bf, "W"), _p(labels, _i32, "labels"),
        _p(loss_rows, _f32, "loss_rows"), _p(lse, _f32, "lse"), _p(logprob, _f32, "logprob"),
        _p(argmax, _i32, "argmax"), _p(loss_mean, _f32, "loss_mean"),
        _p(n_valid, _i32, "n_valid"), _p(n_valid_given, _i32, "n_valid_given"),
        _p(dH, _bf, "dH"), _p(dW, _bf, "dW"), _p(dW_acc, _f32, "dW_acc"),
        _p(workspace, _u8, "workspace"), workspace.numel(), _s(stream))
    _ok("lmh_loss_fwd", st)


def lmh_loss_bwd(shape, mode, H, W, targets, lse, grad, ref_logp=None, dH=None, dW=None,
                 dW_acc=None, *, workspace, stream=None) -> None:
    N, d, V, K = shape.N, shape.d, shape.V, max(shape.K, 1)
    cands = int(mode) in (BWD_SUPPORT_LOGPROB, BWD_SUPPORT_KL)
    g = 1 if shape.flags & F_GRAD_SCALAR else (N * K if int(mode) == BWD_SUPPORT_LOGPROB else N)
    _fits(H=(H, N * d), W=(W, V * d), targets=(targets, N * K if cands else N), lse=(lse, N),
          grad=(grad, g), ref_logp=(ref_logp, N * K), dH=(dH, N * d), dW=(dW, V * d),
          dW_acc=(dW_acc, V * d))
    st = lib().lmh_loss_bwd(
        ctypes.byref(shape), int(mode), _p(H, _bf, "H"), _p(W, _bf, "W"),
        _p(targets, _i32, "targets"), _p(lse, _f32, "lse"), _p(grad, _f32, "grad"),
        _p(ref_logp, _f32, "ref_logp"), _p(dH, _bf, "dH"), _p(dW, _bf, "dW"),
        _p(dW_acc, _f32, "dW_acc"), _p(workspace, _u8, "workspace"), workspace.numel(),
        _s(stream))
    _ok("lmh_loss_bwd", st)


def lmh_loss_fwd_bwd(shape, mode, H, W, labels, grad, loss_rows, lse, logprob=None,
                     argmax=None, loss_mean=None, n_valid=None, n_valid_given=None, dH=None,
                     dW=None, dW_acc=None, *, workspace, stream=None) -> None:
    N, d, V = shape.N, shape.d, shape.V
    _fits(H=(H, N * d), W=(W, V * d), labels=(labels, N),
          grad=(grad, 1 if shape.flags & F_GRAD_SCALAR else N), loss_rows=(loss_rows, N),
          lse=(lse, N), logprob=(logprob, N), argmax=(argmax, N), loss_mean=(loss_mean, 1),
          n_valid=(n_valid, 1), n_valid_given=(n_valid_given, 1), dH=(dH, N * d),
          dW=(dW, V * d), dW_acc=(dW_acc, V * d))
    st = lib().lmh_loss_fwd_bwd(
        ctypes.byref(shape), int(mode), _p(H, _bf, "H"), _p(W, _bf, "W"),
        _p(labels, _i32, "labels"), _p(grad, _f32, "grad"), _p(loss_rows, _f32, "loss_rows"),
        _p(lse, _f32, "lse"), _p(logprob, _f32, "logprob"), _p(argmax, _i32, "argmax"),
        _p(loss_mean, _f32, "loss_mean"), _p(n_valid, _i32, "n_valid"),
        _p(n_valid_given, _i32, "n_valid_given"), _p(dH, _bf, "dH"), _p(dW, _bf, "dW"),
        _p(dW_acc, _f32, "dW_acc"), _p(workspace, _u8, "workspace"), workspace.numel(),
        _s(stream))
    _ok("lmh_loss_fwd_bwd", st)


def lmh_logprob(shape, H, W, labels, logprob, lse, *, workspace, stream=None) -> None:
    N, d, V = shape.N, shape.d, shape.V
    _fits(H=(H, N * d), W=(W, V * d), labels=(labels, N), logprob=(logprob, N), lse=(lse, N))
    st = lib().lmh_logprob(ctypes.byref(shape), _p(H, _bf, "H"), _p(W, _bf, "W"),
                           _p(labels, _i32, "labels"), _p(logprob, _f32, "logprob"),
                           _p(lse, _f32, "lse"), _p(workspace, _u8, "workspace"),
                           workspace.numel(), _s(stream))
    _ok("lmh_logprob", st)


def lmh_support_logprob(shape, H, W, ids, lp, lse, *, workspace, stream=None) -> None:
    N, d, V, K = shape.N, shape.d, shape.V, shape.K
    _fits(H=(H, N * d), W=(W, V * d), ids=(ids, N * K), lp=(lp, N * K), lse=(lse, N))
    st = lib().lmh_support_logprob(ctypes.byref(shape), _p(H, _bf, "H"), _p(W, _bf, "W"),
                                   _p(ids, _i32, "ids"), _p(lp, _f32, "lp"), _p(lse, _f32, "lse"),
                                   _p(workspace, _u8, "workspace"), workspace.numel(),
                                   _s(stream))
    _ok("lmh_support_logprob", st)


def lmh_support_kl(shape, H, W, ids, ref_logp, kl_rows, kl_mean=None, lp=None, lse=None, *,
                   workspace, stream=None) -> None:
    N, d, V, K = shape.N, shape.d, shape.V, shape.K
    _fits(H=(H, N * d), W=(W, V * d), ids=(ids, N * K), ref_logp=(ref_logp, N * K),
          kl_rows=(kl_rows, N), kl_mean=(kl_mean, 1), lp=(lp, N * K), lse=(lse, N))
    st = lib().lmh_support_kl(ctypes.byref(shape), _p(H, _bf, "H"), _p(W, _bf, "W"),
                              _p(ids, _i32, "ids"), _p(ref_logp, _f32, "ref_logp"),
                              _p(kl_rows, _f32, "kl_rows"), _p(kl_mean, _f32, "kl_mean"),
                              _p(lp, _f32, "lp"), _p(lse, _f32, "lse"),
                              _p(workspace, _u8, "workspace"), workspace.numel(), _s(stream))
    _ok("lmh_support_kl", st)


def lmh_support_kl_fwd_bwd(shape, H, W, ids, ref_logp, kl_rows, kl_mean=None, lp=None,
                           lse=None, dH=None, dW=None, dW_acc=None, *, workspace,
                           stream=None) -> None:
    N, d, V, K = shape.N, shape.d, shape.V, shape.K
    _fits(H=(H, N * d), W=(W, V * d), ids=(ids, N * K), ref_logp=(ref_logp, N * K),
          kl_rows=(kl_rows, N), kl_mean=(kl_mean, 1), lp=(lp, N * K), lse=(lse, N),
          dH=(dH, N * d), dW=(dW, V * d), dW_acc=(dW_acc, V * d))
    st = lib().lmh_support_kl_fwd_bwd(
        ctypes.byref(shape), _p(H, _bf, "H"), _p(W, _bf, "W"), _p(ids, _i32, "ids"),
        _p(ref_logp, _f32, "ref_logp"), _p(kl_rows, _f32, "kl_rows"),
        _p(kl_mean, _f32, "kl_mean"), _p(lp, _f32, "lp"), _p(lse, _f32, "lse"),
        _p(dH, _bf, "dH"), _p(dW, _bf, "dW"), _p(dW_acc, _f32, "dW_acc"),
        _p(workspace, _u8, "workspace"), workspace.numel(), _s(stream))
    _ok("lmh_support_kl_fwd_bwd", st)


def lmh_support_fwd_bwd(shape, mode, H, W, ids, ref_logp, grad, kl_rows=None, kl_mean=None,
                        lp=None, lse=None, dH=None, dW=None, dW_acc=None, *, workspace,
                        stream=None) -> None:
    N, d, V, K = shape.N, shape.d, shape.V, shape.K
    g = 1 if shape.flags & F_GRAD_SCALAR else (N * K if int(mode) == BWD_SUPPORT_LOGPROB else N)
    _fits(H=(H, N * d), W=(W, V * d), ids=(ids, N * K), ref_logp=(ref_logp, N * K),
          grad=(grad, g), kl_rows=(kl_rows, N), kl_mean=(kl_mean, 1), lp=(lp, N * K),
          lse=(lse, N), dH=(dH, N * d), dW=(dW, V * d), dW_acc=(dW_acc, V * d))
    st = lib().lmh_support_fwd_bwd(
        ctypes.byref(shape), int(mode), _p(H, _bf, "H"), _p(W, _bf, "W"), _p(ids, _i32, "ids"),
        _p(ref_logp, _f32, "ref_logp"), _p(grad, _f32, "grad"), _p(kl_rows, _f32, "kl_rows"),
        _p(kl_mean, _f32, "kl_mean"), _p(lp, _f32, "lp"), _p(lse, _f32, "lse"),
        _p(dH, _bf, "dH"), _p(dW, _bf, "dW"), _p(dW_acc, _f32, "dW_acc"),
        _p(workspace, _u8, "workspace"), workspace.numel(), _s(stream))
    _ok("lmh_support_fwd_bwd", st)


def support_fwd_bwd(mode: int, H, W, ids, grad=None, ref_logp=None, *, chunk_rows: int = 0,
                    mean: bool = False, scalar_grad: bool = False, dW_acc=None,
                    temperature=None, want_dH: bool = True, want_dW: bool = True, ws=None,
                    stream=None) -> dict:
    """The support forward (lp, lse; kl_rows, kl_mean for BWD_SUPPORT_KL) plus dH, dW of
    sum_i g_i KL_i or sum_ik g_ik lp_ik in one pass, the weights known before the call.
    want_dH / want_dW False leaves that gradient out (its GEMM is skipped)."""
    N, d = H.shape
    V, K = W.shape[0], ids.shape[1]
    dev = H.device
    flags = (F_FUSED_BWD | (F_MEAN if mean else 0) | (F_GRAD_SCALAR if scalar_grad else 0)
             | (F_DW_ACC_GIVEN if dW_acc is not None else 0))
    shape = make_shape(N, d, V, K, chunk_rows, flags, temperature)
    kl = int(mode) == BWD_SUPPORT_KL
    out = dict(lp=torch.empty(N, K, dtype=_f32, device=dev),
               lse=torch.empty(N, dtype=_f32, device=dev),
               dH=torch.empty(N, d, dtype=_bf, device=dev) if want_dH else None,
               dW=torch.empty(V, d, dtype=_bf, device=dev) if want_dW else None)
    if kl:
        out["kl_rows"] = torch.empty(N, dtype=_f32, device=dev)
        out["kl_mean"] = torch.empty(1, dtype=_f32, device=dev)
    ws = workspace(shape, ENTRY_SUPPORT_KL, dev) if ws is None else ws
    lmh_support_fwd_bwd(shape, mode, H, W, ids, ref_logp, grad, out.get("kl_rows"),
                        out.get("kl_mean"), out["lp"], out["lse"], out["dH"], out["dW"], dW_acc,
                        workspace=ws, stream=stream)
    out["workspace"] = ws
    return out


def lmh_vp_partials(shard, v0, V_total, H, W_shard, labels, records, *, workspace,
                    stream=None) -> None:
    N, d = shard.N, shard.d
    _fits(H=(H, N * d), W_shard=(W_shard, shard.V * d), labels=(labels, N),
          records=(records, N * 4))
    st = lib().lmh_vp_partials(ctypes.byref(shard), int(v0), int(V_total), _p(H, _bf, "H"),
                               _p(W_shard, _bf, "W_shard"), _p(labels, _i32, "labels"),
                               _p(records, _f32, "records"), _p(workspace, _u8, "workspace"),
                               workspace.numel(), _s(stream))
    _ok("lmh_vp_partials", st)


def lmh_vp_combine(shape, R, records, labels, loss_rows, lse, logprob=None, argmax=None,
                   loss_mean=None, n_valid=None, n_valid_given=None, *, workspace,
                   stream=None) -> None:
    N = shape.N
    _fits(records=(records, int(R) * N * 4), labels=(labels, N), loss_rows=(loss_rows, N),
          lse=(lse, N), logprob=(logprob, N), argmax=(argmax, N), loss_mean=(loss_mean, 1),
          n_valid=(n_valid, 1), n_valid_given=(n_valid_given, 1))
    st = lib().lmh_vp_combine(ctypes.byref(shape), int(R), _p(records, _f32, "records"),
                              _p(labels, _i32, "labels"), _p(loss_rows, _f32, "loss_rows"),
                              _p(lse, _f32, "lse"), _p(logprob, _f32, "logprob"),
                              _p(argmax, _i32, "argmax"), _p(loss_mean, _f32, "loss_mean"),
                              _p(n_valid, _i32, "n_valid"),
                              _p(n_valid_given, _i32, "n_valid_given"),
                              _p(workspace, _u8, "workspace"), workspace.numel(), _s(stream))
    _ok("lmh_vp_combine", st)


def _dest(dest):
    """(recv pointer table: an int64 CUDA tensor of R device addresses, R, rank) -> struct."""
    if dest is None:
        return None
    table, R, rank = dest
    if table.dtype != torch.int64 or table.numel() < int(R):
        raise ValueError("the receive-buffer table must hold R int64 device addresses")
    return ctypes.byref(lmh_vp_dest(_p(table, None, "recv table"), int(R), int(rank)))


def lmh_vp_loss_bwd(shard, mode, v0, V_total, H, W_shard, labels, lse, grad=None, dH_part=None,
                    dW_shard=None, dW_acc_shard=None, dest=None, *, workspace,
                    stream=None) -> None:
    N, d, Vr = shard.N, shard.d, shard.V
    _fits(H=(H, N * d), W_shard=(W_shard, Vr * d), labels=(labels, N), lse=(lse, N),
          grad=(grad, 1 if shard.flags & F_GRAD_SCALAR else N), dH_part=(dH_part, N * d),
          dW_shard=(dW_shard, Vr * d), dW_acc_shard=(dW_acc_shard, Vr * d))
    st = lib().lmh_vp_loss_bwd(ctypes.byref(shard), int(mode), int(v0), int(V_total),
                               _p(H, _bf, "H"), _p(W_shard, _bf, "W_shard"),
                               _p(labels, _i32, "labels"), _p(lse, _f32, "lse"),
                               _p(grad, _f32, "grad"), _p(dH_part, _f32, "dH_part"),
                               _p(dW_shard, _bf, "dW_shard"), _p(dW_acc_shard, _f32, "dW_acc_shard"),
                               _dest(dest), _p(workspace, _u8, "workspace"), workspace.numel(),
                               _s(stream))
    _ok("lmh_vp_loss_bwd", st)


def lmh_vp_fused_bwd(shard, v0, V_total, H, W_shard, labels, lse, n_valid_given=None,
                     dH_part=None, dW_shard=None, dW_acc_shard=None, dest=None, *, workspace,
                     stream=None) -> None:
    N, d, Vr = shard.N, shard.d, shard.V
    _fits(H=(H, N * d), W_shard=(W_shard, Vr * d), labels=(labels, N), lse=(lse, N),
          n_valid_given=(n_valid_given, 1), dH_part=(dH_part, N * d),
          dW_shard=(dW_shard, Vr * d), dW_acc_shard=(dW_acc_shard, Vr * d))
    st = lib().lmh_vp_fused_bwd(ctypes.byref(shard), int(v0), int(V_total), _p(H, _bf, "H"),
                                _p(W_shard, _bf, "W_shard"), _p(labels, _i32, "labels"),
                                _p(lse, _f32, "lse"), _p(n_valid_given, _i32, "n_valid_given"),
                                _p(dH_part, _f32, "dH_part"), _p(dW_shard, _bf, "dW_shard"),
                                _p(dW_acc_shard, _f32, "dW_acc_shard"), _dest(dest),
                                _p(workspace, _u8, "workspace"), workspace.numel(), _s(stream))
    _ok("lmh_vp_fused_bwd", st)


def lmh_vp_support_partials(shard, v0, V_total, H, W_shard, ids, records, *, workspace,
                            stream=None) -> None:
    N, d, K = shard.N, shard.d, shard.K
    _fits(H=(H, N * d), W_shard=(W_shard, shard.V * d), ids=(ids, N * K),
          records=(records, N * (K + 1)))
    st = lib().lmh_vp_support_partials(ctypes.byref(shard), int(v0), int(V_total),
                                       _p(H, _bf, "H"), _p(W_shard, _bf, "W_shard"),
                                       _p(ids, _i32, "ids"), _p(records, _f32, "records"),
                                       _p(workspace, _u8, "workspace"), workspace.numel(),
                                       _s(stream))
    _ok("lmh_vp_support_partials", st)


def lmh_vp_support_combine(shape, R, records, ids, ref_logp, lp, lse, kl_rows=None,
                           kl_mean=None, *, workspace, stream=None) -> None:
    N, K = shape.N, shape.K
    _fits(records=(records, int(R) * N * (K + 1)), ids=(ids, N * K), ref_logp=(ref_logp, N * K),
          lp=(lp, N * K), lse=(lse, N), kl_rows=(kl_rows, N), kl_mean=(kl_mean, 1))
    st = lib().lmh_vp_support_combine(ctypes.byref(shape), int(R), _p(records, _f32, "records"),
                                      _p(ids, _i32, "ids"), _p(ref_logp, _f32, "ref_logp"),
                                      _p(lp, _f32, "lp"), _p(lse, _f32, "lse"),
                                      _p(kl_rows, _f32, "kl_rows"), _p(kl_mean, _f32, "kl_mean"),
                                      _p(workspace, _u8, "workspace"), workspace.numel(),
                                      _s(stream))
    _ok("lmh_vp_support_combine", st)


def lmh_vp_support_bwd(shard, mode, v0, V_total, H, W_shard, ids, lse, grad=None, ref_logp=None,
                       dH_part=None, dW_shard=None, dW_acc_shard=None, dest=None, *, workspace,
                       stream=None) -> None:
    N, d, Vr, K = shard.N, shard.d, shard.V, shard.K
    g = 1 if shard.flags & F_GRAD_SCALAR else (N * K if int(mode) == BWD_SUPPORT_LOGPROB else N)
    _fits(H=(H, N * d), W_shard=(W_shard, Vr * d), ids=(ids, N * K), lse=(lse, N),
          grad=(grad, g), ref_logp=(ref_logp, N * K), dH_part=(dH_part, N * d),
          dW_shard=(dW_shard, Vr * d), dW_acc_shard=(dW_acc_shard, Vr * d))
    st = lib().lmh_vp_support_bwd(ctypes.byref(shard), int(mode), int(v0), int(V_total),
                                  _p(H, _bf, "H"), _p(W_shard, _bf, "W_shard"),
                                  _p(ids, _i32, "ids"), _p(lse, _f32, "lse"),
                                  _p(grad, _f32, "grad"), _p(ref_logp, _f32, "ref_logp"),
                                  _p(dH_part, _f32, "dH_part"), _p(dW_shard, _bf, "dW_shard"),
                                  _p(dW_acc_shard, _f32, "dW_acc_shard"), _dest(dest),
                                  _p(workspace, _u8, "workspace"), workspace.numel(), _s(stream))
    _ok("lmh_vp_support_bwd", st)


def lmh_vp_reduce_rows(parts, out, stream=None) -> None:
    """parts [R, rows, d] fp32 -> out [rows, d] bf16, summed in ascending R."""
    R, rows, d = parts.shape
    _fits(out=(out, rows * d))
    st = lib().lmh_vp_reduce_rows(int(R), int(rows), int(d), _p(parts, _f32, "parts"),
                                  _p(out, _bf, "out"), _s(stream))
    _ok("lmh_vp_reduce_rows", st)


def lmh_vp_reduce_rows_to(parts, outs, n_out, row_offset, stream=None) -> None:
    """parts [R, rows, d] fp32 summed in ascending R into rows row_offset.. of every output;
    outs: an int64 CUDA tensor of n_out device addresses of [*, d] bf16 buffers."""
    R, rows, d = parts.shape
    if outs.dtype != torch.int64 or outs.numel() < int(n_out):
        raise ValueError("outs must hold n_out int64 device addresses")
    st = lib().lmh_vp_reduce_rows_to(int(R), int(rows), int(d), _p(parts, _f32, "parts"),
                                     _p(outs, None, "outs"), int(n_out), int(row_offset),
                                     _s(stream))
    _ok("lmh_vp_reduce_rows_to", st)


def lmh_count_valid(labels, V, n_valid, stream=None) -> None:
    """n_valid[0] = the rows with 0 <= label < V (int32, on the device)."""
    _fits(n_valid=(n_valid, 1))
    st = lib().lmh_count_valid(int(labels.numel()), int(V), _p(labels, _i32, "labels"),
                               _p(n_valid, _i32, "n_valid"), _s(stream))
    _ok("lmh_count_valid", st)


def lmh_dp_loss_fwd_bwd(shape, mode, H, W, labels, grad, loss_rows, lse, logprob=None,
                        argmax=None, loss_mean=None, n_valid_given=None, dH=None, dest=None, *,
                        workspace, stream=None) -> None:
    """dest: (int64 CUDA tensor of the R receive-buffer addresses, R, rank)."""
    N, d, V = shape.N, shape.d, shape.V
    _fits(H=(H, N * d), W=(W, V * d), labels=(labels, N),
          grad=(grad, 1 if shape.flags & F_GRAD_SCALAR else N), loss_rows=(loss_rows, N),
          lse=(lse, N), logprob=(logprob, N), argmax=(argmax, N), loss_mean=(loss_mean, 1),
          n_valid_given=(n_valid_given, 1), dH=(dH, N * d))
    st = lib().lmh_dp_loss_fwd_bwd(
        ctypes.byref(shape), int(mode), _p(H, _bf, "H"), _p(W, _bf, "W"),
        _p(labels, _i32, "labels"), _p(grad, _f32, "grad"), _p(loss_rows, _f32, "loss_rows"),
        _p(lse, _f32, "lse"), _p(logprob, _f32, "logprob"), _p(argmax, _i32, "argmax"),
        _p(loss_mean, _f32, "loss_mean"), _p(n_valid_given, _i32, "n_valid_given"),
        _p(dH, _bf, "dH"), _dest(dest), _p(workspace, _u8, "workspace"), workspace.numel(),
        _s(stream))
    _ok("lmh_dp_loss_fwd_bwd", st)


def lmh_reduce_ranks_f32(parts, out, stream=None) -> None:
    """parts [R, n] fp32 -> out [n] fp32, summed in ascending R."""
    R, n = parts.shape
    _fits(out=(out, n))
    st = lib().lmh_reduce_ranks_f32(int(R), int(n), _p(parts, _f32, "parts"),
                                    _p(out, _f32, "out"), _s(stream))
    _ok("lmh_reduce_ranks_f32", st)


def lmh_scale_bf16(x, g, stream=None) -> None:
    """x *= g[0] in place (x bf16 with a multiple of 4 elements; g a one-element device fp32)."""
    _fits(g=(g, 1))
    st = lib().lmh_scale_bf16(_p(x, _bf, "x"), int(x.numel()), _p(g, _f32, "g"), _s(stream))
    _ok("lmh_scale_bf16", st)


def lmh_peer_barrier(workspace, signals, R: int, rank: int, epoch: int,
                     timeout_ms: int = 4000, stream=None) -> None:
    """Barrier number ``epoch`` of R ranks through peer memory: signals is an int64 CUDA
    tensor [R] of the ranks' signal-array addresses (each R uint32 words, zeroed before the
    first barrier); a time-out sets LMH_DEVERR_TIMEOUT in the workspace's error word."""
    _fits(signals=(signals, R))
    st = lib().lmh_peer_barrier(_p(workspace, _u8, "workspace"),
                                _p(signals, torch.int64, "signals"), int(R), int(rank),
                                int(epoch), int(timeout_ms), _s(stream))
    _ok("lmh_peer_barrier", st)


def lmh_read_errors(workspace: torch.Tensor, stream=None) -> int:
    out = ctypes.c_uint32(0)
    _ok("lmh_read_errors", lib().lmh_read_errors(_p(workspace, _u8, "workspace"),
                                                 ctypes.byref(out), _s(stream)))
    return int(out.value)


# ----------------------------------------------------------------------------- helpers

def workspace(shape: lmh_shape, entry: int, device) -> torch.Tensor:
    n = lmh_workspace_size(shape, entry)
    if n == 0:
        raise ValueError("invalid shape for this entry")
    return torch.empty(n, dtype=_u8, device=device)


def loss_fwd(H, W, labels, *, chunk_rows: int = 0, mean: bool = True, grads: bool = False,
             want_dH: bool = True, want_dW: bool = True, dW_acc=None, n_valid_given=None,
             temperature=None, ws=None, stream=None) -> dict:
    """CE forward (loss_rows, lse, logprob, argmax, loss_mean, n_valid); with grads=True also
    dH / dW of the mean (or summed) loss, fused with the forward."""
    N, d = H.shape
    V = W.shape[0]
    dev = H.device
    flags = (F_MEAN if mean else 0) | (F_FUSED_BWD if grads else 0) | (
        F_DW_ACC_GIVEN if dW_acc is not None else 0)
    shape = make_shape(N, d, V, 0, chunk_rows, flags, temperature)
    out = dict(loss_rows=torch.empty(N, dtype=_f32, device=dev),
               lse=torch.empty(N, dtype=_f32, device=dev),
               logprob=torch.empty(N, dtype=_f32, device=dev),
               argmax=torch.empty(N, dtype=_i32, device=dev),
               loss_mean=torch.empty(1, dtype=_f32, device=dev),
               n_valid=torch.empty(1, dtype=_i32, device=dev))
    if grads:
        out["dH"] = torch.empty(N, d, dtype=_bf, device=dev) if want_dH else None
        out["dW"] = torch.empty(V, d, dtype=_bf, device=dev) if want_dW else None
    ws = workspace(shape, ENTRY_LOSS_FWD, dev) if ws is None else ws
    lmh_loss_fwd(shape, H, W, labels, out["loss_rows"], out["lse"], out["logprob"],
                 out["argmax"], out["loss_mean"], out["n_valid"], n_valid_given,
                 out.get("dH"), out.get("dW"), dW_acc, workspace=ws, stream=stream)
    out["workspace"] = ws
    return out


def loss_fwd_bwd(mode: int, H, W, labels, grad=None, *, chunk_rows: int = 0,
                 mean: bool = False, scalar_grad: bool = False, dW_acc=None,
                 n_valid_given=None, temperature=None, want_dH: bool = True,
                 want_dW: bool = True, ws=None, stream=None) -> dict:
    """Forward outputs plus dH, dW of L = sum_i w_i l_i (l = loss for BWD_CE, log-prob for
    BWD_LOGPROB; w from grad as in loss_bwd) in one pass: the fused path for objectives whose
    row weights are known before the forward, such as policy-gradient losses. want_dH /
    want_dW False: that gradient is not computed (its GEMM is skipped; a frozen input)."""
    N, d = H.shape
    V = W.shape[0]
    dev = H.device
    flags = (F_FUSED_BWD | (F_MEAN if mean else 0) | (F_GRAD_SCALAR if scalar_grad else 0)
             | (F_DW_ACC_GIVEN if dW_acc is not None else 0))
    shape = make_shape(N, d, V, 0, chunk_rows, flags, temperature)
    out = dict(loss_rows=torch.empty(N, dtype=_f32, device=dev),
               lse=torch.empty(N, dtype=_f32, device=dev),
               logprob=torch.empty(N, dtype=_f32, device=dev),
               argmax=torch.empty(N, dtype=_i32, device=dev),
               loss_mean=torch.empty(1, dtype=_f32, device=dev),
               n_valid=torch.empty(1, dtype=_i32, device=dev),
               dH=torch.empty(N, d, dtype=_bf, device=dev) if want_dH else None,
               dW=torch.empty(V, d, dtype=_bf, device=dev) if want_dW else None)
    ws = workspace(shape, ENTRY_LOSS_FWD_BWD, dev) if ws is None else ws
    lmh_loss_fwd_bwd(shape, mode, H, W, labels, grad, out["loss_rows"], out["lse"],
                     out["logprob"], out["argmax"], out["loss_mean"], out["n_valid"],
                     n_valid_given, out["dH"], out["dW"], dW_acc, workspace=ws, stream=stream)
    out["workspace"] = ws
    return out


def loss_bwd(mode: int, H, W, targets, lse, grad, ref_logp=None, *, chunk_rows: int = 0,
             want_dH: bool = True, want_dW: bool = True, dW_acc=None, temperature=None,
             mean: bool = False, renorm: bool = False, scalar_grad: bool = False, ws=None,
             stream=None) -> dict:
    """Backward of one objective (LMH_BWD_*). grad=None: unit row weights, or 1 / count with
    mean=True, taken on the device. scalar_grad=True: grad is a one-element device tensor g
    that multiplies every term's weight (LMH_F_GRAD_SCALAR)."""
    N, d = H.shape
    V = W.shape[0]
    K = targets.shape[1] if targets.dim() == 2 else 1
    dev = H.device
    flags = ((F_DW_ACC_GIVEN if dW_acc is not None else 0) | (F_MEAN if mean else 0)
             | (F_SUPPORT_RENORM if renorm else 0) | (F_GRAD_SCALAR if scalar_grad else 0))
    shape = make_shape(N, d, V, K, chunk_rows, flags, temperature)
    out = dict(dH=torch.empty(N, d, dtype=_bf, device=dev) if want_dH else None,
               dW=torch.empty(V, d, dtype=_bf, device=dev) if want_dW else None)
    ws = workspace(shape, ENTRY_LOSS_BWD, dev) if ws is None else ws
    lmh_loss_bwd(shape, mode, H, W, targets, lse, grad, ref_logp, out["dH"], out["dW"], dW_acc,
                 workspace=ws, stream=stream)
    out["workspace"] = ws
    return out


def logprob(H, W, labels, *, chunk_rows: int = 0, temperature=None, ws=None,
            stream=None) -> dict:
    N, d = H.shape
    shape = make_shape(N, d, W.shape[0], 0, chunk_rows, 0, temperature)
    out = dict(logprob=torch.empty(N, dtype=_f32, device=H.device),
               lse=torch.empty(N, dtype=_f32, device=H.device))
    ws = workspace(shape, ENTRY_LOGPROB, H.device) if ws is None else ws
    lmh_logprob(shape, H, W, labels, out["logprob"], out["lse"], workspace=ws, stream=stream)
    out["workspace"] = ws
    return out


def support_logprob(H, W, ids, *, chunk_rows: int = 0, temperature=None, renorm: bool = False,
                    ws=None, stream=None) -> dict:
    """renorm=True: log-probs normalised over each row's candidates (LMH_F_SUPPORT_RENORM)."""
    N, d = H.shape
    K = ids.shape[1]
    shape = make_shape(N, d, W.shape[0], K, chunk_rows, F_SUPPORT_RENORM if renorm else 0,
                       temperature)
    out = dict(lp=torch.empty(N, K, dtype=_f32, device=H.device),
               lse=torch.empty(N, dtype=_f32, device=H.device))
    ws = workspace(shape, ENTRY_SUPPORT_LOGPROB, H.device) if ws is None else ws
    lmh_support_logprob(shape, H, W, ids, out["lp"], out["lse"], workspace=ws, stream=stream)
    out["workspace"] = ws
    return out


def support_kl(H, W, ids, ref_logp, *, chunk_rows: int = 0, temperature=None,
               renorm: bool = False, grads: bool = False, mean: bool = True, dW_acc=None,
               want_dH: bool = True, want_dW: bool = True, ws=None, stream=None) -> dict:
    """KL(ref || model) over the candidates (kl_rows, kl_mean, lp, lse). grads=True: also dH
    and dW of the mean (or summed) KL in the same pass (lmh_support_kl_fwd_bwd); want_dH /
    want_dW False leaves that gradient out."""
    N, d = H.shape
    V, K = W.shape[0], ids.shape[1]
    flags = (F_SUPPORT_RENORM if renorm else 0) | (F_FUSED_BWD | (F_MEAN if mean else 0)
                                                   if grads else 0) | (
        F_DW_ACC_GIVEN if dW_acc is not None else 0)
    shape = make_shape(N, d, V, K, chunk_rows, flags, temperature)
    dev = H.device
    out = dict(kl_rows=torch.empty(N, dtype=_f32, device=dev),
               kl_mean=torch.empty(1, dtype=_f32, device=dev),
               lp=torch.empty(N, K, dtype=_f32, device=dev),
               lse=torch.empty(N, dtype=_f32, device=dev))
    ws = workspace(shape, ENTRY_SUPPORT_KL, dev) if ws is None else ws
    if grads:
        out["dH"] = torch.empty(N, d, dtype=_bf, device=dev) if want_dH else None
        out["dW"] = torch.empty(V, d, dtype=_bf, device=dev) if want_dW else None
        lmh_support_kl_fwd_bwd(shape, H, W, ids, ref_logp, out["kl_rows"], out["kl_mean"],
                               out["lp"], out["lse"], out["dH"], out["dW"], dW_acc,
                               workspace=ws, stream=stream)
    else:
        lmh_support_kl(shape, H, W, ids, ref_logp, out["kl_rows"], out["kl_mean"], out["lp"],
                       out["lse"], workspace=ws, stream=stream)
    out["workspace"] = ws
    return out
