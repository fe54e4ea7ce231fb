"""lmh_logprob_noalloc: the log-prob entry for callers that may not allocate device memory.

Some callers are handed their input and output buffers and may not call cudaMalloc on the
call path, for example a plugin whose host engine owns the whole device heap, so they cannot
supply the workspace lmh_logprob needs. This entry keeps its scratch in a fixed array inside
the library instead. These tests call it through the C ABI and compare it with lmh_logprob,
twice in a row (the array keeps the previous call's contents, which must not leak into the
next result). This file is named to run last, so that a run stopping at the first failure
has already run every other test.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

import lm_head_cross_tcgen05_b200 as L
from lm_head_cross_tcgen05_b200._abi import lib
from tests.parity import check_rows
from workloads import make_inputs, ragged

pytestmark = pytest.mark.gpu

LMH_ERR_SCRATCH_LIMIT = 6


def noalloc(shape, H, W, y, logprob, lse) -> int:
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return lib().lmh_logprob_noalloc(ctypes.byref(shape), p(H), p(W), p(y), p(logprob), p(lse),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("N,d,V,chunk", [
    (300, 192, 1000, 0),      # one chunk
    (257, 64, 4100, 100),     # the caller's chunk size, ragged tails
    (6000, 128, 128256, 0),   # more partials than the array holds: split into chunks
])
def test_noalloc_matches_logprob_twice(N, d, V, chunk):
    x = make_inputs(ragged(N, d, V, n_ignored=7, seed=4242 + N), device="cuda")
    H, W, y = x["H"], x["W"], x["labels"]
    ref = L.logprob(H, W, y, chunk_rows=chunk)
    shape = L.make_shape(N, d, V, 0, chunk)
    for _ in range(2):
        lp = torch.full((N,), float("nan"), device="cuda")
        lse = torch.full((N,), float("nan"), device="cuda")
        assert noalloc(shape, H, W, y, lp, lse) == 0
        torch.cuda.synchronize()
        check_rows(lp, ref["logprob"], what="logprob")
        check_rows(lse, ref["lse"], what="lse")
        # the header promises more than the tolerance: the same bits as lmh_logprob, whatever
        # chunks the fixed array forces (a row's statistics never depend on its chunk)
        assert torch.equal(lp, ref["logprob"]) and torch.equal(lse, ref["lse"])


def test_noalloc_rejects_shapes_beyond_the_array():
    # one row of per-tile partials for this vocabulary exceeds the fixed array
    H = torch.zeros(2, 64, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(2, dtype=torch.int32, device="cuda")
    out = torch.zeros(2, device="cuda")
    shape = L.make_shape(2, 64, 2_000_000_000)
    assert noalloc(shape, H, W, y, out, out) == LMH_ERR_SCRATCH_LIMIT
