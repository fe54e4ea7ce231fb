"""Failure detection on the GPU without a GPU fault: a bounded wait that runs out reports
LMH_DEVERR_TIMEOUT through the error word and leaves the context usable; bad inputs are
reported on the host or through the error word, never by a trap."""
import ctypes

import pytest
import torch

import lm_head_cross_tcgen05_b200 as L
from lm_head_cross_tcgen05_b200._abi import lib
from tests.gpu_common import device_inputs, ragged

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib().lmh_selftest_wait_timeout(ctypes.c_void_p(ws.data_ptr()), 200, st) == 0
    assert L.lmh_read_errors(ws) == L.DEVERR_TIMEOUT
    # the same context still runs the real path
    x, _ = device_inputs(ragged(130, 64, 300, seed=11))
    out = L.logprob(x["H"], x["W"], x["labels"])
    torch.cuda.synchronize()
    assert L.lmh_read_errors(out["workspace"]) == 0
    assert torch.isfinite(out["lse"]).all()


def test_selftest_argument_checks():
    ws = torch.zeros(512, dtype=torch.uint8, device="cuda")
    p = ctypes.c_void_p(ws.data_ptr())
    assert lib().lmh_selftest_wait_timeout(p, 0, None) == 1
    assert lib().lmh_selftest_wait_timeout(p, 6000, None) == 1
    assert lib().lmh_selftest_wait_timeout(ctypes.c_void_p(ws.data_ptr() + 8), 10, None) == 4
