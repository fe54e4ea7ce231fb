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


# ------------------------------------------------------------------ peer-memory barrier
# One GPU stands in for the ranks' signal arrays with local buffers. Only rank 0's barrier
# ever runs; "rank 1" arriving is a word the host writes before the launch, and a rank that
# never arrives is a word nobody writes. No two launches ever wait on each other.

def _barrier(ws, sig_tab, R, rank, epoch, timeout_ms):
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib().lmh_peer_barrier(ctypes.c_void_p(ws.data_ptr()),
                                  ctypes.c_void_p(sig_tab.data_ptr()), R, rank, epoch,
                                  timeout_ms, st)


def _signals(R):
    sig = [torch.zeros(R, dtype=torch.int32, device="cuda") for _ in range(R)]
    tab = torch.tensor([s.data_ptr() for s in sig], dtype=torch.int64, device="cuda")
    return sig, tab


def test_peer_barrier_times_out_when_a_rank_never_arrives():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    sig, tab = _signals(2)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    assert _barrier(ws, tab, 2, 0, 1, 200) == 0
    t1.record()
    torch.cuda.synchronize()
    assert t0.elapsed_time(t1) >= 190.0            # it waited out its limit, then returned
    assert L.lmh_read_errors(ws) == L.DEVERR_TIMEOUT
    assert sig[1][0].item() == 1 and sig[0][0].item() == 1   # its own signals did land
    assert sig[0][1].item() == 0
    # the context still runs the real path
    x, _ = device_inputs(ragged(130, 64, 300, seed=12))
    out = L.logprob(x["H"], x["W"], x["labels"])
    torch.cuda.synchronize()
    assert L.lmh_read_errors(out["workspace"]) == 0


@pytest.mark.parametrize("epoch,peer_word", [(1, 1), (7, 8), (0xFFFFFFFF, 1), (3, 3)])
def test_peer_barrier_passes_once_every_rank_signalled(epoch, peer_word):
    # the peer's word equal to the epoch, or one barrier ahead (also across the 2^32 wrap)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    R = 3
    sig, tab = _signals(R)
    for j in (1, 2):
        sig[0][j] = torch.tensor(peer_word, dtype=torch.int64).to(torch.int32)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    assert _barrier(ws, tab, R, 0, epoch, 2000) == 0
    t1.record()
    torch.cuda.synchronize()
    assert L.lmh_read_errors(ws) == 0
    assert t0.elapsed_time(t1) < 500.0
    e32 = torch.tensor(epoch, dtype=torch.int64).to(torch.int32).item()
    assert all(sig[j][0].item() == e32 for j in range(R))


def test_peer_barrier_more_ranks_than_a_warp():
    # 40 ranks: a two-warp block; rank 17's barrier with every other word preset passes, and
    # with one word (rank 33's) missing it times out
    R, rank, epoch = 40, 17, 5
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    sig, tab = _signals(R)
    sig[rank].fill_(epoch)
    assert _barrier(ws, tab, R, rank, epoch, 2000) == 0
    torch.cuda.synchronize()
    assert L.lmh_read_errors(ws) == 0
    assert all(sig[j][rank].item() == epoch for j in range(R))
    sig[rank].fill_(epoch + 1)
    sig[rank][33] = epoch                          # rank 33 is one barrier behind
    assert _barrier(ws, tab, R, rank, epoch + 1, 150) == 0
    torch.cuda.synchronize()
    assert L.lmh_read_errors(ws) == L.DEVERR_TIMEOUT


def test_peer_barrier_one_rank_and_argument_checks():
    ws = torch.zeros(512, dtype=torch.uint8, device="cuda")
    sig, tab = _signals(1)
    assert _barrier(ws, tab, 1, 0, 5, 100) == 0
    assert L.lmh_read_errors(ws) == 0 and sig[0][0].item() == 5
    assert _barrier(ws, tab, 1, 0, 0, 100) == 1      # epoch 0 is invalid
    assert _barrier(ws, tab, 1, 1, 1, 100) == 1      # rank >= R
    assert _barrier(ws, tab, 1, 0, 1, 0) == 1        # no time limit
    assert _barrier(ws[8:], tab, 1, 0, 1, 100) == 4  # workspace not 256-byte aligned


def test_exchange_check_raises_after_a_barrier_timed_out():
    # the multi-rank classes' host logic on one device: a group whose peer never arrives
    from lm_head_cross_tcgen05_b200._ranks import RankGroup
    g = RankGroup()
    g.R, g.rank = 2, 0
    g.barrier_timeout_ms = 100
    sig, tab = _signals(2)
    g._sym = dict(key=(0, 0), sig_tab=tab, epoch=0,
                  err=torch.zeros(256, dtype=torch.uint8, device="cuda"))
    g._barrier(g._sym)
    assert g._sym["epoch"] == 1
    with pytest.raises(RuntimeError, match="timed out"):
        g.check_exchange()
    g.check_exchange()                               # the record was cleared when raised
    sig[0][1] = 2                                    # the peer arrives at barrier 2
    g._barrier(g._sym)
    g.check_exchange()
