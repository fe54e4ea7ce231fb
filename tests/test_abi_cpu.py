"""The C ABI without a GPU: every symbol include/lmh.h declares is exported by liblmh.so, the
workspace planner follows its documented rules, and argument errors are reported on the host
before any CUDA call."""
import ctypes

import pytest

from lm_head_cross_tcgen05_b200 import _abi
import lm_head_cross_tcgen05_b200 as L


def test_header_symbols_exported():
    names = _abi.header_symbols()
    assert {"lmh_workspace_size", "lmh_loss_fwd", "lmh_loss_bwd", "lmh_logprob",
            "lmh_support_logprob", "lmh_support_kl", "lmh_read_errors"} <= set(names)
    lib = ctypes.CDLL(_abi.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def ws(N, d, V, K=0, chunk=0, flags=0, entry=L.ENTRY_LOSS_FWD):
    return L.lmh_workspace_size(L.make_shape(N, d, V, K, chunk, flags), entry)


def test_invalid_shapes_size_zero():
    assert ws(10, 96, 100) == 0           # d not a multiple of 64
    assert ws(-1, 64, 100) == 0
    assert ws(10, 64, 0) == 0
    assert ws(10, 64, 100, K=0, entry=L.ENTRY_SUPPORT_KL) == 0
    assert ws(10, 64, 100, K=L.MAX_K + 1, entry=L.ENTRY_SUPPORT_LOGPROB) == 0
    assert ws(10, 64, 100, entry=9) == 0
    assert ws(10, 64, 100, entry=-1) == 0


def test_chunk_buffer_term():
    N, d, V = 8192, 4096, 128256
    base = ws(N, d, V, chunk=N)
    fused = ws(N, d, V, chunk=N, flags=L.F_FUSED_BWD)
    # the fused forward adds one chunk's bf16 softmax buffer [c, round_up(V, 8)] and the fp32
    # partials [2, c, d] of its dH, whose 256 x 512 tiles split the vocabulary in two ranges
    # (256 tiles: 4 rounds of 74 CTA pairs unsplit, 3.5 split in two)
    assert fused - base == pytest.approx(N * 128256 * 2 + 2 * N * d * 4, abs=512)
    # one chunk: no internal dW accumulator
    assert ws(N, d, V, chunk=N, flags=L.F_FUSED_BWD | L.F_DW_ACC_GIVEN) == fused


def test_dh_tile_plan():
    # (rows, d, V) -> (256 x 512 tiles, vocabulary ranges), counted in rounds of 74 CTA pairs
    assert L.lmh_dh_plan(8192, 4096, 128256) == (True, 2)   # 256 wide tiles: 3.5 rounds split
    assert L.lmh_dh_plan(8192, 4096, 151936) == (True, 2)   # the support workload's chunk
    assert L.lmh_dh_plan(2048, 5120, 151936) == (False, 4)  # 160 narrow units x 4: 2.25 rounds
    assert L.lmh_dh_plan(4096, 2048, 32000) == (True, 1)    # V too short to split
    assert L.lmh_dh_plan(1000, 4096, 65536) == (True, 2)
    assert L.lmh_dh_plan(1000, 4352, 65536) == (True, 2)    # last wide tile half outside d
    assert L.lmh_dh_plan(64, 256, 2048) == (False, 1)       # one tile either way
    assert L.lmh_dh_plan(300, 320, 70000) == (False, 2)
    assert L.lmh_dh_plan(600, 1024, 262144) == (True, 8)      # 6 wide tiles: one round in 8
    for bad in ((0, 64, 100), (10, 96, 100), (10, 64, 0), (10, 64, 1 << 31)):
        with pytest.raises(L.LmhError):
            L.lmh_dh_plan(*bad)
    # the plan's split partials are what a fused chunk's workspace adds for dH
    for rows, d, V in ((1000, 4096, 65536), (2048, 5120, 151936), (4096, 2048, 32000)):
        wide, sp = L.lmh_dh_plan(rows, d, V)
        extra = ws(rows, d, V, chunk=rows, flags=L.F_FUSED_BWD) - ws(rows, d, V, chunk=rows)
        assert extra == pytest.approx(rows * ((V + 7) // 8 * 8) * 2 +
                                      (sp * rows * d * 4 if sp > 1 else 0), abs=512)


def test_budgeted_workload_fits_two_gigabytes():
    N, d, V = 16384, 5120, 151936
    b = ws(N, d, V, chunk=2048, flags=L.F_FUSED_BWD | L.F_MEAN | L.F_DW_ACC_GIVEN)
    assert b <= 2 * 1024 ** 3
    # without a caller accumulator the fp32 [V, d] one is added for the multi-chunk plan
    b2 = ws(N, d, V, chunk=2048, flags=L.F_FUSED_BWD)
    assert b2 - b == pytest.approx(V * d * 4, abs=512)


def test_default_chunk_is_4096_rows():
    N, d, V = 10000, 64, 1000
    a = ws(N, d, V, chunk=0, flags=L.F_FUSED_BWD | L.F_DW_ACC_GIVEN)
    b = ws(N, d, V, chunk=4096, flags=L.F_FUSED_BWD | L.F_DW_ACC_GIVEN)
    assert a == b


def test_backward_and_support_sizes():
    assert ws(100, 64, 1000, K=8, entry=L.ENTRY_LOSS_BWD) > ws(100, 64, 1000, entry=L.ENTRY_LOGPROB)
    assert ws(100, 64, 1000, K=8, entry=L.ENTRY_SUPPORT_KL) > 0
    assert ws(0, 64, 1000, entry=L.ENTRY_LOSS_FWD) > 0   # header only


def test_host_argument_errors_without_gpu():
    lib = _abi.lib()
    shape = L.make_shape(4, 64, 100)
    # null H/W with N > 0: rejected on the host before any CUDA call
    st = lib.lmh_loss_fwd(ctypes.byref(shape), *([None] * 13), ctypes.c_void_p(256), 1 << 20, None)
    assert st == 1
    bad = L.make_shape(4, 100, 100)
    st = lib.lmh_logprob(ctypes.byref(bad), *([None] * 6), 0, None)
    assert st == 1
    st = lib.lmh_loss_bwd(ctypes.byref(shape), 9, *([None] * 10), 0, None)
    assert st == 1
    assert lib.lmh_read_errors(None, None, None) == 1


def test_vocab_parallel_sizes():
    # combine: the header only; partials: a shard-local label buffer on top of the log-prob
    # entry's plan; shard backward: the standalone backward's plan without dH split partials
    assert ws(1000, 64, 5000, entry=L.ENTRY_VP_COMBINE) == 256
    assert ws(1000, 64, 5000, entry=L.ENTRY_VP_PARTIALS) == \
        ws(1000, 64, 5000, entry=L.ENTRY_LOGPROB) + 4096
    N, d, Vr = 2048, 5120, 151936 // 4     # few dH tiles, large V: one-device plan would split
    assert ws(N, d, Vr, chunk=N, entry=L.ENTRY_VP_BWD) < ws(N, d, Vr, chunk=N, entry=L.ENTRY_LOSS_BWD)


def test_vocab_parallel_host_errors_without_gpu():
    lib = _abi.lib()
    shard = L.make_shape(4, 64, 100)
    P = [None] * 5
    # shard past the vocabulary, negative offset, empty vocabulary: refused before any CUDA call
    assert lib.lmh_vp_partials(ctypes.byref(shard), 50, 120, *P, 0, None) == 1
    assert lib.lmh_vp_partials(ctypes.byref(shard), -1, 120, *P, 0, None) == 1
    assert lib.lmh_vp_loss_bwd(ctypes.byref(shard), 0, 0, 0, *([None] * 9), None, 0,
                               None) == 1
    assert lib.lmh_vp_loss_bwd(ctypes.byref(shard), 2, 0, 100, *([None] * 9), None, 0,
                               None) == 1
    # a receive table with an out-of-range rank, and one alongside dH_part: refused
    bad = _abi.lmh_vp_dest(ctypes.c_void_p(256), 2, 2)
    assert lib.lmh_vp_loss_bwd(ctypes.byref(shard), 0, 0, 100, *([None] * 8),
                               ctypes.byref(bad), None, 0, None) == 1
    assert lib.lmh_vp_reduce_rows_to(2, 4, 64, None, None, 0, 0, None) == 1   # no output
    assert lib.lmh_vp_combine(ctypes.byref(shard), 0, *([None] * 10), 0, None) == 1
    assert lib.lmh_vp_reduce_rows(2, 4, 96, None, None, None) == 1     # d not a multiple of 64
    assert lib.lmh_vp_reduce_rows(0, 4, 64, None, None, None) == 1
    assert lib.lmh_vp_reduce_rows(2, 0, 64, None, None, None) == 0     # nothing to do


def test_binding_rejects_tensors_smaller_than_the_shape():
    # a W with fewer columns than shape.d would let the tensor maps read past its allocation:
    # the binding refuses it before any pointer reaches the library
    import torch
    shape = L.make_shape(4, 64, 100)
    H = torch.zeros(4, 64, dtype=torch.bfloat16)
    W = torch.zeros(100, 32, dtype=torch.bfloat16)
    y = torch.zeros(4, dtype=torch.int32)
    f = torch.zeros(4, dtype=torch.float32)
    ws = torch.zeros(1 << 16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="W has 3200 elements"):
        L.lmh_loss_fwd(shape, H, W, y, f, f, workspace=ws)
    with pytest.raises(ValueError, match="lse has"):
        L.lmh_logprob(shape, H, torch.zeros(100, 64, dtype=torch.bfloat16), y, f,
                      torch.zeros(3), workspace=ws)
    sup = L.make_shape(4, 64, 100, K=8)
    with pytest.raises(ValueError, match="ids has"):
        L.lmh_support_logprob(sup, H, torch.zeros(100, 64, dtype=torch.bfloat16),
                              torch.zeros(4, 4, dtype=torch.int32),
                              torch.zeros(4, 8), f, workspace=ws)
    with pytest.raises(ValueError, match="records has"):
        L.lmh_vp_combine(shape, 3, torch.zeros(2, 4, 4), y, f, f, workspace=ws)


def test_weighted_fused_size_adds_row_coefficients():
    # lmh_loss_fwd_bwd's plan: the fused forward's plus alpha [N] and beta [N] fp32
    f = ws(1000, 64, 5000, chunk=1000, flags=L.F_FUSED_BWD | L.F_DW_ACC_GIVEN)
    w = ws(1000, 64, 5000, chunk=1000, flags=L.F_FUSED_BWD | L.F_DW_ACC_GIVEN,
           entry=L.ENTRY_LOSS_FWD_BWD)
    assert w - f == 2 * 4096


def test_ctypes_signatures_match_header_parameter_counts():
    # every declaration in include/lmh.h and the binding's ctypes signature agree on the
    # number of parameters (a drifted count would shift every pointer after it)
    import re
    src = open(_abi.HEADER).read()
    decls = re.findall(r"LMH_API\s+[\w\s\*]*?\b(lmh_\w+)\s*\(([^;]*?)\);", src, flags=re.S)
    assert len(decls) == len(_abi.header_symbols())
    for name, params in decls:
        n = 0 if params.strip() in ("", "void") else len(params.split(","))
        assert n == len(_abi._SIGS[name][1]), name


def test_data_parallel_host_errors_without_gpu():
    lib = _abi.lib()
    # refused before any CUDA call: negative rows, empty vocabulary, no output, no labels
    assert lib.lmh_count_valid(-1, 100, None, None, None) == 1
    assert lib.lmh_count_valid(4, 0, None, ctypes.c_void_p(256), None) == 1
    assert lib.lmh_count_valid(4, 100, ctypes.c_void_p(256), None, None) == 1
    assert lib.lmh_count_valid(4, 100, None, ctypes.c_void_p(256), None) == 1
    assert lib.lmh_count_valid(4, 100, ctypes.c_void_p(258), ctypes.c_void_p(256), None) == 4
    assert lib.lmh_reduce_ranks_f32(0, 4, None, None, None) == 1
    assert lib.lmh_reduce_ranks_f32(2, -1, None, None, None) == 1
    assert lib.lmh_reduce_ranks_f32(2, 0, None, None, None) == 0     # nothing to do
    assert lib.lmh_reduce_ranks_f32(2, 4, ctypes.c_void_p(256), None, None) == 1
    assert lib.lmh_reduce_ranks_f32(2, 4, ctypes.c_void_p(256), ctypes.c_void_p(6), None) == 4
    # the row-scattering step: no destination, a rank outside the group, a support mode
    sh = L.make_shape(4, 64, 100, 0, 4, L.F_FUSED_BWD)
    P = [None] * 11
    assert lib.lmh_dp_loss_fwd_bwd(ctypes.byref(sh), 0, *P, None, None, 0, None) == 1
    bad = _abi.lmh_vp_dest(ctypes.c_void_p(256), 2, 2)
    assert lib.lmh_dp_loss_fwd_bwd(ctypes.byref(sh), 0, *P, ctypes.byref(bad), None, 0, None) == 1
    ok = _abi.lmh_vp_dest(ctypes.c_void_p(256), 2, 1)
    assert lib.lmh_dp_loss_fwd_bwd(ctypes.byref(sh), 2, *P, ctypes.byref(ok), None, 0, None) == 1


def test_dw_store_flag_is_sizing_neutral():
    # LMH_F_DW_ACC_STORE changes what the call writes into the caller's accumulator, not the
    # workspace it needs
    for entry in (L.ENTRY_LOSS_FWD, L.ENTRY_LOSS_FWD_BWD, L.ENTRY_LOSS_BWD):
        base = L.F_FUSED_BWD | L.F_DW_ACC_GIVEN
        assert ws(3000, 64, 5000, chunk=1000, flags=base, entry=entry) == \
            ws(3000, 64, 5000, chunk=1000, flags=base | L.F_DW_ACC_STORE, entry=entry)


def test_peer_barrier_host_errors_without_gpu():
    lib = _abi.lib()
    ws, tab = ctypes.c_void_p(256), ctypes.c_void_p(512)
    assert lib.lmh_peer_barrier(None, tab, 2, 0, 1, 100, None) == 1
    assert lib.lmh_peer_barrier(ws, None, 2, 0, 1, 100, None) == 1
    assert lib.lmh_peer_barrier(ws, tab, 0, 0, 1, 100, None) == 1      # no rank
    assert lib.lmh_peer_barrier(ws, tab, 1025, 0, 1, 100, None) == 1   # more than one block
    assert lib.lmh_peer_barrier(ws, tab, 2, 2, 1, 100, None) == 1      # rank outside 0..R-1
    assert lib.lmh_peer_barrier(ws, tab, 2, -1, 1, 100, None) == 1
    assert lib.lmh_peer_barrier(ws, tab, 2, 0, 0, 100, None) == 1      # epoch 0
    assert lib.lmh_peer_barrier(ws, tab, 2, 0, 1, 0, None) == 1        # unbounded wait
    assert lib.lmh_peer_barrier(ws, tab, 2, 0, 1, 60001, None) == 1
    assert lib.lmh_peer_barrier(ctypes.c_void_p(264), tab, 2, 0, 1, 100, None) == 4
    assert lib.lmh_peer_barrier(ws, ctypes.c_void_p(516), 2, 0, 1, 100, None) == 4
