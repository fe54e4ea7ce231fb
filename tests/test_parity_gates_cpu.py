"""The parity gates themselves, on the CPU: the block-by-block gradient gate (used for
full-size dW) gives the whole-array gate's metrics and rejects what it rejects."""
from __future__ import annotations

import numpy as np
import pytest

from tests.parity import GradStats, check_grad, grad_metrics, rejects


def _blocks(got, ref, what="g", rows=37):
    s = GradStats(what)
    for r0 in range(0, ref.shape[0], rows):
        s.add(got[r0:r0 + rows], ref[r0:r0 + rows])
    return s.check()


def test_block_metrics_equal_whole_array_metrics():
    rng = np.random.default_rng(3)
    ref = rng.standard_normal((300, 64))
    got = ref + 1e-4 * rng.standard_normal(ref.shape)
    m, b = grad_metrics(got, ref), _blocks(got, ref)
    for k in ("maxerr", "maxref"):
        assert m[k] == b[k]
    for k in ("cos", "rel_rms"):
        assert abs(m[k] - b[k]) <= 1e-12 * max(1.0, abs(m[k]))


def test_block_gate_rejects_a_two_percent_scale_and_a_dropped_block():
    rng = np.random.default_rng(4)
    ref = rng.standard_normal((200, 32))
    assert rejects(_blocks, ref * 1.02, ref)
    assert rejects(check_grad, ref * 1.02, ref)
    bad = ref.copy()
    bad[40:80] = 0.0
    assert rejects(_blocks, bad, ref)
    bad = ref.copy()
    bad[5, 7] = np.nan
    assert rejects(_blocks, bad, ref)


def test_block_gate_zero_reference():
    z = np.zeros((10, 4))
    _blocks(z, z)
    with pytest.raises(AssertionError):
        _blocks(z + 1e-3, z)
