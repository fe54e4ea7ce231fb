"""The seeded input generators give the shapes and distributions the workloads name."""
import numpy as np
import torch

from workloads import IGNORE_INDEX, WORKLOADS, make_candidates, make_inputs, make_labels, zipf_labels


def test_tiny_inputs():
    wl = WORKLOADS["tiny"]
    x = make_inputs(wl)
    assert x["H"].shape == (64, 256) and x["H"].dtype == torch.bfloat16
    assert x["W"].shape == (2048, 256) and x["W"].dtype == torch.bfloat16
    y = x["labels"]
    assert y.dtype == torch.int32 and int((y == IGNORE_INDEX).sum()) == 8
    assert int(y.max()) < 2048
    assert abs(float(x["W"].float().std()) - 0.02) < 0.002
    # seeded: the same call gives the same bits
    x2 = make_inputs(wl)
    assert torch.equal(x["H"], x2["H"]) and torch.equal(x["labels"], x2["labels"])


def test_ignored_fraction_and_zipf():
    wl = WORKLOADS["small"].scaled(N=2000, d=64)
    y = make_labels(wl, 1)
    assert int((y == IGNORE_INDEX).sum()) == round(0.05 * 2000)
    g = torch.Generator().manual_seed(3)
    z = zipf_labels(200000, 32000, 1.1, g, "cpu").numpy()
    # P(0) / P(1) = 2^1.1 for Zipf(1.1)
    ratio = (z == 0).sum() / (z == 1).sum()
    assert abs(ratio - 2 ** 1.1) < 0.1
    assert z.min() >= 0 and z.max() < 32000


def test_candidates_contain_label_without_repeats():
    y = torch.tensor([5, 0, 99, -100], dtype=torch.int32)
    ids = make_candidates(y, 100, 16, 7).numpy()
    assert ids.shape == (4, 16)
    for i in range(4):
        assert len(set(ids[i].tolist())) == 16
        assert ids[i].min() >= 0 and ids[i].max() < 100
        if y[i] >= 0:
            assert int(y[i]) in ids[i]


def test_support_ref_logprobs_normalised():
    wl = WORKLOADS["support"].scaled(N=32, d=64, V=500)
    x = make_inputs(wl)
    r = x["ref_logp"].double()
    assert r.shape == (32, 64)
    np.testing.assert_allclose(torch.logsumexp(r, 1).numpy(), 0.0, atol=1e-5)
