"""The seeded workload generator: shapes, determinism and calibration."""
import numpy as np
import pytest

from token_dispatch_top_b200 import synth


def test_shapes_and_determinism():
    wl = synth.WORKLOADS["tiny"]
    ids, w = synth.routing(wl, seed=0)
    assert ids.shape == (4, 64, 2) and ids.dtype == np.int32
    assert w.shape == (4, 64, 2) and w.dtype == np.float32
    ids2, w2 = synth.routing(wl, seed=0)
    np.testing.assert_array_equal(ids, ids2)
    np.testing.assert_array_equal(w, w2)
    ids3, _ = synth.routing(wl, seed=1)
    assert not np.array_equal(ids, ids3)
    # top-K ids are distinct within a token and weights are a renormalised softmax
    assert np.all(np.diff(np.sort(ids, axis=2), axis=2) > 0)
    assert np.all(np.abs(w.sum(2) - 1) < 1e-6) and np.all(w[..., 0] >= w[..., 1])
    h = synth.hidden_bits(wl, 0)
    assert h.shape == (4, 64, 128) and h.dtype == np.uint16


def test_hot_share_is_calibrated():
    """The 4 hottest experts of the 'hot' workload take 13% +- 0.5% of
    assignments (ISER-MoE, Key Observations: 13.02% for the top 4 of 384)."""
    wl = synth.WORKLOADS["hot"].with_(S=2048)
    ids, _ = synth.routing(wl, seed=0)
    share = np.isin(ids, np.arange(4)).mean()
    assert abs(share - 0.13) < 0.005
    counts = np.bincount(ids.ravel(), minlength=wl.E)
    assert set(np.argsort(-counts)[:4].tolist()) == {0, 1, 2, 3}


def test_mid_is_permuted_and_zipf():
    wl = synth.WORKLOADS["mid"].with_(S=1024)
    ids, _ = synth.routing(wl, seed=0)
    counts = np.bincount(ids.ravel(), minlength=wl.E)
    b = synth.expert_bias(wl, 0)
    # hottest expert by bias is also among the most routed; ranking is not identity
    assert np.argmax(b) != 0 or np.argmax(counts) != 0
    assert counts[np.argmax(b)] >= np.sort(counts)[-3]


def test_drift_walk_changes_popularity():
    wl = synth.WORKLOADS["drift"]
    b0 = synth.expert_bias(wl, 0, 0)
    b1 = synth.expert_bias(wl, 0, 1)
    b2 = synth.expert_bias(wl, 0, 2)
    d1 = b1 - b0
    d2 = b2 - b1
    assert 0.1 < d1.std() < 0.2 and 0.1 < d2.std() < 0.2
    assert abs(np.corrcoef(d1, d2)[0, 1]) < 0.2
