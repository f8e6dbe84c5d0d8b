"""GPU parity of the relaxed transport (eq. (1) of Zepp 4.1 with its band,
relax = 1) against the oracle: plan tables, rows, dispatch and combine
bit-exact, on small random cases, the named workloads at full size, kept
placements, the merged layout, and the capacity edge."""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_plan_equal, cfgs, gpu_plan, plan_tables
from test_gpu_merge import merge_parity
from test_gpu_parity import SMALL, _rand_bits, _random_placement, full_parity, \
    sampled_data_parity
from token_dispatch_top_b200 import build, synth, zb

pytestmark = pytest.mark.gpu

BANDS = (0.05, 0.1, 0.25, 0.5, 0.9)


@pytest.fixture(scope="module")
def dev(cuda_device):
    build.build()
    zb.load()
    return cuda_device


@pytest.mark.parametrize("k", range(1, len(SMALL), 2))
def test_relaxed_random_small(dev, k):
    kw, ids = SMALL[k]
    rng = np.random.default_rng(3000 + k)
    kw = dict(kw, C=BANDS[k % len(BANDS)], relax=1,
              cap_rows=max(1, kw["P"] * kw["S"] * kw["K"]))
    zc, oc = zb.Config(**kw), oracle.Config(**kw)
    w = rng.dirichlet(np.ones(zc.K), size=(zc.P, zc.S)).astype(np.float32)
    full_parity(zc, oc, ids, w, _rand_bits(rng, (zc.P, zc.S, zc.H)),
                _rand_bits(rng, (zc.P * zc.cap, zc.H)), dev)


@pytest.mark.parametrize("name,seed,C", [("tiny", 0, 0.25), ("tiny", 1, 0.5), ("mid", 0, 0.1),
                                         ("mid", 1, 0.05)])
def test_relaxed_workload_full(dev, name, seed, C):
    """Default buffers floor((1+C) S*K); every element compared."""
    wl = synth.WORKLOADS[name]
    zc, oc = cfgs(wl, relax=1, C=C)
    assert zc.cap == oc.cap() > wl.S * wl.K
    ids, w = synth.routing(wl, seed)
    hidden = synth.hidden_bits(wl, seed)
    y = synth.y_bits(wl, zc.P * zc.cap, seed)
    _, status = full_parity(zc, oc, ids, w, hidden, y, dev, with_row_src=(name == "tiny"))
    assert status == oracle.OK


@pytest.mark.parametrize("name,policy", [("hot", 0), ("hot", 1), ("hier", 0), ("hier", 1)])
def test_relaxed_full_size(dev, name, policy):
    wl = synth.WORKLOADS[name]
    zc, oc = cfgs(wl, cap_rows=2 * wl.S * wl.K, policy=policy, relax=1, C=0.1)
    ids, w = synth.routing(wl, 0)
    p, status, _ = gpu_plan(zc, ids, dev, with_row_src=policy == 0)
    o = oracle.plan(oc, ids, want_M=False)
    assert_plan_equal(plan_tables(p), o, status)
    if policy == 0:
        sampled_data_parity(zc, oc, p, o, ids, w, synth.hidden_device(wl, 0, 0, dev), dev,
                            n=128)
    torch.cuda.empty_cache()


def test_relaxed_drift_steps(dev):
    wl = synth.WORKLOADS["drift"]
    zc, oc = cfgs(wl, cap_rows=2 * wl.S * wl.K, relax=1, C=0.1)
    for step in (0, 17, 63):
        ids, _ = synth.routing(wl, 0, step)
        p, status, _ = gpu_plan(zc, ids, dev, with_row_src=False)
        assert_plan_equal(plan_tables(p), oracle.plan(oc, ids, want_M=False), status)


def test_zero_band_equals_exact(dev):
    wl = synth.WORKLOADS["mid"]
    ids, _ = synth.routing(wl, 2)
    tabs = []
    for relax, C in ((0, 0.1), (1, 0.0)):
        zc, _ = cfgs(wl, relax=relax, C=C)
        p, status, _ = gpu_plan(zc, ids, dev)
        assert status == oracle.OK
        tabs.append(plan_tables(p))
    for k in tabs[0]:
        np.testing.assert_array_equal(tabs[0][k], tabs[1][k], err_msg=k)


@pytest.mark.parametrize("k", range(1, len(SMALL), 4))
def test_relaxed_placed(dev, k):
    kw, ids = SMALL[k]
    if kw["R"] == 0:
        pytest.skip("no slots to place")
    rng = np.random.default_rng(4000 + k)
    kw = dict(kw, C=0.3, relax=1, cap_rows=max(1, kw["P"] * kw["S"] * kw["K"]))
    zc, oc = zb.Config(**kw), oracle.Config(**kw)
    pl = _random_placement(rng, zc.P, zc.E, zc.R)
    p = zb.Plan(zc, dev)
    zb.plan_placed(p, torch.from_numpy(ids).to(dev), torch.from_numpy(pl).to(dev))
    status, _ = zb.plan_status(p)
    assert_plan_equal(plan_tables(p), oracle.plan(oc, ids, placement=pl), status)


def test_relaxed_capacity(dev):
    """The band lets rank 1 receive 5 rows; S*K = 4 rows of buffer is a
    capacity error on both sides, with the same max load."""
    kw = dict(P=2, E=2, K=1, S=4, H=8, R=1, C=0.5, relax=1, cap_rows=4)
    zc, oc = zb.Config(**kw), oracle.Config(**kw)
    ids = np.array([[0, 0, 1, 1], [0, 0, 0, 0]], np.int32).reshape(2, 4, 1)
    p, status, max_load = gpu_plan(zc, ids, dev)
    o = oracle.plan(oc, ids)
    assert status == o["status"] == oracle.ERR_CAPACITY
    assert max_load == o["max_load"] == 5


@pytest.mark.parametrize("name,C", [("tiny", 0.5), ("mid", 0.1)])
def test_relaxed_merge(dev, name, C):
    """The merged layout over a banded plan (rows past each rank's receipt
    marked unused)."""
    wl = synth.WORKLOADS[name]
    zc, oc = cfgs(wl, relax=1, C=C)
    ids, _ = synth.routing(wl, 0)
    merge_parity(zc, oc, ids, synth.hidden_bits(wl, 0), dev)
