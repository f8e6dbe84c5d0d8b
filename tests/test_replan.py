"""The placement policy across invocations (token_dispatch_top_b200.replan):
host logic on CPU, and on the GPU every planned invocation against the
oracle (full plan, or the plan that keeps the previous placement)."""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_plan_equal, cfgs, plan_tables
from token_dispatch_top_b200 import replan, synth, zb


def test_cosine_drift_closed_forms():
    w = np.array([3.0, 1.0, 0.0, 2.0])
    assert replan.cosine_drift(w, w) == pytest.approx(0.0, abs=1e-15)
    assert replan.cosine_drift(w, 5 * w) == pytest.approx(0.0, abs=1e-15)
    assert replan.cosine_drift([1, 0], [0, 1]) == pytest.approx(1.0)
    assert replan.cosine_drift([1, 1], [1, 0]) == pytest.approx(1 - 2 ** -0.5)
    assert replan.cosine_drift([0, 0], [1, 2]) == 0.0


def test_slot_changes_and_decisions():
    old = np.array([[-1, 3], [0, -1]])
    assert replan.slot_changes(None, old) == 2
    assert replan.slot_changes(old, old) == 0
    assert replan.slot_changes(old, np.array([[-1, 4], [0, 5]])) == 2
    assert replan.slot_changes(old, np.array([[-1, -1], [0, -1]])) == 0
    assert replan.decide("every", True, 0.0, 0.05)
    assert replan.decide("static", False, None, 0.05)
    assert not replan.decide("static", True, 0.9, 0.05)
    assert replan.decide("drift", True, 0.051, 0.05)
    assert not replan.decide("drift", True, 0.05, 0.05)
    with pytest.raises(ValueError):
        replan.decide("sometimes", True, 0.0, 0.05)


@pytest.mark.gpu
@pytest.mark.parametrize("strategy", replan.STRATEGIES)
def test_replanner_plans_match_oracle(cuda_device, strategy):
    wl = synth.WORKLOADS["drift"].with_(S=2048)
    zc, oc = cfgs(wl, cap_rows=3 * wl.S * wl.K)
    rp = replan.Replanner(zc, cuda_device, strategy, delta=0.01)
    placement = None
    replaced_later = 0
    hist = []
    for t in range(12):
        ids, _ = synth.routing(wl, 0, t)
        w_ref_before = rp.w_ref
        rep = rp.step(torch.from_numpy(ids).to(cuda_device))
        w = np.bincount(ids.ravel(), minlength=wl.E)
        if rep.drift is not None:
            assert rep.drift == pytest.approx(replan.cosine_drift(w, w_ref_before), abs=1e-12)
        if strategy == "history":
            # placed from the summed counts of the last 10 invocations, at
            # t = 0 (its own counts) and t = 10
            if t % 10 == 0:
                past = hist[-10:] if t else [w]
                placement = oracle.place_by_demand(oc, np.sum(past, axis=0).astype(np.int64))
            o = oracle.plan(oc, ids, want_M=False, placement=placement)
            hist.append(w)
            replaced_later += rep.replaced and t > 0
        elif strategy == "incremental" and t > 0:
            # recalibrated from the kept placement when drift or capacity asks
            kept = oracle.plan(oc, ids, want_M=False, placement=placement)
            if rep.drift > 0.01 or kept["status"] == oracle.ERR_CAPACITY:
                placement = oracle.recalibrate(oc, kept["cnt"], placement, 0, 0.03, 64)[0]
                o = oracle.plan(oc, ids, want_M=False, placement=placement)
            else:
                o = kept
            replaced_later += rep.replaced
        elif rep.replaced:
            o = oracle.plan(oc, ids, want_M=False)
            placement = o["rep_expert"]
            replaced_later += t > 0
        else:
            o = oracle.plan(oc, ids, want_M=False, placement=placement)
        assert_plan_equal(plan_tables(rp.plan), o, rep.status)
    if strategy == "static":
        assert replaced_later == 0
    elif strategy == "every":
        assert replaced_later == 11
    elif strategy == "incremental":
        assert replaced_later > 0
    elif strategy == "history":
        assert replaced_later == 1
    else:
        assert 0 < replaced_later < 11
