"""The plan's device trace (zb_plan_t.trace): a traced plan gives the same
tables as an untraced one, and its stamps respect the order the kernels'
dependency waits impose -- a kernel is released only after the kernel it
waits on has finished -- on the whole-batch plan and on one rank's plan."""
import numpy as np
import pytest
import torch

from parity import PLAN_KEYS
from token_dispatch_top_b200 import build, synth, zb

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev(cuda_device):
    build.build(debug=zb.DEBUG)
    zb.load()
    return cuda_device


def _ordered(k):
    assert k["start"] <= k["released"] <= k["end"], k


@pytest.mark.parametrize("name", ["tiny", "mid", "hier"])
def test_trace_of_the_whole_batch_plan(dev, name):
    wl = synth.WORKLOADS[name]
    cfg = zb.Config(P=wl.P, E=wl.E, K=wl.K, S=wl.S, H=wl.H, R=wl.R, C=wl.C,
                    gpus_per_node=wl.gpus_per_node, cap_rows=2 * wl.S * wl.K)
    ids = torch.from_numpy(synth.routing(wl, 0)[0]).to(dev)
    plain, traced = zb.Plan(cfg, dev), zb.Plan(cfg, dev, trace=True)
    for _ in range(3):  # the trace is reset by every call
        zb.plan(plain, ids)
        zb.plan(traced, ids)
        tl = zb.plan_trace(traced)
        z, h, p, a = (tl[k] for k in zb.TRACE_KERNELS)
        for k in (z, h, p, a):
            _ordered(k)
        assert z["start"] == 0.0  # the first kernel of the call
        assert h["released"] >= z["end"]  # k_hist adds its totals after k_zero
        assert p["released"] >= h["end"]  # the planner reads k_hist's totals
        assert a["released"] >= p["end"]  # k_assign reads the plan
        assert a["end"] < 5000.0  # microseconds: a plan, not a stall
    for key in PLAN_KEYS + ("dst_row", "row_src", "stats"):
        assert torch.equal(getattr(plain, key), getattr(traced, key)), key


def test_trace_of_one_ranks_plan(dev):
    wl = synth.WORKLOADS["mid"]
    cfg = zb.Config(P=wl.P, E=wl.E, K=wl.K, S=wl.S, H=wl.H, R=wl.R, C=wl.C)
    ids_np = synth.routing(wl, 0)[0]
    ids = [torch.from_numpy(np.ascontiguousarray(ids_np[r])).to(dev) for r in range(wl.P)]
    rps = [zb.RankPlan(cfg, r, dev, trace=(r == 3)) for r in range(wl.P)]
    for r in range(wl.P):
        zb.count(rps[r], ids[r])
    table = torch.stack([rp.counts for rp in rps])
    for rp in rps:
        rp.table.copy_(table)
    zb.plan_rank(rps[3], ids[3])
    tl = zb.plan_trace(rps[3])
    assert tl["k_zero"] is None and tl["k_hist"] is None  # zb_count ran them apart
    _ordered(tl["k_planner"])
    _ordered(tl["k_assign"])
    assert tl["k_planner"]["start"] == 0.0
    assert tl["k_assign"]["released"] >= tl["k_planner"]["end"]
    with pytest.raises(zb.ZbError):
        zb.plan_trace(rps[0])  # made without a trace
