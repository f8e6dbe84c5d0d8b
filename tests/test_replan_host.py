"""The replanner's host logic on CPU.  token_dispatch_top_b200.replan decides,
per invocation, whether to keep, re-place, recalibrate or re-derive the
replica placement; the plans themselves come from the library.  Here the
library's device calls are stood in for by the oracle (test scaffolding
only), while zb_place_by_demand (host code in the library) runs for real,
so every strategy's decisions are checked without a GPU against an
independent recomputation of its rule."""
import numpy as np
import pytest
import torch

import oracle
from token_dispatch_top_b200 import build, replan, synth, zb

DELTA = 0.02


def _ocfg(cfg):
    return oracle.Config(P=cfg.P, E=cfg.E, K=cfg.K, S=cfg.S, H=cfg.H, R=cfg.R, C=cfg.C,
                         gpus_per_node=cfg.gpus_per_node, cap_rows=cfg.cap,
                         policy=cfg.policy, relax=cfg.relax, repair=cfg.repair)


def _fill(p, o):
    for k in ("cnt", "rep_expert", "rep_quota", "home_quota", "load_before", "load_after",
              "cu_seqlens", "dst_row"):
        getattr(p, k).copy_(torch.from_numpy(np.ascontiguousarray(o[k])).view_as(getattr(p, k)))
    st = np.zeros(zb.STATS_LEN, np.int64)
    st[zb.STAT_STATUS], st[zb.STAT_MAX_LOAD] = o["status"], o["max_load"]
    st[zb.STAT_N_REPLICAS], st[zb.STAT_N_ITERS] = o["n_replicas"], o["n_iters"]
    st[zb.STAT_WATER_LEVEL], st[zb.STAT_LOCALITY_COST] = o["T"], o["locality_cost"]
    p.stats.copy_(torch.from_numpy(st))


@pytest.fixture
def host_zb(monkeypatch):
    build.build()
    zb.load()
    monkeypatch.setattr(zb, "plan", lambda p, ids: _fill(
        p, oracle.plan(_ocfg(p.cfg), ids.numpy(), want_M=False)))
    monkeypatch.setattr(zb, "plan_placed", lambda p, ids, pl: _fill(
        p, oracle.plan(_ocfg(p.cfg), ids.numpy(), want_M=False, placement=pl.numpy())))
    monkeypatch.setattr(zb, "plan_status", lambda p: (int(p.stats[zb.STAT_STATUS]),
                                                      int(p.stats[zb.STAT_MAX_LOAD])))

    def recal(cfg, cnt, placement, mode=0, eps=0.03, max_swaps=64):
        pl, n, mx = oracle.recalibrate(_ocfg(cfg), cnt.numpy(), placement.numpy(), mode, eps,
                                       max_swaps)
        placement.copy_(torch.from_numpy(pl))
        return n, mx
    monkeypatch.setattr(zb, "recalibrate", recal)


def _workload():
    wl = synth.WORKLOADS["drift"].with_(S=256)
    cfg = zb.Config(P=wl.P, E=wl.E, K=wl.K, S=wl.S, H=wl.H, R=wl.R,
                    gpus_per_node=wl.gpus_per_node, cap_rows=2 * wl.S * wl.K)
    return wl, cfg


@pytest.mark.parametrize("strategy", replan.STRATEGIES)
def test_strategy_decisions(host_zb, strategy):
    wl, cfg = _workload()
    oc = _ocfg(cfg)
    rp = replan.Replanner(cfg, "cpu", strategy, delta=DELTA, window=5)
    placement, w_ref, hist = None, None, []
    replaced_after_0 = 0
    for t in range(16):
        ids, _ = synth.routing(wl, 0, t)
        rep = rp.step(torch.from_numpy(ids))
        w = np.bincount(ids.ravel(), minlength=wl.E)
        # the rule, recomputed here
        if strategy == "history":
            if t % 5 == 0:
                past = hist[-5:] if t else [w]
                placement = oracle.place_by_demand(oc, np.sum(past, axis=0).astype(np.int64))
                want_replaced = True
            else:
                want_replaced = False
            hist.append(w)
        elif placement is None or strategy == "every":
            placement = oracle.plan(oc, ids, want_M=False)["rep_expert"]
            w_ref, want_replaced = w, True
        else:
            kept = oracle.plan(oc, ids, want_M=False, placement=placement)
            d = replan.cosine_drift(w, w_ref)
            if strategy in ("drift", "incremental"):
                assert rep.drift == pytest.approx(d, abs=1e-12)
            else:
                assert rep.drift is None
            trig = strategy in ("drift", "incremental") and (
                d > DELTA or kept["status"] == oracle.ERR_CAPACITY)
            want_replaced = False
            if trig and strategy == "drift":
                placement = oracle.plan(oc, ids, want_M=False)["rep_expert"]
                w_ref, want_replaced = w, True
            elif trig:
                new, n, _ = oracle.recalibrate(oc, kept["cnt"], placement, 0, 0.03, 64)
                placement, w_ref, want_replaced = new, w, n > 0
                assert rep.slot_changes == n
        assert rep.replaced == want_replaced, (t, rep)
        np.testing.assert_array_equal(rp.placement.numpy(), placement)
        np.testing.assert_array_equal(rp.plan.rep_expert.numpy(), placement)
        replaced_after_0 += want_replaced and t > 0
    expect = {"every": 15, "static": 0, "history": 3}
    if strategy in expect:
        assert replaced_after_0 == expect[strategy]
    else:
        assert 0 < replaced_after_0 < 15


def test_unknown_strategy():
    with pytest.raises(ValueError):
        replan.decide("sometimes", True, 0.0, 0.05)
    _, cfg = _workload()
    with pytest.raises(ValueError):
        replan.Replanner(cfg, "cpu", "sometimes")
