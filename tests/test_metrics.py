"""token_dispatch_top_b200.metrics against the oracle's metrics on the same
plans (CPU): R_imb before and after, maxvio and excess removed agree to
rounding, the stats fields pass through, and the log writes one JSON line per
invocation."""
import json

import numpy as np
import pytest

import oracle
from token_dispatch_top_b200 import metrics, synth, zb


@pytest.mark.parametrize("name,seed", [("tiny", 0), ("tiny", 1), ("mid", 0), ("hier", 0)])
def test_metrics_agree_with_oracle(name, seed):
    wl = synth.WORKLOADS[name]
    cfg = oracle.Config(P=wl.P, E=wl.E, K=wl.K, S=wl.S, H=wl.H, R=wl.R, C=wl.C,
                        gpus_per_node=wl.gpus_per_node, cap_rows=2 * wl.S * wl.K)
    ids, _ = synth.routing(wl, seed)
    p = oracle.plan(cfg, ids, want_M=False)
    want = oracle.metrics(cfg, p)
    stats = np.zeros(zb.STATS_LEN, np.int64)
    stats[zb.STAT_STATUS], stats[zb.STAT_LOCALITY_COST] = p["status"], p["locality_cost"]
    stats[zb.STAT_N_REPLICAS], stats[zb.STAT_N_ITERS] = p["n_replicas"], p["n_iters"]
    stats[zb.STAT_WATER_LEVEL] = p["T"]
    got = metrics.plan_metrics(dict(cnt=p["cnt"], load_before=p["load_before"],
                                    load_after=p["load_after"], stats=stats))
    for k in ("r_imb_before", "r_imb_after", "maxvio", "excess_removed"):
        assert got[k] == pytest.approx(want[k], rel=1e-12, abs=1e-12), k
    assert got["status"] == p["status"] and got["locality_cost"] == p["locality_cost"]
    assert got["water_level"] == p["T"] and got["max_load_after"] == p["max_load"]


def test_log_writes_one_line_per_invocation(tmp_path):
    wl = synth.WORKLOADS["tiny"]
    cfg = oracle.Config(P=wl.P, E=wl.E, K=wl.K, S=wl.S, H=wl.H, R=wl.R)
    log = metrics.MetricsLog(str(tmp_path / "m.jsonl"))
    for seed in range(3):
        ids, _ = synth.routing(wl, seed)
        p = oracle.plan(cfg, ids, want_M=False)
        log.log(dict(cnt=p["cnt"], load_before=p["load_before"], load_after=p["load_after"]),
                seed=seed)
    lines = (tmp_path / "m.jsonl").read_text().splitlines()
    recs = [json.loads(x) for x in lines]
    assert [r["invocation"] for r in recs] == [0, 1, 2]
    assert [r["seed"] for r in recs] == [0, 1, 2]
    assert all(r["r_imb_after"] <= r["r_imb_before"] + 1e-12 for r in recs)
