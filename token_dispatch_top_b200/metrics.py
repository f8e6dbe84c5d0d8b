"""Per-invocation metrics of a plan, and a JSON-lines log of them.

From a plan's tables (host copies of its device buffers):
* R_imb before and after: max_j L_j / mean_j L_j, the rank imbalance of
  ISER-MoE ("Background"), on the routed loads and on the planned loads;
* maxvio = max_e T_e / mean_e T_e - 1 (MoonEP, "Variables and core terms");
* excess removed = (max before - max after) / (max before - T), the share of
  the busiest rank's excess over the water level that planning removed (the
  ISER-MoE E1 table reports this share);
* from the plan's stats: status, locality cost sum a_ij M_ij, replicas,
  greedy iterations, rows moved by quota repair, water level T.

``MetricsLog(path).log(plan, **extra)`` appends one JSON object per call.
This reads plan buffers back to the host, so it synchronises with the device;
it is for monitoring, not for the timed path.
"""
from __future__ import annotations

import json
import math
from typing import Mapping

import numpy as np

from . import zb


def _tables(plan) -> Mapping[str, np.ndarray]:
    if isinstance(plan, Mapping):
        return plan
    return {k: getattr(plan, k).cpu().numpy()
            for k in ("cnt", "load_before", "load_after", "stats")}


def plan_metrics(plan) -> dict:
    """Metrics of a plan: a zb.Plan, or a mapping holding numpy arrays
    ``cnt`` [P,E], ``load_before`` [P], ``load_after`` [P] and optionally
    ``stats`` [ZB_STATS_LEN]."""
    t = _tables(plan)
    cnt = np.asarray(t["cnt"], np.int64)
    before = np.asarray(t["load_before"], np.int64)
    after = np.asarray(t["load_after"], np.int64)
    P = len(before)
    total = int(before.sum())
    mean = total / P
    mb, ma = int(before.max(initial=0)), int(after.max(initial=0))
    Te = cnt.sum(0)
    tbar = Te.sum() / len(Te)
    T = math.ceil(total / P)
    out = {
        "r_imb_before": mb / mean if mean > 0 else 1.0,
        "r_imb_after": ma / mean if mean > 0 else 1.0,
        "maxvio": float(Te.max()) / tbar - 1.0 if tbar > 0 else 0.0,
        "excess_removed": (mb - ma) / (mb - T) if mb > T else 1.0,
        "max_load_before": mb,
        "max_load_after": ma,
    }
    if "stats" in t and t["stats"] is not None:
        st = np.asarray(t["stats"], np.int64)
        out.update(status=int(st[zb.STAT_STATUS]), water_level=int(st[zb.STAT_WATER_LEVEL]),
                   locality_cost=int(st[zb.STAT_LOCALITY_COST]),
                   n_replicas=int(st[zb.STAT_N_REPLICAS]), n_iters=int(st[zb.STAT_N_ITERS]),
                   rows_repaired=int(st[zb.STAT_REPAIRED]))
    return out


class MetricsLog:
    """Appends one JSON object per invocation to ``path``."""

    def __init__(self, path: str):
        self.path = path
        self.count = 0

    def log(self, plan, **extra) -> dict:
        rec = {"invocation": self.count, **plan_metrics(plan), **extra}
        with open(self.path, "a") as f:
            f.write(json.dumps(rec) + "\n")
        self.count += 1
        return rec
