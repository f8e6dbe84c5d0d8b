"""When to re-place replicas across invocations: a placement policy over a
stream of MoE-layer invocations, on top of zb_plan / zb_plan_placed.

A replica placement is what costs weight movement: every slot whose expert
changes must receive that expert's weights before the layer can run.  The
pages weigh this three ways:

* ``every``  - re-place on every invocation (ISER-MoE: per-invocation
  replication, because history-based plans remove standing skew but not drift
  between batches);
* ``static`` - place once and keep it; each invocation only re-splits the
  quotas over the existing copies (Zepp 4.1 places replicas from historical
  demand);
* ``drift``  - keep the placement until the expert-load vector has drifted:
  re-place when the cosine distance d = 1 - w.w_ref / (|w| |w_ref|) between
  this invocation's per-expert load w and the load the placement was made for
  exceeds delta (ViBE, drift detection, delta = 0.05), or when the kept
  placement no longer fits the receive buffers;
* ``history`` - Zepp's history-based placement (4.1): the slots go to the
  experts with the highest demand per replica over the last ``window``
  invocations (zb_place_by_demand), placed first at invocation 0 and again
  every ``window`` invocations; quotas are re-split on every invocation;
* ``incremental`` - the drift trigger, but instead of a fresh placement the
  kept one is recalibrated (ViBE's incremental update, zb_recalibrate mode
  0): one helper slot changes per step until every rank is within eps = 0.03
  of the mean or no change helps, so only the changed slots move weights.

Every invocation is planned on the GPU (zb_plan for a new placement,
zb_plan_placed to keep one); the drift decision reads the invocation's
per-expert counts back to the host.  ``python -m token_dispatch_top_b200.replan``
runs the three policies over the drifting workload and prints a summary.
"""
from __future__ import annotations

import argparse
import json
import time
from dataclasses import dataclass

import numpy as np
import torch

from . import zb

STRATEGIES = ("every", "static", "drift", "incremental", "history")


def cosine_drift(w: np.ndarray, w_ref: np.ndarray) -> float:
    """1 - cos(w, w_ref) for non-negative load vectors; 0 when either is zero."""
    w = np.asarray(w, np.float64)
    w_ref = np.asarray(w_ref, np.float64)
    nw, nr = np.linalg.norm(w), np.linalg.norm(w_ref)
    if nw == 0.0 or nr == 0.0:
        return 0.0
    return float(1.0 - np.dot(w, w_ref) / (nw * nr))


def slot_changes(old: np.ndarray | None, new: np.ndarray) -> int:
    """Slots whose expert changes (each needs that expert's weights copied in)."""
    new = np.asarray(new)
    if old is None:
        return int((new >= 0).sum())
    old = np.asarray(old)
    return int(((new != old) & (new >= 0)).sum())


def decide(strategy: str, have_placement: bool, drift: float | None, delta: float) -> bool:
    """True when this invocation should get a new placement."""
    if strategy not in STRATEGIES:
        raise ValueError(f"unknown strategy {strategy!r}")
    if not have_placement or strategy == "every":
        return True
    if strategy in ("static", "history"):
        return False
    return drift is not None and drift > delta  # drift and incremental


@dataclass
class StepReport:
    status: int
    max_load: int
    water_level: int
    replaced: bool
    slot_changes: int
    drift: float | None


class Replanner:
    """Plans a stream of invocations of one shape under a placement policy."""

    def __init__(self, cfg: zb.Config, device, strategy: str = "drift", delta: float = 0.05,
                 eps: float = 0.03, max_swaps: int = 64, window: int = 10):
        if strategy not in STRATEGIES:
            raise ValueError(f"unknown strategy {strategy!r}")
        self.cfg, self.strategy, self.delta = cfg, strategy, delta
        self.eps, self.max_swaps, self.window = eps, max_swaps, window
        self.history: list[np.ndarray] = []  # per-expert loads of recent invocations
        self.count = 0
        self.plan = zb.Plan(cfg, device, with_row_src=False)
        self.placement: torch.Tensor | None = None
        self.w_ref: np.ndarray | None = None

    def _adopt(self, w: np.ndarray) -> int:
        new = self.plan.rep_expert.clone()
        changes = slot_changes(None if self.placement is None else
                               self.placement.cpu().numpy(), new.cpu().numpy())
        self.placement, self.w_ref = new, w
        return changes

    def _history_step(self, ids: torch.Tensor) -> StepReport:
        """Zepp: place from the demand of the last `window` invocations."""
        replaced, changes = False, 0
        if self.placement is None:
            # the first invocation has no history: its own counts stand in
            zb.plan(self.plan, ids)
            zb.plan_status(self.plan)
            self.history.append(self.plan.cnt.sum(0).cpu().numpy())
        if self.count % self.window == 0:
            demand = np.sum(self.history[-self.window:], axis=0).astype(np.int64)
            new = torch.from_numpy(zb.place_by_demand(self.cfg, demand)).to(self.plan.cnt.device)
            changes = slot_changes(None if self.placement is None else
                                   self.placement.cpu().numpy(), new.cpu().numpy())
            self.placement, replaced = new, True
        zb.plan_placed(self.plan, ids, self.placement)
        status, _ = zb.plan_status(self.plan)
        if self.count > 0:
            self.history.append(self.plan.cnt.sum(0).cpu().numpy())
        self.history = self.history[-self.window:]
        self.count += 1
        st = self.plan.stats.cpu().numpy()
        return StepReport(status=int(status), max_load=int(st[zb.STAT_MAX_LOAD]),
                          water_level=int(st[zb.STAT_WATER_LEVEL]), replaced=replaced,
                          slot_changes=changes, drift=None)

    def step(self, ids: torch.Tensor) -> StepReport:
        if self.strategy == "history":
            return self._history_step(ids)
        drift = None
        if self.placement is None or self.strategy == "every":
            zb.plan(self.plan, ids)
            status, _ = zb.plan_status(self.plan)
            w = self.plan.cnt.sum(0).cpu().numpy()
            replaced, changes = True, self._adopt(w)
        else:
            zb.plan_placed(self.plan, ids, self.placement)
            status, _ = zb.plan_status(self.plan)
            w = self.plan.cnt.sum(0).cpu().numpy()
            if self.strategy in ("drift", "incremental"):
                drift = cosine_drift(w, self.w_ref)
            replaced, changes = False, 0
            # a kept placement that no longer fits the buffers forces a new one
            forced = self.strategy in ("drift", "incremental") and status == zb.ERR_CAPACITY
            if self.strategy == "incremental" and (forced or decide(self.strategy, True, drift,
                                                                    self.delta)):
                changes, _ = zb.recalibrate(self.cfg, self.plan.cnt, self.placement,
                                            zb.RECAL_SLOT, self.eps, self.max_swaps)
                zb.plan_placed(self.plan, ids, self.placement)
                status, _ = zb.plan_status(self.plan)
                self.w_ref, replaced = w, changes > 0
            elif forced or decide(self.strategy, True, drift, self.delta):
                zb.plan(self.plan, ids)
                status, _ = zb.plan_status(self.plan)
                replaced, changes = True, self._adopt(w)
        st = self.plan.stats.cpu().numpy()
        return StepReport(status=int(status), max_load=int(st[zb.STAT_MAX_LOAD]),
                          water_level=int(st[zb.STAT_WATER_LEVEL]), replaced=replaced,
                          slot_changes=changes, drift=drift)


def study(workload: str = "drift", steps: int | None = None, seed: int = 0,
          delta: float = 0.05, cap_factor: int = 2) -> dict:
    """Run the three policies over one workload's invocations; summarise."""
    from . import build, synth
    build.build()
    wl = synth.WORKLOADS[workload]
    steps = wl.steps if steps is None else steps
    dev = torch.device("cuda", torch.cuda.current_device())
    cfg = zb.Config(P=wl.P, E=wl.E, K=wl.K, S=wl.S, H=wl.H, R=wl.R, C=wl.C,
                    gpus_per_node=wl.gpus_per_node, cap_rows=cap_factor * wl.S * wl.K)
    planners = {s: Replanner(cfg, dev, s, delta) for s in STRATEGIES}
    rows = {s: [] for s in STRATEGIES}
    for t in range(steps):
        ids_np, _ = synth.routing(wl, seed, t)
        ids = torch.from_numpy(ids_np).to(dev)
        for s, rp in planners.items():
            t0 = time.perf_counter()
            r = rp.step(ids)
            rows[s].append((r, time.perf_counter() - t0))
    out = {"workload": workload, "steps": steps, "seed": seed, "delta": delta,
           "cap_rows": cfg.cap, "strategies": {}}
    for s in STRATEGIES:
        rs = [r for r, _ in rows[s]]
        imb = np.array([r.max_load / r.water_level for r in rs])
        out["strategies"][s] = {
            "replacements": int(sum(r.replaced for r in rs)),
            "slot_changes": int(sum(r.slot_changes for r in rs)),
            "max_over_T_mean": float(imb.mean()), "max_over_T_worst": float(imb.max()),
            "capacity_errors": int(sum(r.status == zb.ERR_CAPACITY for r in rs)),
            "host_ms_per_step": 1e3 * float(np.mean([dt for _, dt in rows[s]])),
        }
    return out


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--workload", default="drift")
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--delta", type=float, default=0.05)
    args = ap.parse_args()
    print(json.dumps(study(args.workload, args.steps, args.seed, args.delta)))


if __name__ == "__main__":
    main()
