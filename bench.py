"""Benchmark: plan + dispatch + combine tokens/s on B200, with the HBM roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload tiny|mid|hot|hier|drift] [--no-extras]

One step is one invocation of the whole hot path (histogram, greedy replica
plan, assignment, dispatch scatter, combine gather) on the headline workload,
by default mid: P=8 virtual ranks, E=64, K=6, S=4096 tokens per rank, H=2048
bf16, R=2, C=0.1, Zipf s=1.2 popularity with a per-seed permuted ranking.  The
expert outputs fed to the combine are the dispatched rows themselves
(identity experts), so the step moves exactly the dispatch and combine
traffic.  Inputs are seeded and synthetic.

* ``value``: tokens/s over all ranks, device-timed with CUDA events with the
  inputs resident in HBM, steps pipelined two deep (the plan of step k+1 on
  its own stream beside the rows of step k).  Every step streams its rows
  through buffers larger than L2.
* ``serial``: the same steps one at a time, L2 flushed before each (outside
  the events) by a 256 MB write and a 256 MB read; per-kernel event times.
  A bounded device spin (about 0.1 ms) precedes each step, so that the host
  has enqueued the step's kernels before its first event: the events time
  the device's latency, not the host's launch overhead.
* ``e2e``: the same metric through the public API with pinned host buffers:
  each step copies ids, weights and hidden rows host->device, runs the path,
  and copies the combined rows and the plan status back; the copies run on
  their own streams with three buffer slots, so the input copy of one step
  overlaps the output copy of the one before.
* ``roofline``: the dominant kernel's algorithmic bytes per launch over its
  event-timed duration, against the measured HBM copy bandwidth.
* ``cpu_baseline``: the CPU oracle (single thread) on full steps of the same
  workload, rank 0 at N=1 only.
* ``extras.workloads`` (N=1): the other four workloads one invocation at a
  time: plan latency, dispatch and combine rates and fractions of the peak,
  and the plan's balance (drift: steps 0, 31 and 63).
* ``plan_timeline_us`` (N=1): per workload, the plan's device timeline from
  its trace stamps: each kernel's start, release from its dependency wait
  and end, in microseconds from the call's first kernel.
* ``extras.rank_path`` (N=1): the entry points one rank of P GPUs calls
  (count, plan_rank, dispatch_rank, combine_rank) for each of the P ranks of
  the same workload in turn, each call timed alone; checked against the
  whole-batch path's rows.

With ``--impl reference`` the CPU oracle itself is timed on the same workload
(rank 0 only; other ranks exit).  With N>1 (torchrun), every rank runs an
independent replica on its own GPU; ``value`` is the sum of tokens over ranks
divided by the slowest rank's time.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "plan+dispatch+combine tokens/s at 1 GPU; achieved HBM GB/s vs B200 peak"
UNIT = "tokens/s"
WORKLOAD = "mid"
FALLBACK_HBM_GBS = 6650.0
SLEEP_CYCLES = 200_000  # ~0.1 ms at 1.965 GHz: longer than the host needs to enqueue a step


def route_steps(wl) -> tuple:
    """The routing steps a run cycles through: step 0 alone, or, for a workload
    that drifts over many steps, 8 of them spread over the walk (a new draw,
    and so a new plan, at every timed step)."""
    return tuple(range(0, wl.steps, max(1, wl.steps // 8))) if wl.steps > 1 else (0,)


def workload_desc(wl) -> str:
    if wl.hot_share is not None:
        pop = (f"4 hottest experts take {wl.hot_share:.0%} of assignments, the rest Zipf "
               f"s={wl.hot_zipf_s}")
    else:
        pop = f"Zipf s={wl.zipf_s} popularity"
    if wl.permute:
        pop += ", permuted ranking"
    if wl.walk_sigma:
        pop += f", log-popularity random walk sigma={wl.walk_sigma} per step"
    nodes = f", {wl.P // wl.gpus_per_node} nodes x {wl.gpus_per_node}" \
        if wl.gpus_per_node > 1 else ""
    steps = route_steps(wl)
    cycle = f"; step k re-plans on walk step {steps[1] - steps[0]}*(k mod {len(steps)})" \
        if len(steps) > 1 else ""
    return (f"{wl.name}: P={wl.P}{nodes} E={wl.E} K={wl.K} S={wl.S} H={wl.H} R={wl.R} "
            f"C={wl.C}, {pop}, seed 0{cycle}")


def config_dict(wl, n_gpus: int) -> dict:
    """The ``config`` both arms print for a workload (identical keys and text)."""
    return {"workload": workload_desc(wl), "tokens_per_step_per_gpu": wl.tokens,
            "l2": "the timed loop streams every step's rows through buffers larger than "
                  "L2 (126 MB); the serial loop also flushes L2 before each step",
            "parallelism": f"replicas x{n_gpus}"}


def data_cap_rows(wl) -> int | None:
    """Receive-buffer rows: the water level S*K for the workloads that balance
    (tiny, mid); twice that for the ones whose slots cannot reach it."""
    return None if wl.name in ("tiny", "mid") else 2 * wl.S * wl.K


def algorithmic_bytes(wl) -> dict:
    """Bytes each step must move at least (bf16 rows, int32 indices, fp32 gates)."""
    P, S, K, H = wl.P, wl.S, wl.K, wl.H
    N = P * S * K
    tok_rows = P * S * H * 2
    ent_rows = N * H * 2
    return {
        "plan": 2 * N * 4 + N * 4,
        "dispatch": tok_rows + ent_rows + N * 4,
        "combine": ent_rows + N * 4 + N * 4 + tok_rows,
    }


def read_peaks() -> tuple[float, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash(files) -> str:
    h = hashlib.sha256()
    for name in files:
        with open(os.path.join(ROOT, "token_dispatch_top_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str) -> float | None:
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the kernels as they are now."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("source_hash") != kernel_source_hash(rec.get("source_files", [])):
        return None
    v = rec.get("kernels", {}).get(kernel, {}).get("dram_bytes_per_launch")
    return float(v) if v is not None else None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while timing."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path:
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(parts)
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def max_over_ranks(values, dist, device):
    """Element-wise max of per-rank timings (the slowest rank sets the time)."""
    if dist is None:
        return list(values)
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def weak_scaling_value(tokens_per_rank: int, world: int, total_ms: float, steps: int) -> float:
    """Tokens/s of the whole job: every rank processes its own batch per step,
    and the job takes the slowest rank's time."""
    return tokens_per_rank * world / (total_ms / steps / 1000.0)


def oracle_steps(wl, routes, hidden_bits, budget_s: float, min_steps: int = 1):
    """Full CPU-oracle steps (plan + dispatch + combine) until the budget is
    spent, step k on routes[k mod len(routes)] (ids, w).  Returns (steps,
    seconds)."""
    import oracle
    cfg = oracle.Config(wl.P, wl.E, wl.K, wl.S, wl.H, wl.R, wl.C, wl.gpus_per_node,
                        data_cap_rows(wl))
    buf = np.empty((wl.P, cfg.cap(), wl.H), np.uint16)
    n = 0
    t0 = time.perf_counter()
    while n < min_steps or time.perf_counter() - t0 < budget_s:
        ids, w = routes[n % len(routes)]
        p = oracle.plan(cfg, ids, want_M=False)
        if p["status"] < 0:
            raise RuntimeError(f"oracle plan failed: status {p['status']}")
        oracle.dispatch(cfg, p["dst_row"], hidden_bits, buf)
        oracle.combine(cfg, p["dst_row"], buf.reshape(-1, wl.H), w)
        n += 1
    return n, time.perf_counter() - t0


def oracle_sampled_step(wl, cfg, ids, w, hidden_bits, buf, n_tok):
    """One reference step: the oracle's full plan, then its dispatch and combine
    on the first ``n_tok`` tokens (a bounded sample).  Returns (t_plan, t_data)."""
    import oracle
    t0 = time.perf_counter()
    p = oracle.plan(cfg, ids, want_M=False)
    t1 = time.perf_counter()
    sub = oracle.Config(1, wl.E, wl.K, n_tok, wl.H, 0, 0.0, 1, n_tok * wl.K)
    dst = np.ascontiguousarray(p["dst_row"].reshape(-1, wl.K)[:n_tok]).reshape(1, n_tok, wl.K)
    hid = np.ascontiguousarray(hidden_bits.reshape(-1, wl.H)[:n_tok]).reshape(1, n_tok, wl.H)
    oracle.dispatch(sub, dst, hid, buf)
    oracle.combine(sub, dst, buf.reshape(-1, wl.H), np.ascontiguousarray(
        w.reshape(-1, wl.K)[:n_tok]).reshape(1, n_tok, wl.K))
    return t1 - t0, time.perf_counter() - t1


def run_reference(args, wl, rank, budget_s: float = 120.0):
    """The oracle, as it stands, timed on the host cores.  Every step plans the
    whole batch and moves a bounded sample of its tokens, sized so that the
    warm-up and timed steps together take about ``budget_s``; the step time is
    scaled to the whole batch (plan time + data time per token x tokens)."""
    if rank != 0:
        return
    import oracle
    from token_dispatch_top_b200 import synth
    routes = [synth.routing(wl, 0, st) for st in route_steps(wl)]
    hidden = synth.hidden_bits(wl, 0)
    cfg = oracle.Config(wl.P, wl.E, wl.K, wl.S, wl.H, wl.R, wl.C, wl.gpus_per_node,
                        data_cap_rows(wl))
    buf = np.empty((wl.P, cfg.cap(), wl.H), np.uint16)
    probe = min(1024, wl.tokens)
    tp, td = oracle_sampled_step(wl, cfg, *routes[0], hidden, buf, probe)
    per_step = budget_s / max(1, args.steps + args.warmup)
    n_tok = int(max(64, min(wl.tokens, probe * (per_step - tp) / max(td, 1e-9))))
    for k in range(args.warmup):
        oracle_sampled_step(wl, cfg, *routes[k % len(routes)], hidden, buf, n_tok)
    t_plan = t_data = 0.0
    for k in range(args.steps):
        a, b = oracle_sampled_step(wl, cfg, *routes[k % len(routes)], hidden, buf, n_tok)
        t_plan += a
        t_data += b
    full_step_s = (t_plan + t_data * wl.tokens / n_tok) / args.steps
    value = wl.tokens / full_step_s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * full_step_s, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_dict(wl, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"per step: the full plan plus dispatch and combine of "
                                   f"{n_tok} of {wl.tokens} tokens, scaled to all tokens; "
                                   "single-threaded C"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def plan_timeline(cfg, ids_list, dev, flush_l2, iters=10):
    """The plan's device timeline from its trace (zb_plan_t.trace), each call
    after an L2 flush and a device hold, on a plan object of its own (the
    timed loops run untraced): per kernel, the median microseconds from the
    call's first stamp to its first CTA's start, its release from its
    dependency wait and its last CTA's end."""
    import torch
    from token_dispatch_top_b200 import zb
    tplan = zb.Plan(cfg, dev, with_row_src=False, trace=True)
    runs = []
    for it in range(3 + iters):
        flush_l2()
        torch.cuda._sleep(SLEEP_CYCLES)
        zb.plan(tplan, ids_list[it % len(ids_list)])
        tl = zb.plan_trace(tplan)
        if it >= 3:
            runs.append(tl)
    out = {}
    for k in zb.TRACE_KERNELS:
        if runs[0][k] is None:
            out[k] = None
            continue
        out[k] = {f: statistics.median(r[k][f] for r in runs)
                  for f in ("start", "released", "end")}
    return out


def measure_workload(wl, dev, flush_l2, peak, iters=10, steps=(0,)):
    """One workload's kernels, one invocation at a time (L2 flushed before
    each, outside the events): plan, dispatch and combine times, their HBM
    rates against the measured peak, and the plan's balance.  Drift steps
    rotate through ``steps``, each with its own ids and gates."""
    import torch
    from token_dispatch_top_b200 import metrics, synth, zb
    cfg = zb.Config(P=wl.P, E=wl.E, K=wl.K, S=wl.S, H=wl.H, R=wl.R, C=wl.C,
                    gpus_per_node=wl.gpus_per_node, cap_rows=data_cap_rows(wl))
    P, S, H, cap = cfg.P, cfg.S, cfg.H, cfg.cap
    inputs = []
    for st in steps:
        ids_np, w_np = synth.routing(wl, 0, st)
        inputs.append((torch.from_numpy(ids_np).to(dev), torch.from_numpy(w_np).to(dev)))
    hidden = synth.hidden_device(wl, 0, 0, dev)
    plan = zb.Plan(cfg, dev, with_row_src=False)
    buf = torch.empty((P, cap, H), dtype=torch.bfloat16, device=dev)
    out = torch.empty((P, S, H), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    t_plan, t_disp, t_comb, balance = [], [], [], []
    for it in range(3 + iters):
        ids, w = inputs[it % len(inputs)]
        flush_l2()
        torch.cuda._sleep(SLEEP_CYCLES)  # time the device, not the host's launches
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        ev[0].record(stream)
        zb.plan(plan, ids)
        ev[1].record(stream)
        zb.dispatch(plan, hidden, buf)
        ev[2].record(stream)
        zb.combine(plan, buf, w, out)
        ev[3].record(stream)
        status, _ = zb.plan_status(plan)
        if status < 0:
            raise RuntimeError(f"{wl.name}: plan failed: {zb.strerror(status)}")
        if it >= 3:
            t_plan.append(ev[0].elapsed_time(ev[1]))
            t_disp.append(ev[1].elapsed_time(ev[2]))
            t_comb.append(ev[2].elapsed_time(ev[3]))
        if it < len(inputs):
            m = metrics.plan_metrics(plan)
            balance.append({"step": steps[it], "status": status,
                            "r_imb_before": m["r_imb_before"], "r_imb_after": m["r_imb_after"],
                            "max_load_over_T": int(plan.stats[zb.STAT_MAX_LOAD]) /
                            max(1, int(plan.stats[zb.STAT_WATER_LEVEL]))})
    ab = algorithmic_bytes(wl)
    d, c, pl = (statistics.median(t_disp), statistics.median(t_comb),
                statistics.median(t_plan))
    rec = {"workload": workload_desc(wl), "cap_rows": cap, "steps": list(steps),
           "iterations": iters, "plan_us": 1000.0 * pl,
           "dispatch": {"ms": d, "gbs": ab["dispatch"] / d / 1e6,
                        "frac": ab["dispatch"] / d / 1e6 / peak,
                        "algorithmic_bytes": ab["dispatch"]},
           "combine": {"ms": c, "gbs": ab["combine"] / c / 1e6,
                       "frac": ab["combine"] / c / 1e6 / peak,
                       "algorithmic_bytes": ab["combine"],
                       "kernel": "k_combine_wide (32-byte loads)"
                       if wl.K in (7, 8) and wl.H >= 4096 else "k_combine"},
           "plan_timeline_us": plan_timeline(cfg, [x for x, _ in inputs], dev, flush_l2),
           "tokens_per_s": wl.tokens / ((pl + d + c) / 1000.0),
           "balance": balance}
    del plan, buf, out, hidden, inputs
    torch.cuda.empty_cache()
    return rec


def measure_rank_path(wl, dev, flush_l2, peak, iters=5):
    """The form one rank of P GPUs runs, its P ranks one after another on this
    GPU: per rank, zb.count on its own ids, zb.plan_rank from the stacked
    count rows (what the all-gather between GPUs yields), and zb.dispatch_rank /
    zb.combine_rank through the table of P buffer pointers, here P parts of
    one allocation.  count and plan_rank are timed one call at a time; the
    P dispatch_rank calls, and then the P combine_rank calls, are timed back
    to back inside one pair of events, since one call alone (about 25 us on
    mid) is short beside the events' own overhead.  L2 is flushed before
    each timed region, outside its events.  Every rank's dst_row and
    combined rows must equal the whole-batch path's."""
    import numpy as np
    import torch
    from token_dispatch_top_b200 import synth, zb
    cfg = zb.Config(P=wl.P, E=wl.E, K=wl.K, S=wl.S, H=wl.H, R=wl.R, C=wl.C,
                    gpus_per_node=wl.gpus_per_node, cap_rows=data_cap_rows(wl))
    P, S, H, cap = cfg.P, cfg.S, cfg.H, cfg.cap
    ids_np, w_np = synth.routing(wl, 0)
    ids_all = torch.from_numpy(ids_np).to(dev)
    w_all = torch.from_numpy(w_np).to(dev)
    hidden = synth.hidden_device(wl, 0, 0, dev)
    ids = [ids_all[r] for r in range(P)]
    rps = [zb.RankPlan(cfg, r, dev) for r in range(P)]
    buf = torch.empty((P, cap, H), dtype=torch.bfloat16, device=dev)
    bufs = list(buf.unbind(0))
    out = torch.empty((P, S, H), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def timed(fn):
        flush_l2()
        torch.cuda._sleep(SLEEP_CYCLES)  # time the device, not the host's launches
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        return a.elapsed_time(b)

    def dispatch_all():
        for r in range(P):
            zb.dispatch_rank(rps[r], hidden[r], bufs)

    def combine_all():
        for r in range(P):
            zb.combine_rank(rps[r], bufs, w_all[r], out[r])

    t = {"count": [], "plan_rank": [], "dispatch_rank": [], "combine_rank": []}
    for it in range(1 + iters):
        tc = [timed(lambda r=r: zb.count(rps[r], ids[r])) for r in range(P)]
        table = torch.stack([rp.counts for rp in rps])  # the exchange (not timed)
        for rp in rps:
            rp.table.copy_(table)
        tp = [timed(lambda r=r: zb.plan_rank(rps[r], ids[r])) for r in range(P)]
        for rp in rps:
            status, _ = zb.plan_status(rp)
            if status < 0:
                raise RuntimeError(f"rank plan failed: {zb.strerror(status)}")
        td = timed(dispatch_all)
        tk = timed(combine_all)
        if it >= 1:
            t["count"].extend(tc)
            t["plan_rank"].extend(tp)
            t["dispatch_rank"].append(td)
            t["combine_rank"].append(tk)
    # the whole-batch path on the same inputs: the same rows, bit for bit
    whole = zb.Plan(cfg, dev, with_row_src=False)
    zb.plan(whole, ids_all)
    wbuf = torch.empty_like(buf)
    wout = torch.empty_like(out)
    zb.dispatch(whole, hidden, wbuf)
    zb.combine(whole, wbuf, w_all, wout)
    same = all(torch.equal(rps[r].dst_row, whole.dst_row[r]) for r in range(P)) and \
        torch.equal(out.view(torch.int16), wout.view(torch.int16))
    if not same:
        raise RuntimeError("per-rank path differs from the whole-batch path")
    ab = algorithmic_bytes(wl)  # summed over the P ranks: the same bytes
    d, c = statistics.median(t["dispatch_rank"]), statistics.median(t["combine_rank"])
    rec = {"what": "the per-rank entry points of the P-GPU form, its P ranks run one after "
                   "another on one GPU, buffers addressed through the P-pointer table; "
                   "not part of the step",
           "workload": workload_desc(wl), "iterations": iters,
           "count_us_per_rank": 1000.0 * statistics.median(t["count"]),
           "plan_rank_us_per_rank": 1000.0 * statistics.median(t["plan_rank"]),
           "dispatch_rank": {"ms_all_ranks": d, "gbs": ab["dispatch"] / d / 1e6,
                             "frac": ab["dispatch"] / d / 1e6 / peak},
           "combine_rank": {"ms_all_ranks": c, "gbs": ab["combine"] / c / 1e6,
                            "frac": ab["combine"] / c / 1e6 / peak},
           "same_rows_as_whole_batch": bool(same)}
    del rps, buf, bufs, out, wbuf, wout, whole, hidden
    torch.cuda.empty_cache()
    return rec


def run_ours(args, wl, rank, world, local_rank):
    import torch
    from token_dispatch_top_b200 import build, synth, zb

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    build.build()
    zb.load()
    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        dist = dist_mod

    seed = rank
    routes_np = [synth.routing(wl, seed, st) for st in route_steps(wl)]
    n_routes = len(routes_np)
    ids_np, w_np = routes_np[0]
    hidden_np = synth.hidden_bits(wl, seed)
    cfg = zb.Config(P=wl.P, E=wl.E, K=wl.K, S=wl.S, H=wl.H, R=wl.R, C=wl.C,
                    gpus_per_node=wl.gpus_per_node, cap_rows=data_cap_rows(wl))
    P, S, K, H, cap = cfg.P, cfg.S, cfg.K, cfg.H, cfg.cap

    ids_l = [torch.from_numpy(a).to(dev) for a, _ in routes_np]
    w_l = [torch.from_numpy(b).to(dev) for _, b in routes_np]
    ids, w = ids_l[0], w_l[0]  # the step-0 draw, for the checks and extras
    hidden = torch.from_numpy(hidden_np.view(np.int16)).to(dev).view(torch.bfloat16)
    plan = zb.Plan(cfg, dev, with_row_src=False)
    buf = torch.empty((P, cap, H), dtype=torch.bfloat16, device=dev)
    out = torch.empty((P, S, H), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    flush_src = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        # write a buffer twice the size of L2, then read another one, so the
        # step starts with L2 holding only clean lines of no use to it
        flush.zero_()
        torch.sum(flush_src, dim=0, out=flush_sink)

    stream = torch.cuda.current_stream()

    def hold_device():
        # keep the device busy (a bounded spin, about 0.1 ms) while the host
        # enqueues the step that follows, so that its events time the
        # device's work and not the host's launch overhead
        torch.cuda._sleep(SLEEP_CYCLES)

    def step(k=0):
        zb.plan(plan, ids_l[k % n_routes])
        zb.dispatch(plan, hidden, buf)
        zb.combine(plan, buf, w_l[k % n_routes], out)

    # every draw's plan must fit the receive buffers
    for k in range(n_routes):
        step(k)
        status, max_load = zb.plan_status(plan)
        if status < 0:
            raise RuntimeError(f"plan failed: {zb.strerror(status)}")

    def barrier():
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()

    for k in range(args.warmup):
        flush_l2()
        step(k)
    barrier()
    n_ev = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_ev)]
    # ---- serial steps, L2 flushed before each (outside the timing): the
    # latency of one invocation and of each kernel
    barrier()
    for k in range(args.steps):
        flush_l2()
        hold_device()
        ev[k][0].record(stream)
        zb.plan(plan, ids_l[k % n_routes])
        ev[k][1].record(stream)
        zb.dispatch(plan, hidden, buf)
        ev[k][2].record(stream)
        zb.combine(plan, buf, w_l[k % n_routes], out)
        ev[k][3].record(stream)
    barrier()
    status, _ = zb.plan_status(plan)
    if status < 0:
        raise RuntimeError(f"plan failed: {zb.strerror(status)}")
    t_plan = [ev[k][0].elapsed_time(ev[k][1]) for k in range(n_ev)]
    t_disp = [ev[k][1].elapsed_time(ev[k][2]) for k in range(n_ev)]
    t_comb = [ev[k][2].elapsed_time(ev[k][3]) for k in range(n_ev)]
    serial_ms = sum(ev[k][0].elapsed_time(ev[k][3]) for k in range(n_ev))  # total over K steps

    # ---- the headline: steps pipelined two deep.  Consecutive invocations are
    # independent, so the plan of step k+1 runs on its own higher-priority
    # stream while the rows of step k move (the plan is latency-bound and
    # leaves HBM idle; dispatch and combine are HBM-bound).  Two slots of plan,
    # receive and output buffers; every step still runs all six kernels.  No
    # L2 flush: each step streams 1.9 GB through buffers larger than L2.
    s_rows = torch.cuda.Stream(device=dev)
    s_plan = torch.cuda.Stream(device=dev, priority=-1)
    plans2 = [plan, zb.Plan(cfg, dev, with_row_src=False)]
    bufs2 = [buf, torch.empty_like(buf)]
    outs2 = [out, torch.empty_like(out)]
    plan_done = [torch.cuda.Event() for _ in range(2)]
    rows_done = [torch.cuda.Event() for _ in range(2)]

    def pipelined(n, pev=None):
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(s_rows)
        s_plan.wait_stream(s_rows)
        for k in range(n):
            sl = k % 2
            with torch.cuda.stream(s_plan):
                if k >= 2:
                    s_plan.wait_event(rows_done[sl])  # step k-2 is done with the slot
                if pev is not None:
                    pev[k][0].record(s_plan)
                zb.plan(plans2[sl], ids_l[k % n_routes])
                if pev is not None:
                    pev[k][1].record(s_plan)
                plan_done[sl].record(s_plan)
            with torch.cuda.stream(s_rows):
                s_rows.wait_event(plan_done[sl])
                if pev is not None:
                    pev[k][2].record(s_rows)
                zb.dispatch(plans2[sl], hidden, bufs2[sl])
                if pev is not None:
                    pev[k][3].record(s_rows)
                zb.combine(plans2[sl], bufs2[sl], w_l[k % n_routes], outs2[sl])
                if pev is not None:
                    pev[k][4].record(s_rows)
                rows_done[sl].record(s_rows)
        end.record(s_rows)
        return start, end

    pipelined(args.warmup)
    barrier()
    pev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(n_ev)]
    with ClockSampler(local_rank) as clocks:
        barrier()
        t0 = time.perf_counter()
        p_start, p_end = pipelined(args.steps, pev)
        barrier()
        wall = time.perf_counter() - t0
    for pl_ in plans2:
        st_, _ = zb.plan_status(pl_)
        if st_ < 0:
            raise RuntimeError(f"plan failed in the pipelined loop: {zb.strerror(st_)}")
    # the last step's output against the same step run alone (into an output
    # of its own: plan, buf and out are pipeline slot 0's)
    last = args.steps - 1
    chk = torch.empty_like(out)
    zb.plan(plan, ids_l[last % n_routes])
    zb.dispatch(plan, hidden, buf)
    zb.combine(plan, buf, w_l[last % n_routes], chk)
    if not torch.equal(outs2[last % 2].view(torch.int16), chk.view(torch.int16)):
        raise RuntimeError("the pipelined loop's output differs from a serial step")
    del chk
    step_ms = p_start.elapsed_time(p_end)  # total over K steps
    p_plan = [pev[k][0].elapsed_time(pev[k][1]) for k in range(n_ev)]
    p_disp = [pev[k][2].elapsed_time(pev[k][3]) for k in range(n_ev)]
    p_comb = [pev[k][3].elapsed_time(pev[k][4]) for k in range(n_ev)]
    del plans2, bufs2, outs2

    # ---- the merged dispatch (Zepp 4.2 merge), timed apart from the step: one
    # row per (token, destination rank) instead of one per (token, k)
    merged = zb.Merge(cfg, dev)
    tbuf = torch.empty_like(buf)
    zb.plan(plan, ids)
    zb.merge(plan, merged)
    zb.dispatch_merged(plan, merged, hidden, tbuf)
    torch.cuda.synchronize()
    m_ms, d_ms = [], []
    for _ in range(max(20, min(args.steps, 100))):
        flush_l2()
        hold_device()
        a0, a1, a2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a0.record(stream)
        zb.merge(plan, merged)
        a1.record(stream)
        zb.dispatch_merged(plan, merged, hidden, tbuf)
        a2.record(stream)
        a2.synchronize()
        m_ms.append(a0.elapsed_time(a1))
        d_ms.append(a1.elapsed_time(a2))
    rows_merged = int(merged.tok_cnt.sum())
    # the merged combine: pre-reduce per (token, rank) into bf16 partials, then
    # add the partials per token; y = the dispatched rows (identity experts)
    part = torch.empty_like(buf)
    out_m = torch.empty((P, S, H), dtype=torch.bfloat16, device=dev)
    zb.dispatch(plan, hidden, buf)
    zb.combine_reduce(plan, merged, buf, w, part)
    zb.combine_merged(plan, merged, part, out_m)
    torch.cuda.synchronize()
    cr_ms, cm_ms = [], []
    for _ in range(max(20, min(args.steps, 100))):
        flush_l2()
        hold_device()
        a0, a1, a2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a0.record(stream)
        zb.combine_reduce(plan, merged, buf, w, part)
        a1.record(stream)
        zb.combine_merged(plan, merged, part, out_m)
        a2.record(stream)
        a2.synchronize()
        cr_ms.append(a0.elapsed_time(a1))
        cm_ms.append(a1.elapsed_time(a2))
    del tbuf, part, out_m

    # ---- the banded plan (eq. (1) with its C band in use), timed apart from
    # the step: the same ids planned with relax = 1 and floor((1+C) S*K) rows
    cfg_b = dataclasses.replace(cfg, relax=1, cap_rows=None)
    plan_b = zb.Plan(cfg_b, dev, with_row_src=False)
    zb.plan(plan_b, ids)
    torch.cuda.synchronize()
    b_ms = []
    for _ in range(max(20, min(args.steps, 100))):
        flush_l2()
        hold_device()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        zb.plan(plan_b, ids)
        a1.record(stream)
        a1.synchronize()
        b_ms.append(a0.elapsed_time(a1))
    st_b = plan_b.stats.cpu().numpy()
    st_x = plan.stats.cpu().numpy()
    banded = {
        "what": f"plan with relax = 1, C = {cfg.C}: hosts receive q +- floor(C q) rows "
                "(Zepp 4.1 eq. (1)); not part of the step",
        "status": int(st_b[zb.STAT_STATUS]), "plan_ms": statistics.median(b_ms),
        "cap_rows": cfg_b.cap, "max_load": int(st_b[zb.STAT_MAX_LOAD]),
        "locality_cost": int(st_b[zb.STAT_LOCALITY_COST]),
        "locality_cost_exact": int(st_x[zb.STAT_LOCALITY_COST])}
    del plan_b

    # ---- quota repair (HALO-Q stage 4) on a kept placement that puts the
    # R = 4 hottest foreign experts on every rank, timed apart from the step
    R4 = min(4, wl.P - 1)
    Te = np.bincount(ids_np.ravel(), minlength=wl.E)
    pl_np = np.full((wl.P, R4), -1, np.int32)
    for j in range(wl.P):
        hot = [e for e in np.argsort(-Te, kind="stable") if e // (wl.E // wl.P) != j][:R4]
        pl_np[j, :len(hot)] = hot
    pl_d = torch.from_numpy(pl_np).to(dev)
    rep = {"what": f"zb_plan_placed with every rank holding the {R4} hottest foreign experts, "
                   "without and with quota repair (ISER-MoE HALO-Q stage 4); not part of the step"}
    for tag, flag in (("kept", 0), ("repaired", 1)):
        cfg_r = dataclasses.replace(cfg, R=R4, repair=flag, cap_rows=2 * wl.S * wl.K)
        plan_r = zb.Plan(cfg_r, dev, with_row_src=False)
        zb.plan_placed(plan_r, ids, pl_d)
        torch.cuda.synchronize()
        r_ms = []
        for _ in range(max(20, min(args.steps, 100))):
            flush_l2()
            hold_device()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            zb.plan_placed(plan_r, ids, pl_d)
            a1.record(stream)
            a1.synchronize()
            r_ms.append(a0.elapsed_time(a1))
        st_r = plan_r.stats.cpu().numpy()
        rep[tag] = {"status": int(st_r[zb.STAT_STATUS]), "plan_ms": statistics.median(r_ms),
                    "locality_cost": int(st_r[zb.STAT_LOCALITY_COST]),
                    "rows_repaired": int(st_r[zb.STAT_REPAIRED])}
        del plan_r

    # ---- end to end through the public API, pinned host buffers.  Every step
    # copies its ids, gates and hidden rows host->device, runs plan, dispatch
    # and combine, and copies its combined rows and plan status back.  Copies
    # run on their own streams with three buffer slots, so one step's input
    # copy overlaps the previous step's output copy (the host link is full
    # duplex); compute stays in order on the compute stream.
    ids_h = [torch.from_numpy(a).pin_memory() for a, _ in routes_np]
    w_h = [torch.from_numpy(b).pin_memory() for _, b in routes_np]
    hid_h = torch.from_numpy(hidden_np.view(np.int16)).pin_memory()
    n_slots = 3
    out_h = [torch.empty((P, S, H), dtype=torch.int16).pin_memory() for _ in range(n_slots)]
    stats_h = torch.empty((max(args.steps, args.warmup), zb.STATS_LEN),
                          dtype=torch.int64).pin_memory()
    ids_d = [torch.empty_like(ids) for _ in range(n_slots)]
    w_d = [torch.empty_like(w) for _ in range(n_slots)]
    hid_d = [torch.empty((P, S, H), dtype=torch.int16, device=dev) for _ in range(n_slots)]
    out_d = [torch.empty((P, S, H), dtype=torch.bfloat16, device=dev) for _ in range(n_slots)]
    plans = [zb.Plan(cfg, dev, with_row_src=False) for _ in range(n_slots)]
    h2d_s = torch.cuda.Stream(device=dev)
    d2h_s = torch.cuda.Stream(device=dev)
    comp_s = stream

    def e2e_run(n_steps):
        h2d_done = [torch.cuda.Event() for _ in range(n_slots)]
        comp_done = [torch.cuda.Event() for _ in range(n_slots)]
        d2h_done = [torch.cuda.Event() for _ in range(n_slots)]
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(comp_s)
        h2d_s.wait_event(t0)
        for k in range(n_steps):
            sl = k % n_slots
            with torch.cuda.stream(h2d_s):
                if k >= n_slots:
                    h2d_s.wait_event(comp_done[sl])  # slot's inputs consumed
                ids_d[sl].copy_(ids_h[k % n_routes], non_blocking=True)
                w_d[sl].copy_(w_h[k % n_routes], non_blocking=True)
                hid_d[sl].copy_(hid_h, non_blocking=True)
                h2d_done[sl].record(h2d_s)
            comp_s.wait_event(h2d_done[sl])
            if k >= n_slots:
                comp_s.wait_event(d2h_done[sl])  # slot's output read back
            with torch.cuda.stream(comp_s):
                zb.plan(plans[sl], ids_d[sl])
                zb.dispatch(plans[sl], hid_d[sl].view(torch.bfloat16), buf)
                zb.combine(plans[sl], buf, w_d[sl], out_d[sl])
                comp_done[sl].record(comp_s)
            d2h_s.wait_event(comp_done[sl])
            with torch.cuda.stream(d2h_s):
                out_h[sl].copy_(out_d[sl].view(torch.int16), non_blocking=True)
                stats_h[k].copy_(plans[sl].stats, non_blocking=True)
                d2h_done[sl].record(d2h_s)
        for ev in d2h_done:
            comp_s.wait_event(ev)
        t1.record(comp_s)
        t1.synchronize()
        if int(stats_h[:n_steps, zb.STAT_STATUS].min()) < 0:
            raise RuntimeError("plan failed in the end-to-end loop")
        return t0.elapsed_time(t1)

    e2e_run(args.warmup)
    barrier()
    e2e_ms = e2e_run(args.steps)
    barrier()
    h2d = ids_np.nbytes + w_np.nbytes + hidden_np.nbytes
    d2h = P * S * H * 2 + zb.STATS_LEN * 8

    # ---- the other workloads, one invocation at a time (N = 1 only): plan
    # latency, dispatch and combine rates, balance
    workloads = {}
    rank_path = None
    event_floor_us = None
    timeline = None
    if world == 1 and args.extras:
        peak_gbs, _ = read_peaks()
        torch.cuda.empty_cache()
        for name in ("tiny", "mid", "hot", "hier", "drift"):
            if name == wl.name:
                continue
            steps = (0, 31, 63) if name == "drift" else (0,)
            workloads[name] = measure_workload(synth.WORKLOADS[name], dev, flush_l2, peak_gbs,
                                               steps=steps)
        # the per-rank entry points of the P-GPU form on this workload
        rank_path = measure_rank_path(wl, dev, flush_l2, peak_gbs)
        timeline = plan_timeline(cfg, ids_l, dev, flush_l2)
        # what the same flush, hold and event pair read around the shortest
        # kernel there is (a one-element fill): the floor under every plan
        # latency above
        one = torch.zeros(1, dtype=torch.int32, device=dev)
        floor = []
        for k in range(13):
            flush_l2()
            hold_device()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            one.fill_(k)
            b.record(stream)
            b.synchronize()
            if k >= 3:
                floor.append(a.elapsed_time(b))
        event_floor_us = 1000.0 * statistics.median(floor)

    # ---- max over ranks
    (step_ms, e2e_ms, disp_ms, comb_ms, plan_ms, serial_ms, s_disp_ms, s_comb_ms,
     s_plan_ms) = max_over_ranks(
        [step_ms, e2e_ms, sum(p_disp), sum(p_comb), sum(p_plan), serial_ms, sum(t_disp),
         sum(t_comb), sum(t_plan)], dist, dev)
    if rank != 0:
        return

    ms_per_step = step_ms / args.steps
    value = weak_scaling_value(wl.tokens, world, step_ms, args.steps)
    e2e_value = weak_scaling_value(wl.tokens, world, e2e_ms, args.steps)
    ab = algorithmic_bytes(wl)
    disp_ms_avg = disp_ms / args.steps
    comb_ms_avg = comb_ms / args.steps
    dom, dom_ms = ("k_combine", comb_ms_avg) if comb_ms_avg >= disp_ms_avg else \
        ("k_dispatch", disp_ms_avg)
    dom_bytes = ab["combine"] if dom == "k_combine" else ab["dispatch"]
    peak, peak_kind = read_peaks()
    achieved = dom_bytes / (dom_ms / 1000.0) / 1e9
    traffic = recorded_traffic(dom)

    cpu = None
    if world == 1:
        n, sec = oracle_steps(wl, routes_np, hidden_np, budget_s=10.0)
        cpu = {"value": wl.tokens * n / sec, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"{n} full steps (plan+dispatch+combine) of the same workload, "
                         "single-threaded C"}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": config_dict(wl, world),
        "method": {"accumulate": "f32", "experts": "identity (y = dispatched rows)",
                   "pipeline": "two steps in flight: the plan of step k+1 runs on a "
                               "high-priority stream while the rows of step k move; two "
                               "slots of plan, receive and output buffers",
                   "l2": f"not flushed in the timed (pipelined) loop: every step streams "
                         f"{sum(algorithmic_bytes(wl).values()) / 1e9:.2f} GB through buffers "
                         f"larger than L2; the serial loop flushes before every step"},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "method": "pinned host buffers; per step H2D of ids, gates and hidden, "
                          "plan+dispatch+combine, D2H of out and status; copies on two "
                          "streams with three slots (input copy of step k+1 overlaps output "
                          "copy of step k); no L2 flush: each step moves 270 MB over the "
                          "host link and 1.9 GB through HBM"},
        # per step: k_zero, k_hist, k_planner, k_assign, k_dispatch, k_combine
        "gpu_launches": 6 * args.steps,
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "algorithmic_bytes": dom_bytes},
        "kernels_ms": {"plan": plan_ms / args.steps, "dispatch": disp_ms_avg,
                       "combine": comb_ms_avg,
                       "note": "in the pipelined loop; the plan overlaps the previous "
                               "step's rows"},
        "serial": {"what": "one step at a time on one stream, L2 flushed before each "
                           "(outside the timing), its kernels enqueued before it starts: "
                           "the device latency of an invocation",
                   "ms_per_step": serial_ms / args.steps,
                   "value": weak_scaling_value(wl.tokens, world, serial_ms, args.steps),
                   "kernels_ms": {"plan": s_plan_ms / args.steps,
                                  "dispatch": s_disp_ms / args.steps,
                                  "combine": s_comb_ms / args.steps}},
        "kernels_gbs": {"dispatch": ab["dispatch"] / disp_ms_avg / 1e6,
                        "combine": ab["combine"] / comb_ms_avg / 1e6},
        "extras": {"merged_dispatch": {
            "what": "one row per (token, destination rank), Zepp 4.2 merge; not part of the step",
            "rows_written": rows_merged, "rows_plain": wl.N,
            "merge_plan_ms": statistics.median(m_ms),
            "dispatch_ms": statistics.median(d_ms),
            "dispatch_gbs": (wl.tokens * wl.H * 2 + rows_merged * wl.H * 2 + wl.N * 4)
            / statistics.median(d_ms) / 1e6},
            "merged_combine": {
                "what": "Zepp 4.2 merge for combine: a bf16 partial per (token, rank), then "
                        "the partials added per token; not part of the step",
                "reduce_ms": statistics.median(cr_ms),
                "reduce_gbs": (wl.N * (wl.H * 2 + 12) + rows_merged * wl.H * 2)
                / statistics.median(cr_ms) / 1e6,
                "combine_ms": statistics.median(cm_ms),
                "combine_gbs": (rows_merged * wl.H * 2 + wl.N * 4 + wl.tokens * wl.H * 2)
                / statistics.median(cm_ms) / 1e6},
            "banded_plan": banded, "quota_repair": rep,
            "workloads": workloads, "rank_path": rank_path,
            "event_floor_us": {"what": "a one-element fill timed like the plan (L2 flushed, "
                                       "device held, one event pair): the events' own "
                                       "floor under plan_latency_us",
                               "value": event_floor_us}},
        "plan_latency_us": dict({wl.name: 1000.0 * s_plan_ms / args.steps},
                                **{k: v["plan_us"] for k, v in workloads.items()}),
        "plan_timeline_us": dict({wl.name: timeline} if timeline else {},
                                 **{k: v["plan_timeline_us"] for k, v in workloads.items()}),
        "wall_s": wall,
        "clocks": clocks.summary(),
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["tiny", "mid", "hot", "hier", "drift"],
                    default=WORKLOAD, help="the headline workload (default: mid)")
    ap.add_argument("--no-extras", dest="extras", action="store_false",
                    help="skip the per-workload records of the other workloads")
    args = ap.parse_args()
    if args.steps < 1:
        ap.error("--steps must be at least 1")
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be at least 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    from token_dispatch_top_b200 import synth
    wl = synth.WORKLOADS[args.workload]

    if args.impl == "reference":
        run_reference(args, wl, rank)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
        try:
            run_ours(args, wl, rank, world, local_rank)
        finally:
            dist.destroy_process_group()
    else:
        run_ours(args, wl, rank, world, local_rank)


if __name__ == "__main__":
    main()
