"""bench.py's roofline inputs, on CPU.

* algorithmic_bytes on the mid workload equals the per-step figures stated in
  the design notes (940.3 MB dispatch, 941.1 MB combine) and the closed forms
  P*S*H*2 + N*H*2 + 4N and N*H*2 + 8N + P*S*H*2, recomputed here.
* recorded_traffic reports the committed ncu DRAM bytes only while the sources
  they were measured on hash to the recorded value, and None for a changed
  source, a missing file or an unknown kernel.
* the peak comes from the measured peaks file when present.
* a drifting workload cycles through 8 draws of its walk, and the CPU
  baseline plans with the same receive buffers as the GPU arm.
"""
import json
import os

import bench
from token_dispatch_top_b200 import synth


def test_algorithmic_bytes_mid():
    wl = synth.WORKLOADS["mid"]
    P, S, K, H = wl.P, wl.S, wl.K, wl.H
    N = P * S * K
    ab = bench.algorithmic_bytes(wl)
    assert ab["dispatch"] == P * S * H * 2 + N * H * 2 + 4 * N == 940_310_528
    assert ab["combine"] == N * H * 2 + 8 * N + P * S * H * 2 == 941_096_960
    assert ab["plan"] == 12 * N


def test_recorded_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    current = rec["source_hash"] == bench.kernel_source_hash(rec["source_files"])
    want = rec["kernels"]["k_dispatch"]["dram_bytes_per_launch"] if current else None
    assert bench.recorded_traffic("k_dispatch") == want
    assert bench.recorded_traffic("k_nothing") is None
    # a copy of the tree with the recorded sources: the record applies
    same = tmp_path / "same"
    (same / "token_dispatch_top_b200" / "csrc").mkdir(parents=True)
    for name in rec["source_files"]:
        data = open(os.path.join(bench.ROOT, "token_dispatch_top_b200", "csrc", name)).read()
        (same / "token_dispatch_top_b200" / "csrc" / name).write_text(data)
    (same / "profiles").mkdir()
    rec_same = dict(rec, source_hash=None)
    monkeypatch.setattr(bench, "ROOT", str(same))
    rec_same["source_hash"] = bench.kernel_source_hash(rec["source_files"])
    (same / "profiles" / "traffic.json").write_text(json.dumps(rec_same))
    assert bench.recorded_traffic("k_dispatch") == rec["kernels"]["k_dispatch"][
        "dram_bytes_per_launch"]
    monkeypatch.undo()
    # a copy of the tree whose kernel source differs: the record no longer applies
    csrc = tmp_path / "token_dispatch_top_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in rec["source_files"]:
        data = open(os.path.join(bench.ROOT, "token_dispatch_top_b200", "csrc", name)).read()
        (csrc / name).write_text(data + "\n// changed\n")
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("k_dispatch") is None
    (tmp_path / "profiles" / "traffic.json").unlink()
    assert bench.recorded_traffic("k_dispatch") is None


def test_peak_from_measured_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.read_peaks() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6508.8}))
    assert bench.read_peaks() == (6508.8, "measured")


def test_route_steps_and_the_shared_config():
    """A drifting workload cycles through 8 draws of its walk; the others use
    one.  Both arms print the same config dict, which names the cycle."""
    assert bench.route_steps(synth.WORKLOADS["mid"]) == (0,)
    drift = synth.WORKLOADS["drift"]
    assert bench.route_steps(drift) == tuple(range(0, 64, 8))
    assert "re-plans on walk step 8*(k mod 8)" in bench.config_dict(drift, 1)["workload"]
    assert bench.config_dict(drift, 2) == bench.config_dict(drift, 2)


def test_oracle_steps_use_the_runs_buffers():
    """The CPU baseline plans with the same receive buffers as the GPU arm:
    on a workload the slots cannot balance to S*K rows (cap_rows = 2*S*K), a
    plan at S*K rows would fail and move nothing."""
    import dataclasses
    hot = synth.WORKLOADS["hot"]
    small = dataclasses.replace(hot, S=64, H=64)
    import oracle
    routes = [synth.routing(small, 0)]
    at_sk = oracle.Config(small.P, small.E, small.K, small.S, small.H, small.R, small.C,
                          small.gpus_per_node, None)
    assert oracle.plan(at_sk, routes[0][0], want_M=False)["status"] == oracle.ERR_CAPACITY
    assert bench.data_cap_rows(small) == 2 * small.S * small.K
    n, sec = bench.oracle_steps(small, routes, synth.hidden_bits(small, 0), budget_s=0.0)
    assert n == 1 and sec >= 0.0  # the baseline's plan fits (it raises otherwise)
