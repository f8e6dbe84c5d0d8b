"""Helpers of the GPU parity tests: run the device path through the C ABI (via
the thin binding) and the CPU oracle on the same seeded inputs, and compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from token_dispatch_top_b200 import synth, zb

PLAN_KEYS = ("cnt", "rep_expert", "rep_quota", "home_quota", "load_before", "load_after",
             "cu_seqlens")
SENTINEL = 0x7E11  # bf16 bit pattern marking rows nobody may write


def cfgs(wl: synth.Workload, cap_rows=None, policy=0, relax=0, C=None, repair=0):
    kw = dict(P=wl.P, E=wl.E, K=wl.K, S=wl.S, H=wl.H, R=wl.R, C=wl.C if C is None else C,
              gpus_per_node=wl.gpus_per_node, cap_rows=cap_rows, policy=policy, relax=relax,
              repair=repair)
    return zb.Config(**kw), oracle.Config(**kw)


def bits_to_bf16(bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device) \
        .view(torch.bfloat16)


def bf16_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def gpu_plan(cfg: zb.Config, ids: np.ndarray, device, with_row_src=True):
    p = zb.Plan(cfg, device, with_row_src=with_row_src)
    ids_d = torch.from_numpy(np.ascontiguousarray(ids, dtype=np.int32)).to(device)
    zb.plan(p, ids_d)
    status, max_load = zb.plan_status(p)
    return p, status, max_load


def plan_tables(p: zb.Plan) -> dict:
    out = {k: getattr(p, k).cpu().numpy() for k in PLAN_KEYS}
    out["dst_row"] = p.dst_row.cpu().numpy()
    if p.row_src is not None:
        out["row_src"] = p.row_src.cpu().numpy()
    out["stats"] = p.stats.cpu().numpy()
    return out


def assert_plan_equal(g: dict, o: dict, status: int, rows=True):
    assert status == o["status"], (status, o["status"])
    if status == oracle.ERR_BAD_ID:
        return
    st = g["stats"]
    assert st[zb.STAT_MAX_LOAD] == o["max_load"]
    assert st[zb.STAT_WATER_LEVEL] == o["T"]
    assert st[zb.STAT_N_REPLICAS] == o["n_replicas"]
    assert st[zb.STAT_N_ITERS] == o["n_iters"]
    assert st[zb.STAT_REPAIRED] == o["repaired"]
    for k in PLAN_KEYS:
        np.testing.assert_array_equal(g[k], o[k], err_msg=k)
    if status >= 0:
        assert st[zb.STAT_LOCALITY_COST] == o["locality_cost"]
        if rows:
            np.testing.assert_array_equal(g["dst_row"], o["dst_row"], err_msg="dst_row")
            if "row_src" in g:
                np.testing.assert_array_equal(g["row_src"], o["row_src"], err_msg="row_src")


def used_rows_mask(cfg, load_after) -> np.ndarray:
    """[P,cap] True where a row lies below its rank's load."""
    return np.arange(cfg.cap)[None, :] < np.asarray(load_after)[:, None]
