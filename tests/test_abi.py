"""The C ABI without a GPU: the library builds, loads, exports every entry
point include/zb.h declares, and its host-side logic (validation, workspace
sizing, status text, argument checks) behaves as documented.  No call here
touches a device."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import oracle
from token_dispatch_top_b200 import build, zb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return zb.load()


def _declared():
    text = open(os.path.join(ROOT, "include", "zb.h")).read()
    return sorted(set(re.findall(r"ZB_API\s+[\w\s\*]*?\b(zb_\w+)\s*\(", text)))


def test_exports_match_header(lib):
    declared = _declared()
    assert set(declared) >= set(zb.EXPORTS)
    out = subprocess.check_output(["nm", "-D", "--defined-only", zb.LIB_PATH], text=True)
    exported = sorted(line.split()[-1] for line in out.splitlines()
                      if line.split()[-1].startswith("zb_"))
    assert exported == declared
    for name in declared:
        assert hasattr(lib, name)


def test_debug_library_exports_the_same_and_release_keeps_no_record(lib):
    """libzb_debug.so (the bounds-checked build) exports what the header
    declares; zb_debug_read answers ZB_ERR_INVALID in the release library,
    and for a NULL record in the debug one, before touching a device."""
    dbg = build.build(debug=True)
    out = subprocess.check_output(["nm", "-D", "--defined-only", dbg], text=True)
    exported = sorted(line.split()[-1] for line in out.splitlines()
                      if line.split()[-1].startswith("zb_"))
    assert exported == _declared()
    rec = zb._DebugRecord()
    release = ctypes.CDLL(build.LIB)
    assert release.zb_debug_read(ctypes.byref(rec), 1) == zb.ERR_INVALID
    assert ctypes.CDLL(dbg).zb_debug_read(None, 0) == zb.ERR_INVALID
    assert ctypes.sizeof(zb._DebugRecord) == 32


def test_strerror(lib):
    for code in (zb.OK, zb.WARN_UNBALANCED, zb.ERR_INVALID, zb.ERR_CAPACITY, zb.ERR_BAD_ID,
                 zb.ERR_TIMEOUT, zb.ERR_CUDA, 12345):
        assert isinstance(zb.strerror(code), str) and zb.strerror(code)
    assert zb.strerror(12345) == "unknown status"


def _both(**kw):
    base = dict(P=4, E=16, K=2, S=64, H=128, R=1, C=0.1, gpus_per_node=1, cap_rows=None)
    base.update(kw)
    return zb.Config(**base), oracle.Config(**base)


@pytest.mark.parametrize("kw", [
    {}, dict(P=0), dict(P=33), dict(E=15), dict(E=400), dict(E=2, P=4), dict(K=0), dict(K=17),
    dict(S=-1), dict(S=0), dict(H=0), dict(H=4), dict(H=12), dict(R=-1), dict(R=4), dict(R=3),
    dict(C=-0.5), dict(C=1.0), dict(C=0.99), dict(gpus_per_node=0), dict(gpus_per_node=3),
    dict(gpus_per_node=2), dict(cap_rows=127), dict(cap_rows=128), dict(P=32, E=384, R=31),
    dict(P=1, E=384, R=0), dict(K=16), dict(S=2 ** 27, K=16), dict(S=2 ** 26, K=8, P=8, E=16),
    dict(policy=1), dict(policy=2), dict(policy=-1),
])
def test_validation_agrees_with_oracle(lib, kw):
    c, o = _both(**kw)
    assert zb.validate(c) == oracle.validate(o), kw


def test_workspace_bytes(lib):
    c, _ = _both()
    n = zb.workspace_bytes(c)
    assert n > 0 and n % 256 == 0
    # grows with the number of chunks
    c2, _ = _both(S=64 * 1024)
    assert zb.workspace_bytes(c2) > n
    bad, _ = _both(P=0)
    assert zb.workspace_bytes(bad) == 0


def test_entry_points_reject_bad_arguments_without_a_device(lib):
    cfg = zb.Config(P=4, E=16, K=2, S=64, H=128, R=1).c()
    plan = zb._Plan()  # all NULL
    # NULL plan buffers / workspace -> invalid, nothing enqueued
    assert lib.zb_plan(ctypes.byref(cfg), None, ctypes.byref(plan), None, 0, None) == \
        zb.ERR_INVALID
    assert lib.zb_dispatch(ctypes.byref(cfg), ctypes.byref(plan), None, None, None) == \
        zb.ERR_INVALID
    assert lib.zb_combine(ctypes.byref(cfg), ctypes.byref(plan), None, None, None, None) == \
        zb.ERR_INVALID
    assert lib.zb_plan_status(ctypes.byref(cfg), ctypes.byref(plan), None, None) == \
        zb.ERR_INVALID
    bad = zb.Config(P=4, E=15, K=2, S=64, H=128, R=1).c()
    assert lib.zb_plan(ctypes.byref(bad), None, ctypes.byref(plan), None, 0, None) == \
        zb.ERR_INVALID
    # misaligned rows are refused before any launch
    fake = zb._Plan(*([16] * 10))
    assert lib.zb_dispatch(ctypes.byref(cfg), ctypes.byref(fake), 8, 16, None) == \
        zb.ERR_INVALID
    assert lib.zb_combine(ctypes.byref(cfg), ctypes.byref(fake), 16, 16, 8, None) == \
        zb.ERR_INVALID
    # a short or misaligned workspace is refused
    ws = zb.workspace_bytes(zb.Config(P=4, E=16, K=2, S=64, H=128, R=1))
    assert lib.zb_plan(ctypes.byref(cfg), 16, ctypes.byref(fake), 256, ws - 1, None) == \
        zb.ERR_INVALID
    assert lib.zb_plan(ctypes.byref(cfg), 16, ctypes.byref(fake), 128, ws, None) == \
        zb.ERR_INVALID
    # a trace array that 64-bit atomics cannot use (not 8-byte aligned)
    traced = zb._Plan(*([16] * 10), 12)
    assert lib.zb_plan(ctypes.byref(cfg), 16, ctypes.byref(traced), 256, ws, None) == \
        zb.ERR_INVALID


def test_rank_entry_points_reject_bad_arguments_without_a_device(lib):
    """The per-rank form (one rank of P GPUs): workspace sizing and argument
    checks, all refused before anything is enqueued."""
    zc = zb.Config(P=4, E=16, K=2, S=64, H=128, R=1)
    cfg = zc.c()
    n = lib.zb_rank_workspace_bytes(ctypes.byref(cfg))
    assert 0 < n < zb.workspace_bytes(zc) and n % 256 == 0  # one source's histograms
    bad = zb.Config(P=4, E=15, K=2, S=64, H=128, R=1).c()
    assert lib.zb_rank_workspace_bytes(ctypes.byref(bad)) == 0
    fake = zb._Plan(*([16] * 10))
    fake.row_src = None
    # zb_count: NULL counts, short or misaligned workspace
    assert lib.zb_count(ctypes.byref(cfg), 16, None, 256, n, None) == zb.ERR_INVALID
    assert lib.zb_count(ctypes.byref(cfg), 16, 16, 256, n - 1, None) == zb.ERR_INVALID
    assert lib.zb_count(ctypes.byref(cfg), 16, 16, 128, n, None) == zb.ERR_INVALID
    # zb_plan_rank: rank out of range, row_src given, NULL counts
    for rank in (-1, 4):
        assert lib.zb_plan_rank(ctypes.byref(cfg), rank, 16, 16, None, ctypes.byref(fake), 256,
                                n, None) == zb.ERR_INVALID
    with_row_src = zb._Plan(*([16] * 10))
    assert lib.zb_plan_rank(ctypes.byref(cfg), 0, 16, 16, None, ctypes.byref(with_row_src), 256,
                            n, None) == zb.ERR_INVALID
    assert lib.zb_plan_rank(ctypes.byref(cfg), 0, None, 16, None, ctypes.byref(fake), 256, n,
                            None) == zb.ERR_INVALID
    # dispatch / combine through a pointer table: a NULL or misaligned entry
    tbl = (ctypes.c_void_p * 4)(16, 32, 48, 64)
    holes = (ctypes.c_void_p * 4)(16, None, 48, 64)
    skew = (ctypes.c_void_p * 4)(16, 40, 48, 64)
    assert lib.zb_dispatch_rank(ctypes.byref(cfg), ctypes.byref(fake), 16, holes, None) == \
        zb.ERR_INVALID
    assert lib.zb_dispatch_rank(ctypes.byref(cfg), ctypes.byref(fake), 16, skew, None) == \
        zb.ERR_INVALID
    assert lib.zb_dispatch_rank(ctypes.byref(cfg), ctypes.byref(fake), 8, tbl, None) == \
        zb.ERR_INVALID
    assert lib.zb_dispatch_rank(ctypes.byref(cfg), ctypes.byref(fake), 16, None, None) == \
        zb.ERR_INVALID
    assert lib.zb_combine_rank(ctypes.byref(cfg), ctypes.byref(fake), holes, 16, 16, None) == \
        zb.ERR_INVALID
    assert lib.zb_combine_rank(ctypes.byref(cfg), ctypes.byref(fake), tbl, 16, 8, None) == \
        zb.ERR_INVALID


def test_plan_trace_conversion_on_the_host():
    """zb.plan_trace turns the twelve stamps into microseconds from the first
    kernel's start; a kernel that did not run (start left at all ones) is
    None; a plan made without a trace is refused."""
    import types

    import torch
    never = np.uint64(0xFFFFFFFFFFFFFFFF)
    t = np.array([never, never, 0,              # k_zero: did not run
                  1_000, 2_500, 3_000,          # k_hist
                  1_800, 3_600, 14_000,         # k_planner
                  4_000, 14_700, 17_500],       # k_assign
                 dtype=np.uint64)
    plan = types.SimpleNamespace(trace=torch.from_numpy(t.view(np.int64)))
    tl = zb.plan_trace(plan)
    assert tl["k_zero"] is None
    assert tl["k_hist"] == {"start": 0.0, "released": 1.5, "end": 2.0}
    assert tl["k_planner"] == {"start": 0.8, "released": 2.6, "end": 13.0}
    assert tl["k_assign"] == {"start": 3.0, "released": 13.7, "end": 16.5}
    with pytest.raises(zb.ZbError):
        zb.plan_trace(types.SimpleNamespace(trace=None))
