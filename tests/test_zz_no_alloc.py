"""zb_plan_noalloc: the plan entry point for callers that cannot allocate.

Some callers of this library cannot give it a scratch buffer: a plugin run
inside a host framework that owns all device memory, or a serving loop that
keeps cudaMalloc/cudaFree off its hot path because they can synchronise the
device.  zb_plan_noalloc serves them from a fixed array inside the library.
This test calls it through the C ABI and checks, on two calls in a row, that
it produces exactly what zb_plan produces with a caller-provided workspace.
The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from token_dispatch_top_b200 import build, synth, zb

pytestmark = pytest.mark.gpu

NOALLOC_SCRATCH_BYTES = 4 << 20
TABLES = ("cnt", "rep_expert", "rep_quota", "home_quota", "load_before", "load_after",
          "cu_seqlens", "dst_row", "row_src", "stats")


@pytest.fixture(scope="module")
def lib(cuda_device):
    build.build()
    lib = zb.load()
    lib.zb_plan_noalloc.argtypes = [ctypes.POINTER(zb._Cfg), ctypes.c_void_p,
                                    ctypes.POINTER(zb._Plan), ctypes.c_void_p]
    lib.zb_plan_noalloc.restype = ctypes.c_int
    return lib


def _noalloc(lib, plan: zb.Plan, ids: torch.Tensor) -> int:
    return lib.zb_plan_noalloc(ctypes.byref(plan._c), ids.data_ptr(), ctypes.byref(plan._p),
                               torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_zb_plan_on_two_calls(lib, cuda_device):
    wl = synth.WORKLOADS["mid"]
    cfg = zb.Config(P=wl.P, E=wl.E, K=wl.K, S=wl.S, H=wl.H, R=wl.R, C=wl.C)
    assert zb.workspace_bytes(cfg) <= NOALLOC_SCRATCH_BYTES
    mine = zb.Plan(cfg, cuda_device)
    for seed in (0, 1):  # two calls in a row into the same shared scratch
        ids_np, _ = synth.routing(wl, seed)
        ids = torch.from_numpy(ids_np).to(cuda_device)
        ref = zb.Plan(cfg, cuda_device)
        zb.plan(ref, ids)
        assert zb.plan_status(ref)[0] == zb.OK
        for t in TABLES:  # stale values must not survive
            getattr(mine, t).fill_(-7)
        assert _noalloc(lib, mine, ids) == zb.OK
        assert zb.plan_status(mine) == zb.plan_status(ref)
        for t in TABLES:
            assert torch.equal(getattr(mine, t), getattr(ref, t)), (seed, t)


def _compare_with_zb_plan(lib, cfg, ids, dev):
    ref = zb.Plan(cfg, dev)
    zb.plan(ref, ids)
    mine = zb.Plan(cfg, dev)
    for t in TABLES:
        getattr(mine, t).fill_(-7)
    assert _noalloc(lib, mine, ids) == zb.OK
    assert zb.plan_status(mine) == zb.plan_status(ref)
    for t in TABLES:
        assert torch.equal(getattr(mine, t), getattr(ref, t)), t


def test_noalloc_band_and_repair(lib, cuda_device):
    """The options that use the most planner state: eq. (1)'s band and quota
    repair, the band's larger receive buffers included."""
    wl = synth.WORKLOADS["mid"]
    cfg = zb.Config(P=wl.P, E=wl.E, K=wl.K, S=wl.S, H=wl.H, R=wl.R, C=wl.C, relax=1, repair=1,
                    policy=zb.POLICY_LOCAL)
    ids_np, _ = synth.routing(wl, 2)
    _compare_with_zb_plan(lib, cfg, torch.from_numpy(ids_np).to(cuda_device), cuda_device)


def test_noalloc_at_the_size_limit(lib, cuda_device):
    """A config whose workspace is exactly the scratch array's size: the whole
    array, its last bytes included, is usable, and the plan matches zb_plan."""
    cfg = zb.Config(P=16, E=176, K=8, S=93952, H=8, R=1, cap_rows=2 * 93952 * 8)
    assert zb.workspace_bytes(cfg) == NOALLOC_SCRATCH_BYTES
    g = torch.Generator(device=cuda_device)
    g.manual_seed(5)
    ids = torch.randint(0, cfg.E, (cfg.P, cfg.S, cfg.K), generator=g, device=cuda_device,
                        dtype=torch.int32)
    _compare_with_zb_plan(lib, cfg, ids, cuda_device)
    # one more entry per rank needs more scratch than the array holds
    over = zb.Config(P=16, E=176, K=8, S=93952 + 256, H=8, R=1)
    assert zb.workspace_bytes(over) > NOALLOC_SCRATCH_BYTES
    plan = zb._Plan(*([256] * 10))
    assert lib.zb_plan_noalloc(ctypes.byref(over.c()), 256, ctypes.byref(plan), None) == \
        zb.ERR_INVALID


def test_noalloc_rejects_configs_beyond_its_scratch(lib, cuda_device):
    big = zb.Config(P=32, E=384, K=16, S=32768, H=8, R=2)
    assert zb.validate(big) == zb.OK
    assert zb.workspace_bytes(big) > NOALLOC_SCRATCH_BYTES
    plan = zb._Plan(*([256] * 10))  # never touched: the call must refuse first
    assert lib.zb_plan_noalloc(ctypes.byref(big.c()), 256, ctypes.byref(plan), None) == \
        zb.ERR_INVALID
