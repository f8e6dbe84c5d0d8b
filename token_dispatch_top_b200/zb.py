"""Python binding of libzb (ctypes): argument marshalling only.

Every step of plan, dispatch and combine runs in the CUDA kernels of
``libzb.so``; this module passes ``torch.Tensor`` device pointers, sizes and
the current CUDA stream to the C ABI declared in ``include/zb.h``.  There is
no CPU fallback: if the library is missing or fails to load, every call
raises.  With ``ZB_DEBUG=1`` in the environment the bounds-checked build,
``libzb_debug.so``, is loaded instead (see ``debug_read``).
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
DEBUG = os.environ.get("ZB_DEBUG", "") == "1"
LIB_PATH = os.path.join(_HERE, "libzb_debug.so" if DEBUG else "libzb.so")

OK = 0
WARN_UNBALANCED = 1
ERR_INVALID = -1
ERR_CAPACITY = -2
ERR_BAD_ID = -3
ERR_TIMEOUT = -4
ERR_CUDA = -5

POLICY_ROOM = 0   # receiver with the most room (after node coverage)
POLICY_LOCAL = 1  # the largest move, then the most rows served locally

STAT_STATUS, STAT_MAX_LOAD, STAT_N_REPLICAS, STAT_N_ITERS, STAT_WATER_LEVEL, \
    STAT_LOCALITY_COST, STAT_BAD_IDS, STAT_REPAIRED = range(8)
STATS_LEN = 8
TRACE_LEN = 12
TRACE_KERNELS = ("k_zero", "k_hist", "k_planner", "k_assign")  # ZB_TRACE_* / 3

EXPORTS = ("zb_strerror", "zb_validate", "zb_workspace_bytes", "zb_plan", "zb_plan_placed",
           "zb_plan_status", "zb_dispatch", "zb_combine", "zb_merge_workspace_bytes",
           "zb_merge", "zb_dispatch_merged", "zb_combine_reduce", "zb_combine_merged",
           "zb_recalibrate_workspace_bytes", "zb_recalibrate", "zb_place_by_demand",
           "zb_rank_workspace_bytes", "zb_count", "zb_plan_rank", "zb_dispatch_rank",
           "zb_combine_rank", "zb_debug_read")


class ZbError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {strerror(status)} (status {status})")
        self.status = status


class _Cfg(ctypes.Structure):
    _fields_ = [("P", ctypes.c_int), ("E", ctypes.c_int), ("K", ctypes.c_int),
                ("S", ctypes.c_int), ("H", ctypes.c_int), ("R", ctypes.c_int),
                ("C", ctypes.c_float), ("gpus_per_node", ctypes.c_int),
                ("cap_rows", ctypes.c_int), ("policy", ctypes.c_int),
                ("relax", ctypes.c_int), ("repair", ctypes.c_int)]


class _Plan(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("cnt", "rep_expert", "rep_quota", "home_quota", "load_before", "load_after",
                 "cu_seqlens", "dst_row", "row_src", "stats", "trace")]


class _Merge(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("tok_row", "grp_tok", "tok_cnt")]


_lib = None


def load() -> ctypes.CDLL:
    """Load libzb.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{os.path.basename(LIB_PATH)} not built at {LIB_PATH}; run "
                              "`python -m token_dispatch_top_b200.build"
                              f"{' --debug' if LIB_PATH.endswith('_debug.so') else ''}`")
        lib = ctypes.CDLL(LIB_PATH)
        vp, cfgp, planp = ctypes.c_void_p, ctypes.POINTER(_Cfg), ctypes.POINTER(_Plan)
        lib.zb_strerror.argtypes = [ctypes.c_int]
        lib.zb_strerror.restype = ctypes.c_char_p
        lib.zb_validate.argtypes = [cfgp]
        lib.zb_workspace_bytes.argtypes = [cfgp]
        lib.zb_workspace_bytes.restype = ctypes.c_size_t
        lib.zb_plan.argtypes = [cfgp, vp, planp, vp, ctypes.c_size_t, vp]
        lib.zb_plan_placed.argtypes = [cfgp, vp, vp, planp, vp, ctypes.c_size_t, vp]
        lib.zb_plan_status.argtypes = [cfgp, planp, vp, ctypes.POINTER(ctypes.c_int32)]
        lib.zb_dispatch.argtypes = [cfgp, planp, vp, vp, vp]
        lib.zb_combine.argtypes = [cfgp, planp, vp, vp, vp, vp]
        mergep = ctypes.POINTER(_Merge)
        lib.zb_merge_workspace_bytes.argtypes = [cfgp]
        lib.zb_merge_workspace_bytes.restype = ctypes.c_size_t
        lib.zb_merge.argtypes = [cfgp, planp, mergep, vp, ctypes.c_size_t, vp]
        lib.zb_dispatch_merged.argtypes = [cfgp, planp, mergep, vp, vp, vp]
        lib.zb_combine_reduce.argtypes = [cfgp, planp, mergep, vp, vp, vp, vp]
        lib.zb_combine_merged.argtypes = [cfgp, planp, mergep, vp, vp, vp]
        lib.zb_recalibrate_workspace_bytes.argtypes = [cfgp, ctypes.c_int]
        lib.zb_recalibrate_workspace_bytes.restype = ctypes.c_size_t
        i32p = ctypes.POINTER(ctypes.c_int32)
        lib.zb_recalibrate.argtypes = [cfgp, vp, vp, ctypes.c_int, ctypes.c_float, ctypes.c_int,
                                       vp, ctypes.c_size_t, vp, i32p, i32p]
        lib.zb_place_by_demand.argtypes = [cfgp, vp, vp]
        lib.zb_rank_workspace_bytes.argtypes = [cfgp]
        lib.zb_rank_workspace_bytes.restype = ctypes.c_size_t
        lib.zb_count.argtypes = [cfgp, vp, vp, vp, ctypes.c_size_t, vp]
        lib.zb_plan_rank.argtypes = [cfgp, ctypes.c_int, vp, vp, vp, planp, vp, ctypes.c_size_t,
                                     vp]
        lib.zb_dispatch_rank.argtypes = [cfgp, planp, vp, ctypes.POINTER(ctypes.c_void_p), vp]
        lib.zb_combine_rank.argtypes = [cfgp, planp, ctypes.POINTER(ctypes.c_void_p), vp, vp, vp]
        lib.zb_debug_read.argtypes = [ctypes.POINTER(_DebugRecord), ctypes.c_int]
        _lib = lib
    return _lib


def strerror(status: int) -> str:
    return load().zb_strerror(int(status)).decode()


def plan_trace(p) -> dict:
    """The device timeline of the last plan call on ``p`` (a Plan or RankPlan
    made with ``trace=True``; synchronises): per kernel, microseconds from the
    first stamp of the call to the first of its CTAs to start, the first
    released by its dependency wait, and the last to finish (None for a
    kernel the call did not run)."""
    if p.trace is None:
        raise ZbError(ERR_INVALID, "plan_trace: the plan was made without trace=True")
    t = p.trace.cpu().numpy().view(np.uint64)
    never = np.uint64(0xFFFFFFFFFFFFFFFF)
    t0 = min(int(t[3 * k]) for k in range(len(TRACE_KERNELS)) if t[3 * k] != never)
    out = {}
    for k, name in enumerate(TRACE_KERNELS):
        st, rel, en = (int(x) for x in t[3 * k:3 * k + 3])
        out[name] = None if t[3 * k] == never else {
            "start": (st - t0) / 1000.0, "released": (rel - t0) / 1000.0,
            "end": (en - t0) / 1000.0}
    return out


class _DebugRecord(ctypes.Structure):
    _fields_ = [("count", ctypes.c_uint64), ("site", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("index", ctypes.c_int64),
                ("bound", ctypes.c_int64)]


# ZB_SITE_* of include/zb.h
SITES = {1: "assign: expert id", 2: "assign: segment index", 3: "assign: row",
         4: "planner: segment write", 5: "planner: slot or holder", 6: "dispatch: row",
         7: "combine: row", 8: "merge: row"}


def debug_read(reset: bool = True) -> dict:
    """The bounds-checked build's record (synchronises the device): failed
    checks since the last reset, and the site, index and bound of the first.
    Raises in the release build, which keeps no record."""
    rec = _DebugRecord()
    st = load().zb_debug_read(ctypes.byref(rec), int(bool(reset)))
    if st != OK:
        raise ZbError(st, "zb_debug_read (the release library keeps no record)")
    return {"count": int(rec.count), "site": SITES.get(int(rec.site), int(rec.site)),
            "index": int(rec.index), "bound": int(rec.bound)}


@dataclass(frozen=True)
class Config:
    """Problem shape; see ``zb_config`` in include/zb.h for the bounds."""
    P: int
    E: int
    K: int
    S: int
    H: int
    R: int
    C: float = 0.0
    gpus_per_node: int = 1
    cap_rows: int | None = None  # default S*K, or floor((1+C) S*K) with relax
    policy: int = 0              # POLICY_ROOM or POLICY_LOCAL
    relax: int = 0               # 1: receipts within q +- floor(C q), eq. (1)
    repair: int = 0              # 1: quota repair between rank pairs

    @property
    def cap(self) -> int:
        if self.cap_rows is not None:
            return self.cap_rows
        sk = self.S * self.K
        if not self.relax:
            return sk
        c20 = int(math.floor(float(ctypes.c_float(self.C).value) * 1048576.0))
        return sk + ((sk * c20) >> 20)

    @property
    def Eh(self) -> int:
        return self.E // self.P

    def c(self) -> _Cfg:
        return _Cfg(self.P, self.E, self.K, self.S, self.H, self.R, float(self.C),
                    self.gpus_per_node, self.cap, self.policy, self.relax, self.repair)


def validate(cfg: Config) -> int:
    return int(load().zb_validate(ctypes.byref(cfg.c())))


def workspace_bytes(cfg: Config) -> int:
    return int(load().zb_workspace_bytes(ctypes.byref(cfg.c())))


class Plan:
    """Device buffers of one plan plus its scratch workspace (torch-owned)."""

    def __init__(self, cfg: Config, device, with_row_src: bool = True, trace: bool = False):
        if validate(cfg) != OK:
            raise ZbError(ERR_INVALID, f"config {cfg}")
        i32 = dict(dtype=torch.int32, device=device)
        P, E, R = cfg.P, cfg.E, cfg.R
        self.cfg = cfg
        self.cnt = torch.empty((P, E), **i32)
        self.rep_expert = torch.empty((P, R), **i32)
        self.rep_quota = torch.empty((P, R), **i32)
        self.home_quota = torch.empty((E,), **i32)
        self.load_before = torch.empty((P,), **i32)
        self.load_after = torch.empty((P,), **i32)
        self.cu_seqlens = torch.empty((P, cfg.Eh + R + 1), **i32)
        self.dst_row = torch.empty((P, cfg.S, cfg.K), **i32)
        self.row_src = torch.empty((P, cfg.cap), **i32) if with_row_src else None
        self.stats = torch.zeros((STATS_LEN,), dtype=torch.int64, device=device)
        self.trace = torch.zeros((TRACE_LEN,), dtype=torch.int64, device=device) \
            if trace else None
        self.ws_bytes = workspace_bytes(cfg)
        self.workspace = torch.empty((self.ws_bytes + 256,), dtype=torch.uint8, device=device)
        self.ws_ptr = (self.workspace.data_ptr() + 255) & ~255  # 256-byte aligned
        self._c = cfg.c()

        def p(t):
            return None if t is None or t.numel() == 0 else t.data_ptr()
        self._p = _Plan(p(self.cnt), p(self.rep_expert), p(self.rep_quota), p(self.home_quota),
                        p(self.load_before), p(self.load_after), p(self.cu_seqlens),
                        p(self.dst_row), p(self.row_src), p(self.stats), p(self.trace))


def _stream(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check(t: torch.Tensor, shape, dtype, name):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous() \
            or not t.is_cuda:
        raise ZbError(ERR_INVALID, f"{name}: want contiguous cuda {dtype} {tuple(shape)}, got "
                                   f"{t.dtype} {tuple(t.shape)} on {t.device}")


def plan(p: Plan, topk_ids: torch.Tensor, stream=None) -> None:
    """Steps 1-3 (asynchronous).  ``topk_ids``: int32 [P,S,K] on the device."""
    cfg = p.cfg
    _check(topk_ids, (cfg.P, cfg.S, cfg.K), torch.int32, "topk_ids")
    st = load().zb_plan(ctypes.byref(p._c), topk_ids.data_ptr(), ctypes.byref(p._p),
                        p.ws_ptr, p.ws_bytes, _stream(stream))
    if st != OK:
        raise ZbError(st, "zb_plan")


def plan_placed(p: Plan, topk_ids: torch.Tensor, placement: torch.Tensor, stream=None) -> None:
    """Steps 1-3 keeping a given replica placement (asynchronous).
    ``placement``: int32 [P,R] on the device, -1 = empty slot; it may be the
    ``rep_expert`` of this or another plan of the same shape."""
    cfg = p.cfg
    _check(topk_ids, (cfg.P, cfg.S, cfg.K), torch.int32, "topk_ids")
    _check(placement, (cfg.P, cfg.R), torch.int32, "placement")
    st = load().zb_plan_placed(ctypes.byref(p._c), topk_ids.data_ptr(),
                               placement.data_ptr() if placement.numel() else None,
                               ctypes.byref(p._p), p.ws_ptr, p.ws_bytes, _stream(stream))
    if st != OK:
        raise ZbError(st, "zb_plan_placed")


def plan_status(p: Plan, stream=None) -> tuple[int, int]:
    """Synchronise the stream and return (status, max_load) of the plan."""
    ml = ctypes.c_int32(0)
    st = load().zb_plan_status(ctypes.byref(p._c), ctypes.byref(p._p), _stream(stream),
                               ctypes.byref(ml))
    if st in (ERR_INVALID, ERR_CUDA):
        raise ZbError(st, "zb_plan_status")
    return int(st), int(ml.value)


def dispatch(p: Plan, hidden: torch.Tensor, buf: torch.Tensor, stream=None) -> None:
    """Step 4 (asynchronous): ``hidden`` bf16 [P,S,H] -> ``buf`` bf16 [P,cap,H]."""
    cfg = p.cfg
    _check(hidden, (cfg.P, cfg.S, cfg.H), torch.bfloat16, "hidden")
    _check(buf, (cfg.P, cfg.cap, cfg.H), torch.bfloat16, "buf")
    st = load().zb_dispatch(ctypes.byref(p._c), ctypes.byref(p._p), hidden.data_ptr(),
                            buf.data_ptr(), _stream(stream))
    if st != OK:
        raise ZbError(st, "zb_dispatch")


def combine(p: Plan, y: torch.Tensor, topk_weights: torch.Tensor, out: torch.Tensor,
            stream=None) -> None:
    """Step 5 (asynchronous): ``y`` bf16 [P,cap,H], ``topk_weights`` fp32 [P,S,K]
    -> ``out`` bf16 [P,S,H]."""
    cfg = p.cfg
    _check(y, (cfg.P, cfg.cap, cfg.H), torch.bfloat16, "y")
    _check(topk_weights, (cfg.P, cfg.S, cfg.K), torch.float32, "topk_weights")
    _check(out, (cfg.P, cfg.S, cfg.H), torch.bfloat16, "out")
    st = load().zb_combine(ctypes.byref(p._c), ctypes.byref(p._p), y.data_ptr(),
                           topk_weights.data_ptr(), out.data_ptr(), _stream(stream))
    if st != OK:
        raise ZbError(st, "zb_combine")


class Merge:
    """Device buffers of the merged dispatch layout of one plan shape."""

    def __init__(self, cfg: Config, device):
        i32 = dict(dtype=torch.int32, device=device)
        self.cfg = cfg
        self.tok_row = torch.empty((cfg.P, cfg.S, cfg.K), **i32)
        self.grp_tok = torch.empty((cfg.P, cfg.cap), **i32)
        self.tok_cnt = torch.empty((cfg.P,), **i32)
        self.ws_bytes = int(load().zb_merge_workspace_bytes(ctypes.byref(cfg.c())))
        self.workspace = torch.empty((self.ws_bytes + 256,), dtype=torch.uint8, device=device)
        self.ws_ptr = (self.workspace.data_ptr() + 255) & ~255

        def p(t):
            return None if t.numel() == 0 else t.data_ptr()
        self._m = _Merge(p(self.tok_row), p(self.grp_tok), p(self.tok_cnt))


def merge(p: Plan, m: Merge, stream=None) -> None:
    """The merged layout of plan ``p`` (asynchronous, after zb.plan)."""
    st = load().zb_merge(ctypes.byref(p._c), ctypes.byref(p._p), ctypes.byref(m._m), m.ws_ptr,
                         m.ws_bytes, _stream(stream))
    if st != OK:
        raise ZbError(st, "zb_merge")


def dispatch_merged(p: Plan, m: Merge, hidden: torch.Tensor, tbuf: torch.Tensor,
                    stream=None) -> None:
    """One row per (token, destination rank): ``hidden`` bf16 [P,S,H] ->
    ``tbuf`` bf16 [P,cap,H] (rows past m.tok_cnt untouched)."""
    cfg = p.cfg
    _check(hidden, (cfg.P, cfg.S, cfg.H), torch.bfloat16, "hidden")
    _check(tbuf, (cfg.P, cfg.cap, cfg.H), torch.bfloat16, "tbuf")
    st = load().zb_dispatch_merged(ctypes.byref(p._c), ctypes.byref(p._p), ctypes.byref(m._m),
                                   hidden.data_ptr(), tbuf.data_ptr(), _stream(stream))
    if st != OK:
        raise ZbError(st, "zb_dispatch_merged")


def combine_reduce(p: Plan, m: Merge, y: torch.Tensor, topk_weights: torch.Tensor,
                   part: torch.Tensor, stream=None) -> None:
    """Destination side of the merged combine: ``y`` bf16 [P,cap,H] (expert
    outputs in grouped rows), ``topk_weights`` fp32 [P,S,K] -> ``part`` bf16
    [P,cap,H], one partial per merged row (rows past m.tok_cnt untouched)."""
    cfg = p.cfg
    _check(y, (cfg.P, cfg.cap, cfg.H), torch.bfloat16, "y")
    _check(topk_weights, (cfg.P, cfg.S, cfg.K), torch.float32, "topk_weights")
    _check(part, (cfg.P, cfg.cap, cfg.H), torch.bfloat16, "part")
    st = load().zb_combine_reduce(ctypes.byref(p._c), ctypes.byref(p._p), ctypes.byref(m._m),
                                  y.data_ptr(), topk_weights.data_ptr(), part.data_ptr(),
                                  _stream(stream))
    if st != OK:
        raise ZbError(st, "zb_combine_reduce")


def combine_merged(p: Plan, m: Merge, part: torch.Tensor, out: torch.Tensor,
                   stream=None) -> None:
    """Source side of the merged combine: ``part`` bf16 [P,cap,H] -> ``out``
    bf16 [P,S,H], the float sum of each token's partials rounded once."""
    cfg = p.cfg
    _check(part, (cfg.P, cfg.cap, cfg.H), torch.bfloat16, "part")
    _check(out, (cfg.P, cfg.S, cfg.H), torch.bfloat16, "out")
    st = load().zb_combine_merged(ctypes.byref(p._c), ctypes.byref(p._p), ctypes.byref(m._m),
                                  part.data_ptr(), out.data_ptr(), _stream(stream))
    if st != OK:
        raise ZbError(st, "zb_combine_merged")


RECAL_SLOT = 0   # ViBE incremental update: one helper slot takes another expert
RECAL_INTRA = 1  # Zepp eq. (4): two slots of one node exchange their experts


def recalibrate(cfg: Config, cnt: torch.Tensor, placement: torch.Tensor, mode: int = RECAL_SLOT,
                eps: float = 0.03, max_swaps: int = 64, stream=None) -> tuple[int, int]:
    """Placement recalibration between invocations (synchronises the stream).
    ``cnt`` int32 [P,E] (route counts, e.g. a plan's ``cnt``), ``placement``
    int32 [P,R], changed in place.  Returns (steps taken, final max load)."""
    _check(cnt, (cfg.P, cfg.E), torch.int32, "cnt")
    _check(placement, (cfg.P, cfg.R), torch.int32, "placement")
    lib = load()
    nbytes = int(lib.zb_recalibrate_workspace_bytes(ctypes.byref(cfg.c()), int(mode)))
    if nbytes == 0:
        raise ZbError(ERR_INVALID, "zb_recalibrate_workspace_bytes")
    ws = torch.empty((nbytes + 256,), dtype=torch.uint8, device=cnt.device)
    ws_ptr = (ws.data_ptr() + 255) & ~255
    swaps, mx = ctypes.c_int32(0), ctypes.c_int32(0)
    st = lib.zb_recalibrate(ctypes.byref(cfg.c()), cnt.data_ptr(),
                            placement.data_ptr() if placement.numel() else None, int(mode),
                            float(eps), int(max_swaps), ws_ptr, nbytes, _stream(stream),
                            ctypes.byref(swaps), ctypes.byref(mx))
    if st != OK:
        raise ZbError(st, "zb_recalibrate")
    return int(swaps.value), int(mx.value)


def place_by_demand(cfg: Config, demand) -> np.ndarray:
    """Replica placement int32 [P,R] from historical per-expert demand (host
    int64 [E]); runs on the host, for zb.plan_placed."""
    d = np.ascontiguousarray(np.asarray(demand), dtype=np.int64)
    if d.shape != (cfg.E,):
        raise ValueError(f"demand: expected shape ({cfg.E},), got {d.shape}")
    pl = np.full((cfg.P, cfg.R), -1, np.int32)
    st = load().zb_place_by_demand(ctypes.byref(cfg.c()), d.ctypes.data,
                                   pl.ctypes.data if pl.size else None)
    if st != OK:
        raise ZbError(st, "zb_place_by_demand")
    return pl


# --------------------------------------------------- the path on one of P GPUs

class RankPlan:
    """Device buffers of the plan of one rank of P GPUs: the plan tables (as
    :class:`Plan`), ``dst_row`` [S,K] for this rank's entries, this rank's
    count row ``counts`` [E+1], the all-gathered table ``table`` [P,E+1] and
    the scratch workspace that ``count`` fills and ``plan_rank`` reads."""

    def __init__(self, cfg: Config, rank: int, device, trace: bool = False):
        if validate(cfg) != OK or not 0 <= rank < cfg.P:
            raise ZbError(ERR_INVALID, f"config {cfg}, rank {rank}")
        i32 = dict(dtype=torch.int32, device=device)
        P, E, R = cfg.P, cfg.E, cfg.R
        self.cfg, self.rank = cfg, rank
        self.cnt = torch.empty((P, E), **i32)
        self.rep_expert = torch.empty((P, R), **i32)
        self.rep_quota = torch.empty((P, R), **i32)
        self.home_quota = torch.empty((E,), **i32)
        self.load_before = torch.empty((P,), **i32)
        self.load_after = torch.empty((P,), **i32)
        self.cu_seqlens = torch.empty((P, cfg.Eh + R + 1), **i32)
        self.dst_row = torch.empty((cfg.S, cfg.K), **i32)
        self.stats = torch.zeros((STATS_LEN,), dtype=torch.int64, device=device)
        self.trace = torch.zeros((TRACE_LEN,), dtype=torch.int64, device=device) \
            if trace else None
        self.counts = torch.empty((E + 1,), **i32)
        self.table = torch.empty((P, E + 1), **i32)
        self.ws_bytes = int(load().zb_rank_workspace_bytes(ctypes.byref(cfg.c())))
        self.workspace = torch.empty((self.ws_bytes + 256,), dtype=torch.uint8, device=device)
        self.ws_ptr = (self.workspace.data_ptr() + 255) & ~255
        self._c = cfg.c()

        def p(t):
            return None if t is None or t.numel() == 0 else t.data_ptr()
        self._p = _Plan(p(self.cnt), p(self.rep_expert), p(self.rep_quota), p(self.home_quota),
                        p(self.load_before), p(self.load_after), p(self.cu_seqlens),
                        p(self.dst_row), None, p(self.stats), p(self.trace))


def count(rp: RankPlan, topk_ids: torch.Tensor, stream=None) -> None:
    """Step 1 on one rank (asynchronous): ``rp.counts`` = the per-expert counts
    of this rank's ids int32 [S,K], then the number of ids outside [0, E)."""
    cfg = rp.cfg
    _check(topk_ids, (cfg.S, cfg.K), torch.int32, "topk_ids")
    st = load().zb_count(ctypes.byref(rp._c), topk_ids.data_ptr(), rp.counts.data_ptr(),
                         rp.ws_ptr, rp.ws_bytes, _stream(stream))
    if st != OK:
        raise ZbError(st, "zb_count")


def exchange_counts(counts: torch.Tensor, table: torch.Tensor, group=None) -> torch.Tensor:
    """The count exchange: every rank's ``counts`` row [E+1] gathered, in rank
    order, into ``table`` [P,E+1] with torch.distributed (NCCL on GPUs; any
    backend whose all-gather takes these tensors).  Without an initialised
    process group, P must be 1."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        if table.shape[0] != 1:
            raise ZbError(ERR_INVALID, "exchange_counts: no process group and P > 1")
        table[0].copy_(counts)
        return table
    if dist.get_world_size(group) != table.shape[0]:
        raise ZbError(ERR_INVALID, "exchange_counts: world size differs from P")
    dist.all_gather(list(table.unbind(0)), counts, group=group)
    return table


def plan_rank(rp: RankPlan, topk_ids: torch.Tensor, placement: torch.Tensor | None = None,
              stream=None) -> None:
    """Steps 2-3 on one rank (asynchronous), from ``rp.table`` (the exchanged
    counts) and this rank's ids; ``count`` must have run on the same ids."""
    cfg = rp.cfg
    _check(topk_ids, (cfg.S, cfg.K), torch.int32, "topk_ids")
    _check(rp.table, (cfg.P, cfg.E + 1), torch.int32, "table")
    pl = None
    if placement is not None:
        _check(placement, (cfg.P, cfg.R), torch.int32, "placement")
        pl = placement.data_ptr() if placement.numel() else None
    st = load().zb_plan_rank(ctypes.byref(rp._c), rp.rank, rp.table.data_ptr(),
                             topk_ids.data_ptr(), pl, ctypes.byref(rp._p), rp.ws_ptr,
                             rp.ws_bytes, _stream(stream))
    if st != OK:
        raise ZbError(st, "zb_plan_rank")


def _pointer_table(cfg: Config, rows, what: str):
    """A host array of P device pointers from P tensors bf16 [cap,H] or P
    integer addresses (peer memory mapped into this process)."""
    if len(rows) != cfg.P:
        raise ZbError(ERR_INVALID, f"{what}: want {cfg.P} buffers, got {len(rows)}")
    tbl = (ctypes.c_void_p * cfg.P)()
    for j, r in enumerate(rows):
        if isinstance(r, torch.Tensor):
            _check(r, (cfg.cap, cfg.H), torch.bfloat16, f"{what}[{j}]")
            tbl[j] = r.data_ptr()
        else:
            tbl[j] = int(r)
    return tbl


def dispatch_rank(rp: RankPlan, hidden: torch.Tensor, bufs, stream=None) -> None:
    """Step 4 on one rank (asynchronous): ``hidden`` bf16 [S,H] into the P
    receive buffers ``bufs`` (bf16 [cap,H] tensors or device addresses)."""
    cfg = rp.cfg
    _check(hidden, (cfg.S, cfg.H), torch.bfloat16, "hidden")
    tbl = _pointer_table(cfg, bufs, "bufs")
    st = load().zb_dispatch_rank(ctypes.byref(rp._c), ctypes.byref(rp._p), hidden.data_ptr(),
                                 tbl, _stream(stream))
    if st != OK:
        raise ZbError(st, "zb_dispatch_rank")


def combine_rank(rp: RankPlan, ys, topk_weights: torch.Tensor, out: torch.Tensor,
                 stream=None) -> None:
    """Step 5 on one rank (asynchronous): this rank's tokens gathered from the
    P expert-output buffers ``ys`` (bf16 [cap,H] tensors or device addresses)
    with ``topk_weights`` fp32 [S,K] into ``out`` bf16 [S,H]."""
    cfg = rp.cfg
    _check(topk_weights, (cfg.S, cfg.K), torch.float32, "topk_weights")
    _check(out, (cfg.S, cfg.H), torch.bfloat16, "out")
    tbl = _pointer_table(cfg, ys, "ys")
    st = load().zb_combine_rank(ctypes.byref(rp._c), ctypes.byref(rp._p), tbl,
                                topk_weights.data_ptr(), out.data_ptr(), _stream(stream))
    if st != OK:
        raise ZbError(st, "zb_combine_rank")
