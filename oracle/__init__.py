"""CPU oracle for load-balanced MoE token dispatch/combine -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this package.  The product path (the CUDA library and
its Python binding) never imports, calls or falls back to it.

The arithmetic lives in ``zb_oracle.c`` (plain C, single-threaded, compiled
with ``-ffp-contract=off`` and without fast-math); this module only compiles it
with gcc, marshals numpy arrays and returns the results.  Every function of
the C file cites the web-page passage it follows (Zepp 4.1 eq. (1); ISER-MoE
HALO-Q Scheduler; MoonEP "What MoonEP enforces and how").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "zb_oracle.c")
_LIB = os.path.join(_HERE, "libzb_oracle.so")

OK = 0
UNBALANCED = 1
ERR_INVALID = -1
ERR_CAPACITY = -2
ERR_BAD_ID = -3


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no CUDA involved) and return the .so path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-Wall", "-ffp-contract=off", "-fno-fast-math",
             "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [("P", ctypes.c_int), ("E", ctypes.c_int), ("K", ctypes.c_int),
                ("S", ctypes.c_int), ("H", ctypes.c_int), ("R", ctypes.c_int),
                ("C", ctypes.c_double), ("gpus_per_node", ctypes.c_int),
                ("cap_rows", ctypes.c_int), ("policy", ctypes.c_int),
                ("relax", ctypes.c_int), ("repair", ctypes.c_int)]


_P32 = ctypes.POINTER(ctypes.c_int32)


class _Out(ctypes.Structure):
    _fields_ = [("cnt", _P32), ("rep_expert", _P32), ("rep_quota", _P32),
                ("home_quota", _P32), ("load_before", _P32), ("load_after", _P32),
                ("cu_seqlens", _P32), ("dst_row", _P32), ("row_src", _P32), ("M", _P32),
                ("locality_cost", ctypes.c_int64), ("max_load", ctypes.c_int32),
                ("n_replicas", ctypes.c_int32), ("n_iters", ctypes.c_int32),
                ("water_level", ctypes.c_int32), ("repaired", ctypes.c_int32)]


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.zbo_validate.argtypes = [ctypes.POINTER(_Cfg)]
        lib.zbo_plan.argtypes = [ctypes.POINTER(_Cfg), _P32, ctypes.POINTER(_Out)]
        lib.zbo_plan_placed.argtypes = [ctypes.POINTER(_Cfg), _P32, _P32, ctypes.POINTER(_Out)]
        lib.zbo_placement_valid.argtypes = [ctypes.POINTER(_Cfg), _P32]
        vp = ctypes.c_void_p
        lib.zbo_dispatch.argtypes = [ctypes.POINTER(_Cfg), vp, vp, vp]
        lib.zbo_dispatch.restype = None
        lib.zbo_combine.argtypes = [ctypes.POINTER(_Cfg), vp, vp, vp, vp]
        lib.zbo_combine.restype = None
        lib.zbo_count.argtypes = [ctypes.POINTER(_Cfg), vp, vp]
        lib.zbo_count.restype = None
        lib.zbo_plan_rank.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int, _P32, _P32, _P32,
                                      ctypes.POINTER(_Out)]
        lib.zbo_dispatch_ranks.argtypes = [ctypes.POINTER(_Cfg), vp, vp, vp]
        lib.zbo_dispatch_ranks.restype = None
        lib.zbo_combine_ranks.argtypes = [ctypes.POINTER(_Cfg), vp, vp, vp, vp]
        lib.zbo_combine_ranks.restype = None
        lib.zbo_f32_to_bf16.argtypes = [ctypes.c_float]
        lib.zbo_f32_to_bf16.restype = ctypes.c_uint16
        lib.zbo_bf16_to_f32.argtypes = [ctypes.c_uint16]
        lib.zbo_bf16_to_f32.restype = ctypes.c_float
        lib.zbo_merge.argtypes = [ctypes.POINTER(_Cfg), vp, vp, vp, vp]
        lib.zbo_merge.restype = None
        lib.zbo_dispatch_merged.argtypes = [ctypes.POINTER(_Cfg), vp, vp, vp]
        lib.zbo_dispatch_merged.restype = None
        lib.zbo_place_by_demand.argtypes = [ctypes.POINTER(_Cfg), vp, _P32, _P32]
        lib.zbo_place_by_demand.restype = ctypes.c_int
        lib.zbo_recalibrate.argtypes = [ctypes.POINTER(_Cfg), _P32, _P32, ctypes.c_int,
                                        ctypes.c_double, ctypes.c_int, _P32]
        lib.zbo_recalibrate.restype = ctypes.c_int
        lib.zbo_combine_reduce.argtypes = [ctypes.POINTER(_Cfg), vp, vp, vp, vp, vp]
        lib.zbo_combine_reduce.restype = None
        lib.zbo_combine_merged.argtypes = [ctypes.POINTER(_Cfg), vp, vp, vp]
        lib.zbo_combine_merged.restype = None
        d = ctypes.POINTER(ctypes.c_double)
        lib.zbo_metrics.argtypes = [ctypes.POINTER(_Cfg), _P32, _P32, _P32, d, d, d, d]
        lib.zbo_metrics.restype = None
        _lib = lib
    return _lib


@dataclass
class Config:
    """Problem shape.  ``cap_rows`` defaults to S*K (the water level), or with
    ``relax`` to floor((1+C) S*K), C taken to 20 fractional bits (eq. (1))."""
    P: int
    E: int
    K: int
    S: int
    H: int
    R: int
    C: float = 0.0
    gpus_per_node: int = 1
    cap_rows: int | None = None
    policy: int = 0  # receiver choice: 0 most room, 1 most local rows
    relax: int = 0   # 1: hosts receive within q +- floor(C q) (eq. (1))
    repair: int = 0  # 1: quota repair between rank pairs (HALO-Q stage 4)

    def cap(self) -> int:
        if self.cap_rows is not None:
            return self.cap_rows
        sk = self.S * self.K
        if not self.relax:
            return sk
        cfix = int(np.floor(float(np.float32(self.C)) * 1048576.0))
        return sk + ((sk * cfix) >> 20)

    def c(self) -> _Cfg:
        return _Cfg(self.P, self.E, self.K, self.S, self.H, self.R, float(self.C),
                    self.gpus_per_node, self.cap(), self.policy, self.relax, self.repair)


def _ptr(a: np.ndarray):
    assert a.flags.c_contiguous
    return a.ctypes.data_as(_P32)


def validate(cfg: Config) -> int:
    return int(_load().zbo_validate(ctypes.byref(cfg.c())))


def plan(cfg: Config, ids: np.ndarray, want_M: bool = True,
         placement: np.ndarray | None = None) -> dict:
    """Steps 1-3 on host arrays.  ``ids`` is int32 ``[P,S,K]``.  With
    ``placement`` (int32 ``[P,R]``, -1 = empty slot) the replica placement is
    kept and only the quotas are planned.

    Returns a dict with ``status`` and the plan tables (numpy int32 arrays
    shaped as the C comments state), ``M`` ``[E,P,P]`` when requested, and the
    scalars ``locality_cost``, ``max_load``, ``n_replicas``, ``n_iters``, ``T``.
    """
    lib = _load()
    P, E, K, S, R = cfg.P, cfg.E, cfg.K, cfg.S, cfg.R
    Eh = E // max(P, 1)
    cap = cfg.cap()
    ids = np.ascontiguousarray(ids, dtype=np.int32).reshape(P, S, K)
    r = dict(
        cnt=np.zeros((P, E), np.int32), rep_expert=np.zeros((P, R), np.int32),
        rep_quota=np.zeros((P, R), np.int32), home_quota=np.zeros(E, np.int32),
        load_before=np.zeros(P, np.int32), load_after=np.zeros(P, np.int32),
        cu_seqlens=np.zeros((P, Eh + R + 1), np.int32), dst_row=np.zeros((P, S, K), np.int32),
        row_src=np.zeros((P, cap), np.int32))
    if want_M:
        r["M"] = np.zeros((E, P, P), np.int32)
    out = _Out(*[_ptr(r[k]) for k in ("cnt", "rep_expert", "rep_quota", "home_quota",
                                       "load_before", "load_after", "cu_seqlens",
                                       "dst_row", "row_src")],
               _ptr(r["M"]) if want_M else _P32(), 0, 0, 0, 0, 0, 0)
    if placement is None:
        st = lib.zbo_plan(ctypes.byref(cfg.c()), _ptr(ids), ctypes.byref(out))
    else:
        pl = np.ascontiguousarray(placement, dtype=np.int32).reshape(P, R)
        st = lib.zbo_plan_placed(ctypes.byref(cfg.c()), _ptr(ids), _ptr(pl), ctypes.byref(out))
    r.update(status=int(st), locality_cost=int(out.locality_cost), max_load=int(out.max_load),
             n_replicas=int(out.n_replicas), n_iters=int(out.n_iters), T=int(out.water_level),
             repaired=int(out.repaired))
    return r


def dispatch(cfg: Config, dst_row: np.ndarray, hidden_bits: np.ndarray,
             buf_bits: np.ndarray | None = None) -> np.ndarray:
    """Step 4.  ``hidden_bits`` is uint16 (bf16 bit patterns) ``[P,S,H]``.

    Writes into ``buf_bits`` (uint16 ``[P,cap,H]``) if given, else into a
    zero-filled new buffer, and returns it.
    """
    P, S, H = cfg.P, cfg.S, cfg.H
    hidden_bits = np.ascontiguousarray(hidden_bits, dtype=np.uint16).reshape(P, S, H)
    dst_row = np.ascontiguousarray(dst_row, dtype=np.int32)
    if buf_bits is None:
        buf_bits = np.zeros((P, cfg.cap(), H), np.uint16)
    assert buf_bits.dtype == np.uint16 and buf_bits.flags.c_contiguous
    _load().zbo_dispatch(ctypes.byref(cfg.c()), dst_row.ctypes.data, hidden_bits.ctypes.data,
                         buf_bits.ctypes.data)
    return buf_bits


def combine(cfg: Config, dst_row: np.ndarray, y_bits: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Step 5.  ``y_bits`` uint16 ``[rows,H]`` indexed by ``dst_row``; ``w``
    float32 ``[P,S,K]``.  Returns uint16 ``[P,S,H]``."""
    P, S, H = cfg.P, cfg.S, cfg.H
    dst_row = np.ascontiguousarray(dst_row, dtype=np.int32)
    y_bits = np.ascontiguousarray(y_bits, dtype=np.uint16)
    w = np.ascontiguousarray(w, dtype=np.float32)
    out = np.zeros((P, S, H), np.uint16)
    _load().zbo_combine(ctypes.byref(cfg.c()), dst_row.ctypes.data, y_bits.ctypes.data,
                        w.ctypes.data, out.ctypes.data)
    return out


def count(cfg: Config, ids_i: np.ndarray) -> np.ndarray:
    """Step 1 on one rank of a P-rank group: int32 ``[E+1]``, the counts of the
    rank's own ids ``[S,K]`` per expert, then the number of ids outside
    [0, E).  These rows are what the ranks exchange."""
    ids_i = np.ascontiguousarray(ids_i, dtype=np.int32).reshape(cfg.S, cfg.K)
    row = np.zeros(cfg.E + 1, np.int32)
    _load().zbo_count(ctypes.byref(cfg.c()), ids_i.ctypes.data, row.ctypes.data)
    return row


def plan_rank(cfg: Config, rank: int, counts: np.ndarray, ids_i: np.ndarray,
              placement: np.ndarray | None = None) -> dict:
    """Steps 2-3 as one rank computes them from the exchanged count rows
    ``counts`` int32 ``[P,E+1]`` and its own ids ``[S,K]``.  Returns the plan
    tables (as :func:`plan`) with ``dst_row`` ``[S,K]`` for this rank's
    entries only, and no ``row_src``."""
    lib = _load()
    P, E, K, S, R = cfg.P, cfg.E, cfg.K, cfg.S, cfg.R
    Eh = E // max(P, 1)
    counts = np.ascontiguousarray(counts, dtype=np.int32).reshape(P, E + 1)
    ids_i = np.ascontiguousarray(ids_i, dtype=np.int32).reshape(S, K)
    r = dict(
        cnt=np.zeros((P, E), np.int32), rep_expert=np.zeros((P, R), np.int32),
        rep_quota=np.zeros((P, R), np.int32), home_quota=np.zeros(E, np.int32),
        load_before=np.zeros(P, np.int32), load_after=np.zeros(P, np.int32),
        cu_seqlens=np.zeros((P, Eh + R + 1), np.int32), dst_row=np.zeros((S, K), np.int32))
    out = _Out(*[_ptr(r[k]) for k in ("cnt", "rep_expert", "rep_quota", "home_quota",
                                       "load_before", "load_after", "cu_seqlens", "dst_row")],
               _P32(), _P32(), 0, 0, 0, 0, 0, 0)
    pl = None if placement is None else \
        np.ascontiguousarray(placement, dtype=np.int32).reshape(P, R)
    st = lib.zbo_plan_rank(ctypes.byref(cfg.c()), int(rank), _ptr(counts), _ptr(ids_i),
                           _ptr(pl) if pl is not None else _P32(), ctypes.byref(out))
    r.update(status=int(st), locality_cost=int(out.locality_cost), max_load=int(out.max_load),
             n_replicas=int(out.n_replicas), n_iters=int(out.n_iters), T=int(out.water_level),
             repaired=int(out.repaired))
    return r


def _row_pointers(arrays, rows: int, H: int):
    ptrs = (ctypes.c_void_p * len(arrays))()
    for j, a in enumerate(arrays):
        assert a.dtype == np.uint16 and a.flags.c_contiguous and a.shape == (rows, H)
        ptrs[j] = a.ctypes.data
    return ptrs


def dispatch_ranks(cfg: Config, dst_i: np.ndarray, hidden_i: np.ndarray, bufs) -> None:
    """Step 4 on one rank: its rows ``hidden_i`` uint16 ``[S,H]`` written into
    the receive buffers ``bufs`` (P arrays uint16 ``[cap,H]``, one per
    destination rank) at the rows ``dst_i`` ``[S,K]`` name."""
    dst_i = np.ascontiguousarray(dst_i, dtype=np.int32).reshape(cfg.S, cfg.K)
    hidden_i = np.ascontiguousarray(hidden_i, dtype=np.uint16).reshape(cfg.S, cfg.H)
    ptrs = _row_pointers(bufs, cfg.cap(), cfg.H)
    _load().zbo_dispatch_ranks(ctypes.byref(cfg.c()), dst_i.ctypes.data, hidden_i.ctypes.data,
                               ptrs)


def combine_ranks(cfg: Config, dst_i: np.ndarray, ys, w_i: np.ndarray) -> np.ndarray:
    """Step 5 on one rank: uint16 ``[S,H]`` from the expert outputs ``ys`` (P
    arrays uint16 ``[cap,H]``, one per rank that computed them) and the
    rank's gates ``w_i`` float32 ``[S,K]``."""
    dst_i = np.ascontiguousarray(dst_i, dtype=np.int32).reshape(cfg.S, cfg.K)
    w_i = np.ascontiguousarray(w_i, dtype=np.float32).reshape(cfg.S, cfg.K)
    ptrs = _row_pointers(ys, cfg.cap(), cfg.H)
    out = np.zeros((cfg.S, cfg.H), np.uint16)
    _load().zbo_combine_ranks(ctypes.byref(cfg.c()), dst_i.ctypes.data, ptrs, w_i.ctypes.data,
                              out.ctypes.data)
    return out


def merge(cfg: Config, dst_row: np.ndarray) -> dict:
    """Merged dispatch layout of a plan: ``tok_row`` [P,S,K], ``grp_tok``
    [P,cap] and ``tok_cnt`` [P] (int32)."""
    P, S, K = cfg.P, cfg.S, cfg.K
    dst_row = np.ascontiguousarray(dst_row, dtype=np.int32)
    r = dict(tok_row=np.zeros((P, S, K), np.int32), grp_tok=np.zeros((P, cfg.cap()), np.int32),
             tok_cnt=np.zeros(P, np.int32))
    _load().zbo_merge(ctypes.byref(cfg.c()), dst_row.ctypes.data, r["tok_row"].ctypes.data,
                      r["grp_tok"].ctypes.data, r["tok_cnt"].ctypes.data)
    return r


def dispatch_merged(cfg: Config, tok_row: np.ndarray, hidden_bits: np.ndarray,
                    tbuf_bits: np.ndarray | None = None) -> np.ndarray:
    """Merged dispatch: one row per (token, destination rank) into ``tbuf``."""
    P, S, H = cfg.P, cfg.S, cfg.H
    hidden_bits = np.ascontiguousarray(hidden_bits, dtype=np.uint16).reshape(P, S, H)
    tok_row = np.ascontiguousarray(tok_row, dtype=np.int32)
    if tbuf_bits is None:
        tbuf_bits = np.zeros((P, cfg.cap(), H), np.uint16)
    _load().zbo_dispatch_merged(ctypes.byref(cfg.c()), tok_row.ctypes.data,
                                hidden_bits.ctypes.data, tbuf_bits.ctypes.data)
    return tbuf_bits


def place_by_demand(cfg: Config, demand: np.ndarray, with_blocked: bool = False):
    """Replica placement [P,R] from historical per-expert demand (int64 [E]);
    with ``with_blocked`` also the number of picks that fit nowhere."""
    demand = np.ascontiguousarray(demand, dtype=np.int64)
    pl = np.zeros((cfg.P, cfg.R), np.int32)
    blocked = np.zeros(1, np.int32)
    st = _load().zbo_place_by_demand(ctypes.byref(cfg.c()), demand.ctypes.data, _ptr(pl),
                                     _ptr(blocked))
    if st != OK:
        raise ValueError(f"zbo_place_by_demand: status {st}")
    return (pl, int(blocked[0])) if with_blocked else pl


def recalibrate(cfg: Config, cnt: np.ndarray, placement: np.ndarray, mode: int, eps: float,
                max_swaps: int) -> tuple[np.ndarray, int, int]:
    """Placement recalibration (mode 0: one slot changed per step; mode 1:
    intra-node slot swaps).  Returns (new placement, steps, final max load)."""
    cnt = np.ascontiguousarray(cnt, dtype=np.int32).reshape(cfg.P, cfg.E)
    pl = np.ascontiguousarray(placement, dtype=np.int32).reshape(cfg.P, cfg.R).copy()
    mx = np.zeros(1, np.int32)
    n = _load().zbo_recalibrate(ctypes.byref(cfg.c()), _ptr(cnt), _ptr(pl), int(mode),
                                float(eps), int(max_swaps), _ptr(mx))
    if n < 0:
        raise ValueError(f"zbo_recalibrate: status {n}")
    return pl, int(n), int(mx[0])


def combine_reduce(cfg: Config, dst_row: np.ndarray, tok_row: np.ndarray, y_bits: np.ndarray,
                   w: np.ndarray, part_bits: np.ndarray | None = None) -> np.ndarray:
    """Destination side of the merged combine: one bf16 partial per merged
    row, ``part`` uint16 ``[P,cap,H]`` (rows no token names keep their value)."""
    P, H = cfg.P, cfg.H
    dst_row = np.ascontiguousarray(dst_row, dtype=np.int32)
    tok_row = np.ascontiguousarray(tok_row, dtype=np.int32)
    y_bits = np.ascontiguousarray(y_bits, dtype=np.uint16)
    w = np.ascontiguousarray(w, dtype=np.float32)
    if part_bits is None:
        part_bits = np.zeros((P, cfg.cap(), H), np.uint16)
    _load().zbo_combine_reduce(ctypes.byref(cfg.c()), dst_row.ctypes.data, tok_row.ctypes.data,
                               y_bits.ctypes.data, w.ctypes.data, part_bits.ctypes.data)
    return part_bits


def combine_merged(cfg: Config, tok_row: np.ndarray, part_bits: np.ndarray) -> np.ndarray:
    """Source side of the merged combine: ``out`` uint16 ``[P,S,H]``."""
    P, S, H = cfg.P, cfg.S, cfg.H
    tok_row = np.ascontiguousarray(tok_row, dtype=np.int32)
    part_bits = np.ascontiguousarray(part_bits, dtype=np.uint16)
    out = np.zeros((P, S, H), np.uint16)
    _load().zbo_combine_merged(ctypes.byref(cfg.c()), tok_row.ctypes.data, part_bits.ctypes.data,
                               out.ctypes.data)
    return out


def f32_to_bf16(x: float) -> int:
    return int(_load().zbo_f32_to_bf16(ctypes.c_float(x)))


def bf16_to_f32(b: int) -> float:
    return float(_load().zbo_bf16_to_f32(ctypes.c_uint16(b)))


def metrics(cfg: Config, p: dict) -> dict:
    lib = _load()
    vals = [ctypes.c_double() for _ in range(4)]
    lib.zbo_metrics(ctypes.byref(cfg.c()), _ptr(p["cnt"]), _ptr(p["load_before"]),
                    _ptr(p["load_after"]), *[ctypes.byref(v) for v in vals])
    return dict(r_imb_before=vals[0].value, r_imb_after=vals[1].value, maxvio=vals[2].value,
                excess_removed=vals[3].value)
