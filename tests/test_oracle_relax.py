"""Pins of the relaxed transport: eq. (1) of Zepp 4.1 with its band
|sum_i M_ij - q_j| <= C q_j in use (relax = 1).

* A band of zero width (C = 0, or C below 1/q for every quota) reproduces the
  exact-quota plan table for table, and C is ignored while relax is off.
* eq. (1)'s constraints hold: every source's demand is routed, every host's
  receipt lies within its band; the greedy's quotas are untouched.
* With the flat cost the oracle's locality cost equals the optimum of eq. (1)
  solved as a linear program by scipy (the constraint matrix is a network
  matrix, so the LP optimum is the integer optimum).  With the two-level cost
  the LP is a lower bound, and the gap is reported.
* The band never serves fewer rows locally than exact quotas do.
"""
import numpy as np
import pytest
from scipy.optimize import linprog

import oracle

PLAN_KEYS = ("cnt", "rep_expert", "rep_quota", "home_quota", "load_before", "load_after",
             "cu_seqlens", "dst_row", "row_src", "M")


def _cost(gpn, i, j):
    if i == j:
        return 0
    if gpn > 1 and i // gpn != j // gpn:
        return 4
    return 1


def _case(rng, P, Eh, K, S, R, gpn, C, skew=1.3):
    E = P * Eh
    p = 1.0 / np.arange(1, E + 1) ** skew
    p = p[rng.permutation(E)]
    ids = rng.choice(E, size=(P, S, K), p=p / p.sum()).astype(np.int32)
    cfg = oracle.Config(P=P, E=E, K=K, S=S, H=8, R=R, C=C, gpus_per_node=gpn,
                        cap_rows=P * S * K + 1, relax=1)
    return cfg, ids


def _quotas(cfg, p, e):
    """q[j]: rows the plan's quotas give rank j for expert e."""
    Eh = cfg.E // cfg.P
    q = np.zeros(cfg.P, np.int64)
    q[e // Eh] = p["home_quota"][e]
    for j in range(cfg.P):
        for s in range(cfg.R):
            if p["rep_expert"][j, s] == e:
                q[j] = p["rep_quota"][j, s]
    return q


def _hosts(cfg, p, e):
    Eh = cfg.E // cfg.P
    return sorted({e // Eh} | {int(j) for j in np.nonzero((p["rep_expert"] == e).any(1))[0]})


def _c20(C):
    # C as the band uses it: float32, truncated to 20 fractional bits
    return np.floor(float(np.float32(C)) * 2.0 ** 20) / 2.0 ** 20


def _band_lp(cfg, e, cnt, q, hosts):
    """min sum a_ij M_ij s.t. sum_j M_ij = d_i, lo_j <= sum_i M_ij <= hi_j."""
    P = cfg.P
    srcs = [i for i in range(P) if cnt[i, e] > 0]
    if not srcs:
        return 0.0
    c20 = _c20(cfg.C)
    nh = len(hosts)
    nv = len(srcs) * nh
    c = [_cost(cfg.gpus_per_node, i, j) for i in srcs for j in hosts]
    A_eq = np.zeros((len(srcs), nv))
    for x, i in enumerate(srcs):
        A_eq[x, x * nh:(x + 1) * nh] = 1
    b_eq = [cnt[i, e] for i in srcs]
    A_ub, b_ub = [], []
    for y, j in enumerate(hosts):
        row = np.zeros(nv)
        row[y::nh] = 1
        dl = np.floor(q[j] * c20)
        A_ub.append(row); b_ub.append(q[j] + dl)
        A_ub.append(-row); b_ub.append(-(q[j] - dl))
    res = linprog(c, A_ub=np.array(A_ub), b_ub=np.array(b_ub), A_eq=A_eq, b_eq=b_eq,
                  bounds=(0, None), method="highs")
    assert res.status == 0
    return res.fun


def _cases(n, seed, gpns=(1, 2, 4)):
    rng = np.random.default_rng(seed)
    out = []
    for t in range(n):
        gpn = gpns[t % len(gpns)]
        P = int(rng.choice([4, 8])) if gpn > 1 else int(rng.choice([2, 3, 4, 8]))
        C = float(rng.choice([0.05, 0.1, 0.25, 0.5, 0.9]))
        out.append(_case(rng, P, int(rng.integers(1, 4)), int(rng.integers(1, 5)),
                         int(rng.integers(0, 40)), int(rng.integers(0, P)), gpn, C,
                         skew=float(rng.uniform(0.5, 2.5))))
    return out


CASES = _cases(60, 2024)


def test_zero_band_is_exact():
    rng = np.random.default_rng(5)
    for _ in range(30):
        cfg, ids = _case(rng, 4, 2, 3, int(rng.integers(1, 30)), 2, 2, 0.0)
        exact = oracle.plan(oracle.Config(**{**cfg.__dict__, "relax": 0}), ids)
        for C, relax in ((0.0, 1), (0.9, 0), (0.5 / (cfg.P * cfg.S * cfg.K + 1), 1)):
            p = oracle.plan(oracle.Config(**{**cfg.__dict__, "C": C, "relax": relax}), ids)
            assert p["status"] == exact["status"]
            for k in PLAN_KEYS:
                np.testing.assert_array_equal(p[k], exact[k], err_msg=(k, C, relax))
            assert p["locality_cost"] == exact["locality_cost"]


@pytest.mark.parametrize("k", range(len(CASES)))
def test_band_invariants(k):
    cfg, ids = CASES[k]
    P, E, K, S, R = cfg.P, cfg.E, cfg.K, cfg.S, cfg.R
    Eh, cap, N = E // P, cfg.cap(), P * S * K
    p = oracle.plan(cfg, ids)
    ex = oracle.plan(oracle.Config(**{**cfg.__dict__, "relax": 0}), ids)
    # the greedy (steps 1-2) is untouched by the band
    for key in ("cnt", "rep_expert", "rep_quota", "home_quota", "load_before"):
        np.testing.assert_array_equal(p[key], ex[key], err_msg=key)
    assert (p["n_iters"], p["n_replicas"], p["T"]) == (ex["n_iters"], ex["n_replicas"], ex["T"])
    quota_load = ex["load_after"]
    assert (p["status"] == oracle.UNBALANCED) == (quota_load.max(initial=0) > p["T"])

    M = p["M"]
    assert np.all(M >= 0)
    np.testing.assert_array_equal(M.sum(2), p["cnt"].T)  # every demand routed
    local_relaxed = local_exact = 0
    for e in range(E):
        q = _quotas(cfg, p, e)
        recv = M[e].sum(0)
        assert np.all(np.abs(recv - q) <= cfg.C * q), (e, recv, q)
        hosts = _hosts(cfg, p, e)
        off = np.ones(P, bool)
        off[hosts] = False
        assert np.all(M[e][:, off] == 0)
        local_relaxed += int(np.trace(M[e]))
        local_exact += int(np.trace(ex["M"][e]))
    assert local_relaxed >= local_exact

    # what each rank receives, and the buffers
    la = p["load_after"]
    assert la.sum() == N and p["max_load"] == la.max(initial=0)
    c20 = _c20(cfg.C)
    for j in range(P):
        assert la[j] == sum(M[e][:, j].sum() for e in range(E))
        assert la[j] <= quota_load[j] + np.floor(quota_load[j] * c20)
    cu = p["cu_seqlens"]
    np.testing.assert_array_equal(cu[:, -1], la)
    assert np.all(np.diff(cu, axis=1) >= 0)
    A = np.array([[_cost(cfg.gpus_per_node, i, j) for j in range(P)] for i in range(P)])
    assert p["locality_cost"] == int((M * A[None]).sum())

    # rows: each (token,k) once, in a group of its expert, below its rank's
    # load; groups ordered by (source rank, flat index)
    dst = p["dst_row"].ravel()
    valid = np.concatenate([j * cap + np.arange(la[j]) for j in range(P)])
    assert sorted(dst.tolist()) == sorted(valid.tolist())
    rs = p["row_src"].ravel()
    np.testing.assert_array_equal(rs[dst], np.arange(N))
    flat = ids.ravel()
    for g, row in enumerate(dst):
        j, r = divmod(int(row), cap)
        grp = int(np.searchsorted(cu[j], r, side="right") - 1)
        assert (j * Eh + grp if grp < Eh else p["rep_expert"][j, grp - Eh]) == flat[g]
    for j in range(P):
        src = rs[j * cap:j * cap + la[j]]
        for grp in range(Eh + R):
            assert np.all(np.diff(src[cu[j, grp]:cu[j, grp + 1]]) > 0)


def test_default_buffers_hold_a_balanced_plan():
    rng = np.random.default_rng(11)
    for C in (0.05, 0.1, 0.3, 0.5, 0.99):
        for _ in range(8):
            cfg, ids = _case(rng, 8, 2, 4, int(rng.integers(1, 64)), 3, 2, C, skew=0.8)
            cfg.cap_rows = None
            sk = cfg.S * cfg.K
            assert cfg.cap() == sk + int(np.floor(sk * _c20(C)))
            p = oracle.plan(cfg, ids)
            if p["status"] == oracle.OK:
                assert p["max_load"] <= cfg.cap()
            else:  # quota loads above T may overflow the band's buffers
                assert p["status"] in (oracle.UNBALANCED, oracle.ERR_CAPACITY)


def test_band_capacity_error():
    # the band lets a rank receive more than S*K: with S*K buffers that is a
    # capacity error, with rows left unassigned
    cfg = oracle.Config(P=2, E=2, K=1, S=4, H=8, R=1, C=0.5, relax=1, cap_rows=4)
    ids = np.array([[0, 0, 1, 1], [0, 0, 0, 0]], np.int32).reshape(2, 4, 1)
    p = oracle.plan(cfg, ids)
    assert p["status"] == oracle.ERR_CAPACITY and p["max_load"] == 5
    assert np.all(p["dst_row"] == -1) and np.all(p["row_src"] == -1)


@pytest.mark.parametrize("seed", range(4))
def test_flat_band_is_lp_optimal(seed):
    for cfg, ids in _cases(12, 300 + seed, gpns=(1,)):
        p = oracle.plan(cfg, ids)
        lp = sum(_band_lp(cfg, e, p["cnt"], _quotas(cfg, p, e), _hosts(cfg, p, e))
                 for e in range(cfg.E))
        assert p["locality_cost"] == pytest.approx(lp, abs=1e-6), (cfg, ids.tolist())


def test_two_level_band_lp_gap():
    gaps = []
    for cfg, ids in _cases(40, 77, gpns=(2, 4)):
        p = oracle.plan(cfg, ids)
        lp = sum(_band_lp(cfg, e, p["cnt"], _quotas(cfg, p, e), _hosts(cfg, p, e))
                 for e in range(cfg.E))
        assert p["locality_cost"] >= lp - 1e-6
        gaps.append(p["locality_cost"] - lp)
    # reported, not asserted: the greedy third step against the LP optimum
    print("two-level band: cost - LP:", np.round(sorted(gaps), 1).tolist())
