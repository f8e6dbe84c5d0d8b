"""Pins of placement recalibration between invocations: ViBE's incremental
update (mode 0: one helper slot changes per step) and Zepp's intra-node swaps
(eq. (4); mode 1: two slots of one node exchange their experts).

* A hand-worked case: one slot change balances two ranks.
* Already within eps of the mean: nothing changes.
* Each step equals a brute force over every candidate, enumerated here in the
  stated order and scored by the oracle's own kept-placement plan
  (max_load), with the first strict minimum taken; whole searches match the
  brute force step by step.
* Invariants: the max load never rises, placements stay valid, intra-node
  swaps keep each node's set of held experts, and a search that stops early
  stops because no candidate improves.
"""
import numpy as np
import pytest

import oracle


def test_hand_example():
    # P = 2, E = 2, R = 1, slots empty.  Rank 0 sends [0,0,0,0], rank 1 sends
    # [0,0,1,1]: T_0 = 6, T_1 = 2, L = [6, 2], T = 4; the kept (empty)
    # placement leaves max load 6 > 1.03 * 4.  Candidates in order: slot 0
    # (rank 0) can take only expert 1 (expert 0 is homed there): no help, max
    # 6.  Slot 1 (rank 1) takes expert 0: the greedy moves m = min(6-4, 4-2,
    # 6) = 2, loads [4, 4], max 4 <= 4.12: one step, then done.
    cfg = oracle.Config(P=2, E=2, K=1, S=4, H=8, R=1)
    ids = np.array([[0, 0, 0, 0], [0, 0, 1, 1]], np.int32).reshape(2, 4, 1)
    cnt = oracle.plan(cfg, ids, want_M=False, placement=np.full((2, 1), -1, np.int32))["cnt"]
    pl, n, mx = oracle.recalibrate(cfg, cnt, np.full((2, 1), -1, np.int32), 0, 0.03, 10)
    assert (n, mx) == (1, 4)
    np.testing.assert_array_equal(pl, [[-1], [0]])


def _max_load(cfg, ids, pl):
    return oracle.plan(cfg, ids, want_M=False, placement=pl)["max_load"]


def _valid(cfg, pl, r, s, e):
    Eh = cfg.E // cfg.P
    return e // Eh != r and all(pl[r, t] != e for t in range(cfg.R) if t != s)


def _candidates(cfg, pl, mode):
    P, R, E = cfg.P, cfg.R, cfg.E
    out = []
    if mode == 0:
        for x in range(P * R):
            r, s = divmod(x, R)
            for e in range(E):
                if e != pl[r, s] and _valid(cfg, pl, r, s, e):
                    q = pl.copy()
                    q[r, s] = e
                    out.append(q)
    else:
        g = cfg.gpus_per_node
        for x1 in range(P * R):
            for x2 in range(x1 + 1, P * R):
                (r1, s1), (r2, s2) = divmod(x1, R), divmod(x2, R)
                e1, e2 = pl[r1, s1], pl[r2, s2]
                if r1 == r2 or r1 // g != r2 // g or e1 == e2:
                    continue
                if e2 >= 0 and not _valid(cfg, pl, r1, s1, e2):
                    continue
                if e1 >= 0 and not _valid(cfg, pl, r2, s2, e1):
                    continue
                q = pl.copy()
                q[r1, s1], q[r2, s2] = e2, e1
                out.append(q)
    return out


def _brute(cfg, ids, pl, mode, eps, max_swaps):
    """The whole search, step by step, scored by the oracle's plan."""
    total = cfg.P * cfg.S * cfg.K
    bound = (1.0 + float(np.float32(eps))) * total / cfg.P
    cur = _max_load(cfg, ids, pl)
    steps = 0
    while steps < max_swaps and cur > bound:
        best, pick = cur, None
        for q in _candidates(cfg, pl, mode):
            m = _max_load(cfg, ids, q)
            if m < best:
                best, pick = m, q
        if pick is None:
            break
        pl, cur, steps = pick, best, steps + 1
    return pl, steps, cur


def _case(rng, P, Eh, K, S, R, gpn, skew):
    E = P * Eh
    pop = 1.0 / np.arange(1, E + 1) ** skew
    ids = rng.choice(E, size=(P, S, K), p=pop / pop.sum()).astype(np.int32)
    pl = np.full((P, R), -1, np.int32)
    for j in range(P):  # a random valid start
        foreign = [e for e in range(E) if e // Eh != j]
        k = int(rng.integers(0, R + 1))
        pl[j, :k] = rng.choice(foreign, size=k, replace=False)
    cfg = oracle.Config(P=P, E=E, K=K, S=S, H=8, R=R, gpus_per_node=gpn,
                        cap_rows=P * S * K)
    return cfg, ids, pl


@pytest.mark.parametrize("seed", range(12))
def test_search_matches_brute_force(seed):
    rng = np.random.default_rng(900 + seed)
    mode = seed % 2
    P = 4
    gpn = 2 if mode == 1 else int(rng.choice([1, 2]))
    cfg, ids, pl = _case(rng, P, int(rng.integers(1, 3)), int(rng.integers(1, 3)),
                         int(rng.integers(2, 10)), int(rng.integers(1, 3)), gpn,
                         float(rng.uniform(1.0, 2.5)))
    cnt = oracle.plan(cfg, ids, want_M=False, placement=pl)["cnt"]
    got = oracle.recalibrate(cfg, cnt, pl, mode, 0.03, 6)
    want = _brute(cfg, ids, pl.copy(), mode, 0.03, 6)
    np.testing.assert_array_equal(got[0], want[0])
    assert got[1:] == want[1:]


@pytest.mark.parametrize("seed", [2, 5, 10, 22, 24, 26, 28, 29])
def test_intra_node_search_matches_brute_force(seed):
    # seeds where an intra-node swap lowers the max load (nodes of P/2 or 3)
    rng = np.random.default_rng(5000 + seed)
    P = int(rng.choice([4, 6]))
    cfg, ids, pl = _case(rng, P, int(rng.integers(1, 3)), int(rng.integers(1, 4)),
                         int(rng.integers(4, 16)), int(rng.integers(1, 3)),
                         P // 2 if P == 4 else 3, float(rng.uniform(1.0, 2.5)))
    cnt = oracle.plan(cfg, ids, want_M=False, placement=pl)["cnt"]
    got = oracle.recalibrate(cfg, cnt, pl, 1, 0.03, 6)
    want = _brute(cfg, ids, pl.copy(), 1, 0.03, 6)
    assert got[1] >= 1
    np.testing.assert_array_equal(got[0], want[0])
    assert got[1:] == want[1:]


@pytest.mark.parametrize("seed", range(20))
def test_invariants(seed):
    rng = np.random.default_rng(1200 + seed)
    mode = seed % 2
    P = int(rng.choice([4, 6, 8]))
    gpn = 2 if mode == 1 else 1
    cfg, ids, pl = _case(rng, P, int(rng.integers(1, 4)), int(rng.integers(1, 5)),
                         int(rng.integers(4, 40)), int(rng.integers(1, 4)), gpn,
                         float(rng.uniform(0.8, 2.5)))
    cnt = oracle.plan(cfg, ids, want_M=False, placement=pl)["cnt"]
    before = _max_load(cfg, ids, pl)
    prev = before
    cur_pl = pl
    for step in range(4):  # one step at a time: the max load never rises
        nxt, n, mx = oracle.recalibrate(cfg, cnt, cur_pl, mode, 0.03, 1)
        assert n in (0, 1) and mx <= prev and mx == _max_load(cfg, ids, nxt)
        assert oracle.plan(cfg, ids, want_M=False, placement=nxt)["status"] >= 0
        if mode == 1:  # each node keeps its set of held experts
            g = cfg.gpus_per_node
            for nd in range(P // g):
                a = sorted(e for e in cur_pl[nd * g:(nd + 1) * g].ravel() if e >= 0)
                b = sorted(e for e in nxt[nd * g:(nd + 1) * g].ravel() if e >= 0)
                assert a == b
        if n == 0:
            bound = (1 + float(np.float32(0.03))) * P * cfg.S * cfg.K / P
            if mx > bound:  # stopped early: no candidate improves
                assert all(_max_load(cfg, ids, q) >= mx
                           for q in _candidates(cfg, cur_pl, mode)[:200])
            break
        cur_pl, prev = nxt, mx


def test_within_eps_changes_nothing():
    rng = np.random.default_rng(5)
    cfg, ids, pl = _case(rng, 4, 2, 2, 16, 2, 1, 0.0)  # uniform popularity
    cnt = oracle.plan(cfg, ids, want_M=False, placement=pl)["cnt"]
    mx0 = _max_load(cfg, ids, pl)
    eps = (mx0 * cfg.P / (cfg.P * cfg.S * cfg.K)) - 1 + 1e-3  # loose enough to hold
    out, n, mx = oracle.recalibrate(cfg, cnt, pl, 0, eps, 5)
    assert n == 0 and mx == mx0
    np.testing.assert_array_equal(out, pl)
