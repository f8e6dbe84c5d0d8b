"""Pins of the oracle's plan with a given replica placement (quotas only).

A placement kept across invocations (Zepp 4.1: replicas from historical
demand; ViBE: re-placement only on drift) leaves one decision per invocation:
how many rows each existing copy takes.  The oracle answers with the greedy
of the full planner restricted to existing copies.  Pinned by a hand-worked
example, the plan invariants, and a max-flow optimum for the fixed placement.
"""
import numpy as np
import pytest
from scipy.sparse import csr_matrix
from scipy.sparse.csgraph import maximum_flow

import oracle


def test_hand_example_useless_copy():
    # Ex1's routing (P=2, E=4, rank 0 homes experts 0 and 1; T = 4, L = [7, 1]).
    # With rank 1's slot holding expert 1 instead of expert 0: the only
    # movable rows are expert 1's 2; after that rank 0 is stuck at 5.
    ids = np.array([[0, 0, 0, 1], [0, 1, 0, 2]], np.int32).reshape(2, 4, 1)
    cfg = oracle.Config(P=2, E=4, K=1, S=4, H=8, R=1, cap_rows=5)
    p = oracle.plan(cfg, ids, placement=np.array([[-1], [1]], np.int32))
    assert p["status"] == oracle.UNBALANCED
    np.testing.assert_array_equal(p["rep_expert"], [[-1], [1]])
    np.testing.assert_array_equal(p["rep_quota"], [[0], [2]])
    np.testing.assert_array_equal(p["home_quota"], [5, 0, 1, 0])
    np.testing.assert_array_equal(p["load_after"], [5, 3])
    # with the copy of expert 0 the full planner would have chosen, the
    # restricted greedy reproduces the full plan (one move of 3 rows)
    full = oracle.plan(cfg, ids)
    kept = oracle.plan(cfg, ids, placement=full["rep_expert"])
    for k in ("rep_expert", "rep_quota", "home_quota", "load_after", "cu_seqlens", "dst_row"):
        np.testing.assert_array_equal(kept[k], full[k], err_msg=k)


def test_invalid_placements():
    # P=3, E=6: rank 0 homes experts 0,1; rank 1 experts 2,3; rank 2 experts 4,5
    cfg = oracle.Config(P=3, E=6, K=1, S=2, H=8, R=2, cap_rows=6)
    ids = np.zeros((3, 2, 1), np.int32)
    empty = [[-1, -1], [-1, -1]]
    for bad in ([[0, -1]] + empty,        # expert 0 is homed on rank 0
                [[2, 2]] + empty,         # twice on one rank
                [[6, -1]] + empty,        # outside [0, E)
                [[-2, -1]] + empty):
        assert oracle.plan(cfg, ids, placement=np.array(bad, np.int32))["status"] == \
            oracle.ERR_INVALID
    ok = oracle.plan(cfg, ids, placement=np.array([[2, 4], [0, -1], [-1, 1]], np.int32))
    assert ok["status"] in (oracle.OK, oracle.UNBALANCED)


def _random_placement(rng, P, E, R):
    Eh = E // P
    pl = np.full((P, R), -1, np.int32)
    for j in range(P):
        others = [e for e in range(E) if e // Eh != j]
        n = int(rng.integers(0, min(R, len(others)) + 1))
        pl[j, :n] = rng.choice(others, size=n, replace=False)
    return pl


def _opt_fixed(P, E, Eh, Te, pl):
    """Least feasible max rank load for a fixed placement (max-flow, bisection)."""
    N = int(Te.sum())
    hosts = [{e // Eh} for e in range(E)]
    for j in range(P):
        for e in pl[j]:
            if e >= 0:
                hosts[e].add(j)
    lo, hi = -(-N // P), N
    while lo < hi:
        mid = (lo + hi) // 2
        n = E + P + 2
        src, dst, cap = [], [], []
        for e in range(E):
            if Te[e]:
                src.append(0); dst.append(1 + e); cap.append(int(Te[e]))
                for j in hosts[e]:
                    src.append(1 + e); dst.append(1 + E + j); cap.append(int(Te[e]))
        for j in range(P):
            src.append(1 + E + j); dst.append(n - 1); cap.append(mid)
        g = csr_matrix((np.array(cap, np.int32), (src, dst)), shape=(n, n))
        if maximum_flow(g, 0, n - 1).flow_value == N:
            hi = mid
        else:
            lo = mid + 1
    return lo


@pytest.mark.parametrize("seed", range(4))
def test_placed_invariants_and_optimum(seed):
    rng = np.random.default_rng(50 + seed)
    gaps = []
    for _ in range(40):
        P = int(rng.choice([2, 3, 4, 6]))
        Eh = int(rng.integers(1, 4))
        E = P * Eh
        K = int(rng.integers(1, 4))
        S = int(rng.integers(1, 20))
        R = int(rng.integers(1, P))
        p = rng.dirichlet(np.full(E, 0.5))
        ids = rng.choice(E, size=(P, S, K), p=p).astype(np.int32)
        pl = _random_placement(rng, P, E, R)
        cfg = oracle.Config(P=P, E=E, K=K, S=S, H=8, R=R, cap_rows=P * S * K)
        out = oracle.plan(cfg, ids, placement=pl)
        assert out["status"] in (oracle.OK, oracle.UNBALANCED)
        np.testing.assert_array_equal(out["rep_expert"], pl)
        T, L, la = out["T"], out["load_before"], out["load_after"]
        assert la.sum() == P * S * K
        for j in range(P):
            if L[j] <= T:
                assert la[j] <= T
            else:
                assert T <= la[j] <= L[j]
        assert out["n_iters"] <= 3 * P + E
        Te = out["cnt"].sum(0)
        tot = out["home_quota"].astype(np.int64).copy()
        for j in range(P):
            for s in range(R):
                if pl[j, s] >= 0:
                    tot[pl[j, s]] += out["rep_quota"][j, s]
                else:
                    assert out["rep_quota"][j, s] == 0
        np.testing.assert_array_equal(tot, Te)
        # rows: a bijection onto the filled rows, as for a chosen placement
        dst = np.sort(out["dst_row"].ravel())
        cap = cfg.cap()
        want = np.sort(np.concatenate([j * cap + np.arange(la[j]) for j in range(P)]))
        np.testing.assert_array_equal(dst, want)
        opt = _opt_fixed(P, E, Eh, Te, pl)
        assert opt <= out["max_load"]
        if out["max_load"] == T:
            assert opt == T
        gaps.append(out["max_load"] - opt)
    print("restricted greedy - OPT(placement):", np.bincount(gaps).tolist())
