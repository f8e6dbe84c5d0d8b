"""Pins of quota repair (ISER-MoE, HALO-Q stage 4: a circle-method
tournament over disjoint rank pairs that cancels opposite token flows).

* Every pair is visited: with P(P-1)/2 pairs that each hold one private pair
  of mutually copied experts with one row to cancel, repair cancels exactly
  one row per pair and every row is served locally (P = 2..9, odd P with a
  bye).
* One pair (P = 2) is one match: the rows moved equal min(sum a, sum b), with
  a and b computed here from the unrepaired quotas.
* Over random kept placements: rank loads and each expert's total quota are
  unchanged, quotas stay non-negative, only held copies change, and every
  row moved cancels one remote row each way, so the rows served locally
  rise by exactly twice the rows moved (and the flat cost falls by as much).
* One tournament is a fixed point: no pair can cancel in both directions.
"""
import itertools

import numpy as np
import pytest

import oracle


def _quota_table(cfg, p):
    """q[r, e] and held[r, e] from a plan's quota tables."""
    P, E, R = cfg.P, cfg.E, cfg.R
    Eh = E // P
    q = np.zeros((P, E), np.int64)
    held = np.zeros((P, E), bool)
    for e in range(E):
        q[e // Eh, e] = p["home_quota"][e]
        held[e // Eh, e] = True
    for j in range(P):
        for s in range(R):
            e = p["rep_expert"][j, s]
            if e >= 0:
                q[j, e] = p["rep_quota"][j, s]
                held[j, e] = True
    return q, held


def _local_rows(p):
    return int(sum(np.trace(m) for m in p["M"]))


@pytest.mark.parametrize("P", range(2, 10))
def test_every_pair_is_visited_once(P):
    # expert e(i, j) is homed on i (Eh = P-1 per rank) and copied on j; rank i
    # sends 3 rows of e(i, j) and 1 row of e(j, i) for every j != i
    Eh = P - 1
    E = P * Eh

    def ex(i, j):
        return i * Eh + (j if j < i else j - 1)
    pl = np.full((P, P - 1), -1, np.int32)
    ids = []
    for i in range(P):
        others = [j for j in range(P) if j != i]
        pl[i] = [ex(j, i) for j in others]
        ids.append(sum(([ex(i, j)] * 3 + [ex(j, i)] for j in others), []))
    ids = np.array(ids, np.int32)[:, :, None]
    S = ids.shape[1]
    base = dict(P=P, E=E, K=1, S=S, H=8, R=P - 1)
    p0 = oracle.plan(oracle.Config(**base), ids, placement=pl)
    p1 = oracle.plan(oracle.Config(**base, repair=1), ids, placement=pl)
    assert p0["status"] == p1["status"] == oracle.OK
    assert p0["locality_cost"] == P * (P - 1)  # one row each way per pair
    assert p1["repaired"] == P * (P - 1) // 2
    assert p1["locality_cost"] == 0
    np.testing.assert_array_equal(p1["load_after"], p0["load_after"])
    assert np.all(p1["rep_quota"] == 1) and np.all(p1["home_quota"] == 3)


def _random_placed(rng, P, Eh, K, S, R, skew):
    E = P * Eh
    pop = 1.0 / np.arange(1, E + 1) ** skew
    pop = pop[rng.permutation(E)]
    ids = rng.choice(E, size=(P, S, K), p=pop / pop.sum()).astype(np.int32)
    pl = np.full((P, R), -1, np.int32)
    for j in range(P):
        foreign = [e for e in range(E) if e // Eh != j]
        n = int(rng.integers(0, min(R, len(foreign)) + 1))
        pl[j, :n] = rng.choice(foreign, size=n, replace=False)
    return E, ids, pl


def test_one_pair_is_one_match():
    rng = np.random.default_rng(9)
    hits = 0
    for _ in range(200):
        E, ids, pl = _random_placed(rng, 2, int(rng.integers(1, 5)), int(rng.integers(1, 4)),
                                    int(rng.integers(1, 30)), 3 if rng.random() < 0.5 else 1,
                                    float(rng.uniform(0, 2)))
        R = pl.shape[1]
        if R > 1:
            continue  # R <= P - 1 = 1
        base = dict(P=2, E=E, K=ids.shape[2], S=ids.shape[1], H=8, R=R, cap_rows=10 ** 5)
        p0 = oracle.plan(oracle.Config(**base), ids, placement=pl)
        p1 = oracle.plan(oracle.Config(**base, repair=1), ids, placement=pl)
        q, held = _quota_table(oracle.Config(**base), p0)
        d = p0["cnt"].astype(np.int64)
        both = held[0] & held[1]
        sur = np.maximum(d - q, 0)
        spare = np.maximum(q - d, 0)
        sa = int(np.minimum(sur[0], spare[1])[both].sum())
        sb = int(np.minimum(sur[1], spare[0])[both].sum())
        assert p1["repaired"] == min(sa, sb)
        hits += p1["repaired"] > 0
    assert hits > 10


CASES = []
_rng = np.random.default_rng(31)
for _t in range(60):
    _P = int(_rng.choice([2, 3, 4, 5, 8]))
    _R = int(_rng.integers(1, _P))
    CASES.append((_P, _R) + _random_placed(_rng, _P, int(_rng.integers(1, 4)),
                                           int(_rng.integers(1, 5)), int(_rng.integers(0, 40)),
                                           _R, float(_rng.uniform(0, 2))))


@pytest.mark.parametrize("k", range(len(CASES)))
def test_repair_invariants(k):
    P, R, E, ids, pl = CASES[k]
    S, K = ids.shape[1], ids.shape[2]
    gpn = 2 if P % 2 == 0 and k % 3 == 0 else 1
    base = dict(P=P, E=E, K=K, S=S, H=8, R=R, gpus_per_node=gpn, cap_rows=P * S * K + 1)
    cfg = oracle.Config(**base, repair=1)
    for placement in (pl, None):
        p0 = oracle.plan(oracle.Config(**base), ids, placement=placement)
        p1 = oracle.plan(cfg, ids, placement=placement)
        assert p1["status"] == p0["status"]
        for key in ("cnt", "rep_expert", "load_before", "load_after"):
            np.testing.assert_array_equal(p1[key], p0[key], err_msg=key)
        assert p1["max_load"] == p0["max_load"]
        q0, held = _quota_table(cfg, p0)
        q1, _ = _quota_table(cfg, p1)
        np.testing.assert_array_equal(q1.sum(0), q0.sum(0))  # T_e
        np.testing.assert_array_equal(q1.sum(1), q0.sum(1))  # loads
        assert np.all(q1 >= 0) and np.all(q1[~held] == 0)
        if p1["status"] < 0:
            continue
        assert _local_rows(p1) == _local_rows(p0) + 2 * p1["repaired"]
        if gpn == 1:
            assert p1["locality_cost"] == p0["locality_cost"] - 2 * p1["repaired"]
        # rows stay a bijection onto the received rows, each in its expert's group
        cap = cfg.cap()
        dst = p1["dst_row"].ravel()
        la = p1["load_after"]
        valid = np.concatenate([j * cap + np.arange(la[j]) for j in range(P)])
        assert sorted(dst.tolist()) == sorted(valid.tolist())
        cu, Eh = p1["cu_seqlens"], E // P
        for g, row in enumerate(dst):
            j, r = divmod(int(row), cap)
            grp = int(np.searchsorted(cu[j], r, side="right") - 1)
            assert (j * Eh + grp if grp < Eh else p1["rep_expert"][j, grp - Eh]) == \
                ids.ravel()[g]


def test_one_tournament_leaves_no_pair_to_cancel():
    # A match only shrinks surpluses and spares: the rank taking quota of e
    # takes at most its surplus of e, the rank giving it gives at most its
    # spare.  So a pair whose sum a or sum b reached 0 in its match keeps it,
    # and after one tournament no pair can cancel in both directions.
    left = total = 0
    for P, R, E, ids, pl in CASES:
        S, K = ids.shape[1], ids.shape[2]
        cfg = oracle.Config(P=P, E=E, K=K, S=S, H=8, R=R, cap_rows=P * S * K + 1, repair=1)
        p = oracle.plan(cfg, ids, placement=pl)
        q, held = _quota_table(cfg, p)
        d = p["cnt"].astype(np.int64)
        sur, spare = np.maximum(d - q, 0), np.maximum(q - d, 0)
        for i, j in itertools.combinations(range(P), 2):
            both = held[i] & held[j]
            total += 1
            left += (np.minimum(sur[i], spare[j])[both].sum() > 0 and
                     np.minimum(sur[j], spare[i])[both].sum() > 0)
    assert total > 500 and left == 0
