"""Pins of the CPU oracle's plan (steps 1-3) against what the pages fix.

Each test ties the oracle to something other than itself: hand-worked
examples, closed forms (the water level, the transport lower bound), textbook
routines (numpy bincount, a stable argsort), brute-force recomputation, and
the invariants that the method states (every (token,k) routed exactly once,
no rank above T where R permits, eq. (1)'s constraints).
"""
import itertools
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")


def _cfg(d):
    return oracle.Config(P=d["P"], E=d["E"], K=d["K"], S=d["S"], H=d["H"], R=d["R"],
                         C=d.get("C", 0.0), gpus_per_node=d.get("gpus_per_node", 1),
                         cap_rows=d.get("cap_rows"), policy=d.get("policy", 0),
                         relax=d.get("relax", 0), repair=d.get("repair", 0))


def _examples():
    return json.load(open(GOLDEN))["examples"]


@pytest.mark.parametrize("ex", _examples(), ids=lambda e: e["name"])
def test_hand_examples(ex):
    cfg = _cfg(ex["cfg"])
    ids = np.array(ex["ids"], np.int32).reshape(cfg.P, cfg.S, cfg.K)
    pl = np.array(ex["placement"], np.int32) if "placement" in ex else None
    p = oracle.plan(cfg, ids, placement=pl)
    exp = ex["expect"]
    assert p["status"] == exp["status"]
    assert p["T"] == exp["T"]
    for key in ("cnt", "load_before", "load_after", "rep_expert", "rep_quota", "home_quota",
                "cu_seqlens"):
        if key in exp:
            np.testing.assert_array_equal(p[key], np.array(exp[key]), err_msg=key)
    if "dst_row" in exp:
        np.testing.assert_array_equal(p["dst_row"].reshape(cfg.P, -1), np.array(exp["dst_row"]))
    if "locality_cost" in exp:
        assert p["locality_cost"] == exp["locality_cost"]
    m = oracle.metrics(cfg, p)
    for key in ("r_imb_before", "r_imb_after", "maxvio", "excess_removed"):
        if key in exp:
            assert m[key] == pytest.approx(exp[key], abs=1e-12)
    if "cap" in exp:
        assert cfg.cap() == exp["cap"]
    if "locality_cost_exact_quotas" in exp:
        cfg0 = _cfg(dict(ex["cfg"], relax=0, repair=0))
        assert oracle.plan(cfg0, ids, placement=pl)["locality_cost"] == \
            exp["locality_cost_exact_quotas"]
    if "repaired" in exp:
        assert p["repaired"] == exp["repaired"]
    if "status_with_cap_rows_3" in exp:
        cfg.cap_rows = 3
        assert oracle.plan(cfg, ids)["status"] == exp["status_with_cap_rows_3"]


# ---------------------------------------------------------------- random cases

def _random_case(rng, P, Eh, K, S, R, gpn=1, skew=1.5, cap_extra=None, policy=0):
    E = P * Eh
    p = 1.0 / np.arange(1, E + 1) ** skew
    p = p[rng.permutation(E)] if rng.random() < 0.5 else p
    p /= p.sum()
    # each token draws K experts (duplicates within a token are allowed)
    ids = rng.choice(E, size=(P, S, K), p=p).astype(np.int32)
    cap = None if cap_extra is None else S * K + cap_extra
    return oracle.Config(P=P, E=E, K=K, S=S, H=8, R=R, C=0.1, gpus_per_node=gpn,
                         cap_rows=cap, policy=policy), ids


def _cases(n=120, seed=7):
    rng = np.random.default_rng(seed)
    out = []
    for t in range(n):
        P = int(rng.choice([1, 2, 3, 4, 6, 8]))
        gpn = 1
        if P in (4, 6, 8) and rng.random() < 0.4:
            gpn = 2
        Eh = int(rng.integers(1, 5))
        K = int(rng.integers(1, 5))
        S = int(rng.integers(0, 12))
        R = int(rng.integers(0, P)) if P > 1 else 0
        out.append(_random_case(rng, P, Eh, K, S, R, gpn, skew=float(rng.uniform(0, 2.5)),
                                cap_extra=10 ** 6, policy=t % 2))
    return out


CASES = _cases()


def _cost(cfg, i, j):
    if i == j:
        return 0
    if cfg.gpus_per_node > 1 and i // cfg.gpus_per_node != j // cfg.gpus_per_node:
        return 4
    return 1


@pytest.mark.parametrize("k", range(len(CASES)))
def test_plan_invariants(k):
    cfg, ids = CASES[k]
    P, E, K, S, R = cfg.P, cfg.E, cfg.K, cfg.S, cfg.R
    Eh, cap, N = E // P, cfg.cap(), P * S * K
    p = oracle.plan(cfg, ids)
    assert p["status"] in (oracle.OK, oracle.UNBALANCED)

    # step 1: histogram == numpy.bincount per rank
    for i in range(P):
        np.testing.assert_array_equal(p["cnt"][i], np.bincount(ids[i].ravel(), minlength=E))
    Te = p["cnt"].sum(0)
    L = np.array([Te[j * Eh:(j + 1) * Eh].sum() for j in range(P)])
    np.testing.assert_array_equal(p["load_before"], L)

    # water level: ceil(sum L / P), which equals S*K since every entry routes once
    assert p["T"] == -(-int(L.sum()) // P) == S * K

    # loads: conservation, receivers never above T, donors never below T
    la = p["load_after"]
    assert la.sum() == N
    for j in range(P):
        if L[j] <= p["T"]:
            assert la[j] <= p["T"]
        else:
            assert p["T"] <= la[j] <= L[j]
    assert p["max_load"] == la.max(initial=0)
    assert (p["status"] == oracle.UNBALANCED) == (la.max(initial=0) > p["T"])
    assert p["n_iters"] <= P * R + P

    # replica table: filled lowest slot first, never on the home rank, at
    # most one copy of an expert per rank, positive quotas
    re, rq = p["rep_expert"], p["rep_quota"]
    for j in range(P):
        filled = re[j] >= 0
        assert not np.any(filled[1:] & ~filled[:-1])
        assert np.all(rq[j][~filled] == 0) and np.all(rq[j][filled] >= 1)
        assert len(set(re[j][filled].tolist())) == filled.sum()
        assert not np.any(re[j][filled] // Eh == j)
    assert p["n_replicas"] == int((re >= 0).sum())

    # quotas: home + replicas = T_e; rank load = sum of its quotas
    tot = p["home_quota"].astype(np.int64).copy()
    for j in range(P):
        for s in range(R):
            if re[j, s] >= 0:
                tot[re[j, s]] += rq[j, s]
    np.testing.assert_array_equal(tot, Te)
    for j in range(P):
        assert la[j] == p["home_quota"][j * Eh:(j + 1) * Eh].sum() + rq[j].sum()

    # eq. (1): sum_j M_ij = d_i; |sum_i M_ij - q_j| <= C q_j (here exactly 0);
    # M_ij = 0 where j does not host e
    M = p["M"]
    assert np.all(M >= 0)
    np.testing.assert_array_equal(M.sum(2), p["cnt"].T)
    for e in range(E):
        q = np.zeros(P, np.int64)
        q[e // Eh] = p["home_quota"][e]
        for j in range(P):
            for s in range(R):
                if re[j, s] == e:
                    q[j] = rq[j, s]
        recv = M[e].sum(0)
        assert np.all(np.abs(recv - q) <= cfg.C * q)
        np.testing.assert_array_equal(recv, q)
        host = (q > 0) | (np.arange(P) == e // Eh) | np.isin(np.arange(P), np.nonzero(re == e)[0])
        assert np.all(M[e][:, ~host] == 0)

    # locality cost = sum a_ij M^e_ij, and it meets the closed-form lower bound
    A = np.array([[_cost(cfg, i, j) for j in range(P)] for i in range(P)])
    assert p["locality_cost"] == int((M * A[None]).sum())
    x_gpu = 0
    x_node = 0
    gpn = cfg.gpus_per_node
    for e in range(E):
        d = p["cnt"][:, e].astype(np.int64)
        q = M[e].sum(0)
        x_gpu += np.maximum(d - q, 0).sum()
        if gpn > 1:
            Dn = d.reshape(-1, gpn).sum(1)
            Qn = q.reshape(-1, gpn).sum(1)
            x_node += np.maximum(Dn - Qn, 0).sum()
    assert p["locality_cost"] == x_gpu + 3 * x_node

    # cu_seqlens: monotone prefix of per-group receipts, last = load
    cu = p["cu_seqlens"]
    assert cu.shape == (P, Eh + R + 1)
    assert np.all(cu[:, 0] == 0) and np.all(np.diff(cu, axis=1) >= 0)
    np.testing.assert_array_equal(cu[:, -1], la)

    # every (token,k) lands exactly once, inside its rank's filled rows, in a
    # group whose expert is the entry's id; row_src inverts dst_row
    dst = p["dst_row"].ravel()
    valid = np.concatenate([j * cap + np.arange(la[j]) for j in range(P)]) if P else []
    assert sorted(dst.tolist()) == sorted(np.asarray(valid).tolist())
    rs = p["row_src"].ravel()
    np.testing.assert_array_equal(rs[dst], np.arange(N))
    assert np.all(rs[np.setdiff1d(np.arange(P * cap), dst)] == -1)
    flat_ids = ids.ravel()
    for g, row in enumerate(dst):
        j, r = divmod(int(row), cap)
        grp = int(np.searchsorted(cu[j], r, side="right") - 1)
        exp_e = j * Eh + grp if grp < Eh else re[j, grp - Eh]
        assert exp_e == flat_ids[g]
    # inside each group, rows are ordered by (source rank, flat index)
    for j in range(P):
        src = rs[j * cap:j * cap + la[j]]
        for grp in range(Eh + R):
            seg = src[cu[j, grp]:cu[j, grp + 1]]
            assert np.all(np.diff(seg) > 0)


def test_no_slots_is_a_stable_sort():
    """With R = 0 each expert has one host (its home), so dst_row must equal a
    stable argsort of the entries by (home rank, expert, global index)."""
    rng = np.random.default_rng(3)
    for _ in range(20):
        P, Eh, K, S = 4, 3, 3, int(rng.integers(1, 40))
        E = P * Eh
        ids = rng.integers(0, E, size=(P, S, K)).astype(np.int32)
        N = P * S * K
        cfg = oracle.Config(P=P, E=E, K=K, S=S, H=8, R=0, cap_rows=N)
        p = oracle.plan(cfg, ids)
        flat = ids.ravel()
        home = flat // Eh
        for j in range(P):
            mine = np.nonzero(home == j)[0]
            order = mine[np.argsort(flat[mine], kind="stable")]
            exp = np.empty(N, np.int64)
            exp[order] = j * N + np.arange(len(order))
            np.testing.assert_array_equal(p["dst_row"].ravel()[mine], exp[mine])


def test_ties_go_to_lowest_expert_and_rank():
    # two donors tie at load 4 (ranks 0 and 1), T = 2; rank 0 wins.  Its two
    # experts tie at quota 2; expert 0 wins.  Receivers 2 and 3 tie at load 0;
    # rank 2 wins.
    P, E, K, S, R = 4, 8, 1, 2, 1
    ids = np.array([[0, 1], [0, 1], [2, 3], [2, 3]], np.int32).reshape(P, S, K)
    p = oracle.plan(oracle.Config(P=P, E=E, K=K, S=S, H=8, R=R), ids)
    np.testing.assert_array_equal(p["load_before"], [4, 4, 0, 0])
    np.testing.assert_array_equal(p["rep_expert"].ravel(), [-1, -1, 0, 2])
    np.testing.assert_array_equal(p["rep_quota"].ravel(), [0, 0, 2, 2])
    assert p["status"] == oracle.OK


def test_degenerate_shapes():
    # empty input
    cfg = oracle.Config(P=4, E=8, K=2, S=0, H=8, R=1)
    p = oracle.plan(cfg, np.zeros((4, 0, 2), np.int32))
    assert p["status"] == oracle.OK and p["T"] == 0 and p["n_replicas"] == 0
    assert np.all(p["cu_seqlens"] == 0)
    # one rank
    cfg = oracle.Config(P=1, E=5, K=3, S=7, H=8, R=0)
    ids = np.random.default_rng(0).integers(0, 5, (1, 7, 3)).astype(np.int32)
    p = oracle.plan(cfg, ids)
    assert p["status"] == oracle.OK and p["load_after"][0] == 21
    # everything on one expert
    cfg = oracle.Config(P=4, E=4, K=1, S=8, H=8, R=3)
    p = oracle.plan(cfg, np.zeros((4, 8, 1), np.int32))
    assert p["status"] == oracle.OK
    np.testing.assert_array_equal(p["load_after"], [8, 8, 8, 8])
    # uniform routing needs no replica
    ids = np.tile(np.arange(8, dtype=np.int32), (4, 1)).reshape(4, 8, 1)
    p = oracle.plan(oracle.Config(P=4, E=8, K=1, S=8, H=8, R=2), ids)
    assert p["n_replicas"] == 0 and p["n_iters"] == 0


def test_errors():
    ids = np.zeros((2, 2, 1), np.int32)
    for bad in [dict(P=0), dict(E=3), dict(E=400), dict(K=0), dict(K=17), dict(H=12), dict(H=0),
                dict(R=2), dict(R=-1), dict(C=1.0), dict(C=-0.1), dict(gpus_per_node=3),
                dict(policy=2), dict(policy=-1)]:
        d = dict(P=2, E=4, K=1, S=2, H=8, R=1, C=0.0, gpus_per_node=1)
        d.update(bad)
        assert oracle.validate(oracle.Config(**d)) == oracle.ERR_INVALID, bad
    assert oracle.validate(oracle.Config(P=2, E=4, K=1, S=2, H=8, R=1, cap_rows=1)) == \
        oracle.ERR_INVALID
    bad_ids = ids.copy()
    bad_ids[1, 1, 0] = 4
    assert oracle.plan(oracle.Config(P=2, E=4, K=1, S=2, H=8, R=1), bad_ids)["status"] == \
        oracle.ERR_BAD_ID
    bad_ids[1, 1, 0] = -1
    assert oracle.plan(oracle.Config(P=2, E=4, K=1, S=2, H=8, R=1), bad_ids)["status"] == \
        oracle.ERR_BAD_ID


def test_metrics_brute_force():
    """R_imb = max/mean rank load and maxvio = max_e T_e / mean_e T_e - 1,
    recounted with plain Python loops from the raw ids."""
    rng = np.random.default_rng(11)
    for _ in range(10):
        P, Eh, K, S = 4, 3, 2, 20
        E = P * Eh
        ids = rng.choice(E, size=(P, S, K), p=np.arange(E, 0, -1) / (E * (E + 1) / 2))
        ids = ids.astype(np.int32)
        cfg = oracle.Config(P=P, E=E, K=K, S=S, H=8, R=1, cap_rows=P * S * K)
        p = oracle.plan(cfg, ids)
        m = oracle.metrics(cfg, p)
        per_e = [0] * E
        for v in ids.ravel().tolist():
            per_e[v] += 1
        per_rank = [sum(per_e[j * Eh:(j + 1) * Eh]) for j in range(P)]
        mean = sum(per_rank) / P
        assert m["r_imb_before"] == pytest.approx(max(per_rank) / mean, rel=1e-12)
        assert m["r_imb_after"] == pytest.approx(max(p["load_after"].tolist()) / mean, rel=1e-12)
        assert m["maxvio"] == pytest.approx(max(per_e) / (sum(per_e) / E) - 1, rel=1e-12)
