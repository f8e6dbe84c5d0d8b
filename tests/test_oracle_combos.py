"""Invariants of the plan under every combination of its options: receiver
policy (room / local), eq. (1)'s band (relax), quota repair, and greedy versus
kept placement.  Whatever the combination:

* every route count is routed (sum_j M_ij = d_i), only to holders of the expert,
  and each host's receipt lies within q +- floor(C q) (exactly q without the
  band);
* the quotas of every expert sum to its demand T_e and each rank's quotas to
  its quota load, which repair and the band never change;
* load_after is what each rank receives, cu_seqlens its prefix;
* every (token, k) lands exactly once, below its rank's load, in a group of
  its own expert, and groups are ordered by (source rank, flat index).
"""
import itertools

import numpy as np
import pytest

import oracle

COMBOS = list(itertools.product((0, 1), (0, 1), (0, 1), (False, True)))


def _quotas(cfg, p):
    Eh = cfg.E // cfg.P
    q = np.zeros((cfg.P, cfg.E), np.int64)
    for e in range(cfg.E):
        q[e // Eh, e] = p["home_quota"][e]
    for j in range(cfg.P):
        for s in range(cfg.R):
            e = p["rep_expert"][j, s]
            if e >= 0:
                q[j, e] = p["rep_quota"][j, s]
    return q


def _placement(rng, P, E, R):
    Eh = E // P
    pl = np.full((P, R), -1, np.int32)
    for j in range(P):
        foreign = [e for e in range(E) if e // Eh != j]
        n = int(rng.integers(0, min(R, len(foreign)) + 1))
        pl[j, :n] = rng.choice(foreign, size=n, replace=False)
    return pl


@pytest.mark.parametrize("combo", COMBOS, ids=lambda c: f"pol{c[0]}-relax{c[1]}-rep{c[2]}-"
                                                          f"{'kept' if c[3] else 'greedy'}")
def test_invariants_under_every_combination(combo):
    policy, relax, repair, kept = combo
    rng = np.random.default_rng(hash(combo) % 2 ** 32)
    for trial in range(6):
        P = int(rng.choice([2, 3, 4, 6, 8]))
        gpn = int(rng.choice([g for g in (1, 2, 3) if P % g == 0]))
        Eh, K, S = int(rng.integers(1, 4)), int(rng.integers(1, 5)), int(rng.integers(0, 30))
        R = int(rng.integers(0, P))
        E = P * Eh
        pop = 1.0 / np.arange(1, E + 1) ** rng.uniform(0.5, 2.0)
        ids = rng.choice(E, size=(P, S, K), p=pop / pop.sum()).astype(np.int32)
        C = float(rng.choice([0.1, 0.3, 0.6]))
        cfg = oracle.Config(P=P, E=E, K=K, S=S, H=8, R=R, C=C, gpus_per_node=gpn,
                            cap_rows=P * S * K + 1, policy=policy, relax=relax, repair=repair)
        pl = _placement(rng, P, E, R) if kept else None
        p = oracle.plan(cfg, ids, placement=pl)
        assert p["status"] in (oracle.OK, oracle.UNBALANCED)
        base = oracle.plan(oracle.Config(**{**cfg.__dict__, "relax": 0, "repair": 0}), ids,
                           placement=pl)
        q, q0 = _quotas(cfg, p), _quotas(cfg, base)
        Te = p["cnt"].sum(0)
        np.testing.assert_array_equal(q.sum(0), Te)
        np.testing.assert_array_equal(q.sum(1), q0.sum(1))  # quota loads unchanged
        assert np.all(q >= 0)
        M = p["M"]
        np.testing.assert_array_equal(M.sum(2), p["cnt"].T)
        c20 = np.floor(float(np.float32(C)) * 2.0 ** 20) / 2.0 ** 20 if relax else 0.0
        held = np.zeros((P, E), bool)
        Ehh = E // P
        for e in range(E):
            held[e // Ehh, e] = True
        for j in range(P):
            for s in range(R):
                if p["rep_expert"][j, s] >= 0:
                    held[j, p["rep_expert"][j, s]] = True
        for e in range(E):
            recv = M[e].sum(0)
            assert np.all(M[e][:, ~held[:, e]] == 0)
            dl = np.floor(q[:, e] * c20)
            assert np.all(recv >= q[:, e] - dl) and np.all(recv <= q[:, e] + dl)
        la, cu, cap = p["load_after"], p["cu_seqlens"], cfg.cap()
        for j in range(P):
            assert la[j] == sum(M[e][:, j].sum() for e in range(E))
        np.testing.assert_array_equal(cu[:, -1], la)
        dst = p["dst_row"].ravel()
        valid = np.concatenate([j * cap + np.arange(la[j]) for j in range(P)])
        assert sorted(dst.tolist()) == sorted(valid.tolist())
        rs = p["row_src"].ravel()
        np.testing.assert_array_equal(rs[dst], np.arange(P * S * K))
        for g, row in enumerate(dst):
            j, r = divmod(int(row), cap)
            grp = int(np.searchsorted(cu[j], r, side="right") - 1)
            assert (j * Ehh + grp if grp < Ehh else p["rep_expert"][j, grp - Ehh]) == \
                ids.ravel()[g]
        for j in range(P):
            src = rs[j * cap:j * cap + la[j]]
            for grp in range(Ehh + R):
                assert np.all(np.diff(src[cu[j, grp]:cu[j, grp + 1]]) > 0)
