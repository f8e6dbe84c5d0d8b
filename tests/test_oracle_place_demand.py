"""Pins of the placement from historical demand (Zepp 4.1: R extra slots per
GPU go greedily to the experts with the highest demand per replica, spread
round-robin across nodes first, then across a node's GPUs).

* A hand-worked case (P = 4, nodes of 2, R = 1).
* Where no pick was blocked (no expert ever failed to fit), the copy counts
  are those of a divisor method: picking the largest D/n one copy at a time
  leaves every expert a with an extra copy at least as deserving as any other
  expert b, D_a / (n_a - 1) >= D_b / n_b (exact integer cross-multiplication).
* Node coverage: an expert with n copies sits on min(n, nodes) nodes unless
  every node it misses was full; every placement is valid.
"""
import itertools

import numpy as np
import pytest

import oracle


def test_hand_example():
    # E = 8 (two per rank), D = [100,10,10,10,60,10,10,10], nodes {0,1},{2,3}.
    # Picks: e0 (100/1) -> node 1 (node 0 holds e0 at home), rank 2;
    # e4 (60/1 > 100/2) -> node 0 (cursor), rank 0; e0 (50 > 30) -> both
    # nodes hold e0, cursor node 1 from its GPU cursor 1: rank 3; e0 (33.3 >
    # 30) -> node 0 from its GPU cursor 1: rank 1.
    cfg = oracle.Config(P=4, E=8, K=1, S=1, H=8, R=1, gpus_per_node=2)
    pl = oracle.place_by_demand(cfg, np.array([100, 10, 10, 10, 60, 10, 10, 10]))
    np.testing.assert_array_equal(pl, [[4], [0], [0], [0]])


def _copies(cfg, pl):
    n = np.ones(cfg.E, np.int64)
    for e in pl.ravel():
        if e >= 0:
            n[e] += 1
    return n


def test_divisor_method_counts():
    clean = 0
    for seed in range(60):
        rng = np.random.default_rng(seed)
        P = int(rng.choice([2, 4, 8]))
        Eh = int(rng.integers(2, 6))
        R = int(rng.integers(1, min(3, P)))
        gpn = int(rng.choice([g for g in (1, 2, 4) if P % g == 0]))
        cfg = oracle.Config(P=P, E=P * Eh, K=1, S=1, H=8, R=R, gpus_per_node=gpn)
        D = (1000 / np.arange(1, cfg.E + 1) ** rng.uniform(0.3, 1.5)).astype(np.int64)
        D = D[rng.permutation(cfg.E)]
        pl, blocked = oracle.place_by_demand(cfg, D, with_blocked=True)
        n = _copies(cfg, pl)
        # every slot is filled: with R <= 2 and Eh >= 2 some expert always fits
        assert (pl >= 0).all()
        if blocked:
            continue
        clean += 1
        for a, b in itertools.permutations(range(cfg.E), 2):
            if n[a] >= 2:
                assert D[a] * n[b] >= D[b] * (n[a] - 1), (a, b, D[a], D[b], n[a], n[b])
    assert clean >= 20


@pytest.mark.parametrize("seed", range(20))
def test_valid_and_node_coverage(seed):
    rng = np.random.default_rng(100 + seed)
    P, gpn = 8, int(rng.choice([2, 4]))
    cfg = oracle.Config(P=P, E=P * 2, K=1, S=1, H=8, R=int(rng.integers(1, 4)),
                        gpus_per_node=gpn)
    D = rng.integers(0, 10 ** 6, cfg.E).astype(np.int64)
    pl = oracle.place_by_demand(cfg, D)
    assert oracle.validate(cfg) == 0
    for j in range(P):  # valid: never on the home rank, never twice on a rank
        held = [e for e in pl[j] if e >= 0]
        assert len(set(held)) == len(held) and all(e // 2 != j for e in held)
    nodes = P // gpn
    n = _copies(cfg, pl)
    for e in range(cfg.E):
        ranks = {e // 2} | {j for j in range(P) if e in pl[j]}
        covered = {r // gpn for r in ranks}
        if len(covered) < min(n[e], nodes):
            # a copy went to a covered node only when every uncovered node was
            # full; slots only fill up, so those nodes are full at the end
            for nd in set(range(nodes)) - covered:
                assert (pl[nd * gpn:(nd + 1) * gpn] >= 0).all(), (e, nd)


def test_zero_demand_and_errors():
    cfg = oracle.Config(P=4, E=8, K=1, S=1, H=8, R=2)
    pl = oracle.place_by_demand(cfg, np.zeros(8, np.int64))
    assert (pl >= 0).all()  # ties to the lowest expert still fill the slots
    with pytest.raises(ValueError):
        oracle.place_by_demand(cfg, np.array([1, -1, 0, 0, 0, 0, 0, 0]))
