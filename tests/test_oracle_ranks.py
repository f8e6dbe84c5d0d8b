"""Pins of the oracle's per-rank form of the path: the form one of P real ranks
runs when it holds only its own ids and rows.

ISER-MoE (Methodology / HALO-Q Scheduler, stage 1) has the ranks exchange
their route counts and then plan; MoonEP ("What MoonEP enforces and how") has
each rank write its rows straight into the fixed-shape, expert-grouped
buffers of the other ranks.  The oracle states that form as four functions:
``count`` (a rank's counts, plus its ids outside [0, E)), ``plan_rank`` (the
plan from every rank's counts and the rank's own ids), ``dispatch_ranks`` and
``combine_ranks`` (rows moved through one buffer per destination rank).

Pins, none of which is the function re-typed:
* the hand-worked examples: every rank's tables and its row of dst_row;
* ``count`` against numpy's bincount;
* ``plan_rank`` of every rank against the whole-batch plan, under every
  policy, band, repair and kept placement;
* exchanged counts that do not match a rank's ids, or rows that do not sum
  to S*K, are refused; an id out of range on any rank fails every rank;
* ``dispatch_ranks`` against a numpy scatter of the rows dst_row names, and
  against the whole-batch dispatch split by rank;
* ``combine_ranks`` against the fold computed in exact rationals, and
  against the whole-batch combine.
"""
import json
import os

import numpy as np
import pytest

import oracle
from test_oracle_combine import _model, _torch_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")
EXAMPLES = json.load(open(GOLDEN))["examples"]
TABLES = ("cnt", "rep_expert", "rep_quota", "home_quota", "load_before", "load_after",
          "cu_seqlens")
SENTINEL = 0x7E11


def _cfg(d, **over):
    kw = dict(P=d["P"], E=d["E"], K=d["K"], S=d["S"], H=d["H"], R=d["R"], C=d.get("C", 0.0),
              gpus_per_node=d.get("gpus_per_node", 1), cap_rows=d.get("cap_rows"),
              policy=d.get("policy", 0), relax=d.get("relax", 0), repair=d.get("repair", 0))
    kw.update(over)
    return oracle.Config(**kw)


def _exchange(cfg, ids):
    return np.stack([oracle.count(cfg, ids[r]) for r in range(cfg.P)])


@pytest.mark.parametrize("ex", EXAMPLES, ids=lambda e: e["name"])
def test_hand_examples_on_every_rank(ex):
    cfg = _cfg(ex["cfg"])
    ids = np.array(ex["ids"], np.int32).reshape(cfg.P, cfg.S, cfg.K)
    pl = np.array(ex["placement"], np.int32) if "placement" in ex else None
    want = ex["expect"]
    counts = _exchange(cfg, ids)
    for r in range(cfg.P):
        p = oracle.plan_rank(cfg, r, counts, ids[r], placement=pl)
        assert p["status"] == want["status"], (r, p["status"])
        assert p["T"] == want["T"]
        for k in TABLES:
            if k in want:
                np.testing.assert_array_equal(p[k], np.array(want[k]), err_msg=f"{k} rank {r}")
        assert p["locality_cost"] == want["locality_cost"]
        if "dst_row" in want:
            np.testing.assert_array_equal(p["dst_row"].ravel(), np.array(want["dst_row"][r]),
                                          err_msg=f"dst_row rank {r}")
        if "status_with_cap_rows_3" in want:
            c3 = _cfg(ex["cfg"], cap_rows=3)
            q = oracle.plan_rank(c3, r, counts, ids[r], placement=pl)
            assert q["status"] == want["status_with_cap_rows_3"]
            assert (q["dst_row"] == -1).all()


def test_count_is_bincount():
    rng = np.random.default_rng(0)
    cfg = oracle.Config(P=3, E=12, K=4, S=200, H=8, R=1)
    for _ in range(5):
        ids = rng.integers(-3, 15, (cfg.S, cfg.K)).astype(np.int32)
        row = oracle.count(cfg, ids)
        ok = (ids >= 0) & (ids < cfg.E)
        np.testing.assert_array_equal(row[:cfg.E], np.bincount(ids[ok], minlength=cfg.E))
        assert row[cfg.E] == int((~ok).sum())


def _random_case(rng, P, gpn, policy, relax, repair, placed):
    Eh = int(rng.integers(1, 6))
    E, K, S = P * Eh, int(rng.integers(1, 5)), int(rng.integers(0, 60))
    R = int(rng.integers(0, P))
    pop = 1.0 / np.arange(1, E + 1) ** rng.uniform(0.5, 2.0)
    ids = rng.choice(E, size=(P, S, K), p=pop[rng.permutation(E)] / pop.sum()).astype(np.int32)
    cfg = oracle.Config(P=P, E=E, K=K, S=S, H=8, R=R, C=0.3, gpus_per_node=gpn,
                        cap_rows=max(1, P * S * K), policy=policy, relax=relax, repair=repair)
    pl = None
    if placed and R > 0:
        pl = np.full((P, R), -1, np.int32)
        for j in range(P):
            foreign = [e for e in rng.permutation(E) if e // Eh != j]
            n = int(rng.integers(0, min(R, len(foreign)) + 1))
            pl[j, :n] = foreign[:n]
    return cfg, ids, pl


@pytest.mark.parametrize("k", range(48))
def test_every_rank_reproduces_the_whole_plan(k):
    rng = np.random.default_rng(500 + k)
    P = int(rng.choice([1, 2, 3, 4, 6, 8]))
    gpn = int(rng.choice([g for g in (1, 2, 4) if P % g == 0]))
    cfg, ids, pl = _random_case(rng, P, gpn, policy=k % 2, relax=(k // 2) % 2,
                                repair=(k // 4) % 2, placed=(k // 8) % 2)
    ref = oracle.plan(cfg, ids, want_M=False, placement=pl)
    counts = _exchange(cfg, ids)
    for r in range(P):
        p = oracle.plan_rank(cfg, r, counts, ids[r], placement=pl)
        assert p["status"] == ref["status"]
        for key in TABLES:
            np.testing.assert_array_equal(p[key], ref[key], err_msg=key)
        for key in ("locality_cost", "max_load", "n_replicas", "n_iters", "T", "repaired"):
            assert p[key] == ref[key], key
        np.testing.assert_array_equal(p["dst_row"], ref["dst_row"][r])


def test_counts_that_do_not_match_are_refused():
    rng = np.random.default_rng(3)
    cfg = oracle.Config(P=4, E=8, K=2, S=30, H=8, R=1, cap_rows=4 * 60)
    ids = rng.integers(0, 8, (4, 30, 2)).astype(np.int32)
    counts = _exchange(cfg, ids)
    assert oracle.plan_rank(cfg, 1, counts, ids[1])["status"] >= 0
    bad = counts.copy()
    bad[1, 0] += 1
    bad[1, 1] -= 1   # the same total, other counts than rank 1's ids
    assert oracle.plan_rank(cfg, 1, bad, ids[1])["status"] == oracle.ERR_INVALID
    short = counts.copy()
    short[2, 3] -= 1  # rank 2's row no longer sums to S*K
    assert oracle.plan_rank(cfg, 1, short, ids[1])["status"] == oracle.ERR_INVALID
    assert oracle.plan_rank(cfg, 4, counts, ids[1])["status"] == oracle.ERR_INVALID
    ids2 = ids.copy()
    ids2[2, 5, 1] = 8  # out of range on rank 2 only
    counts2 = _exchange(cfg, ids2)
    for r in range(4):
        assert oracle.plan_rank(cfg, r, counts2, ids2[r])["status"] == oracle.ERR_BAD_ID


def _bits(rng, shape):
    return rng.integers(0, 0x7F00, shape).astype(np.uint16)


@pytest.mark.parametrize("seed", range(6))
def test_dispatch_ranks_writes_the_named_rows(seed):
    rng = np.random.default_rng(40 + seed)
    cfg, ids, _ = _random_case(rng, 4, 2, policy=seed % 2, relax=0, repair=0, placed=False)
    cfg = oracle.Config(**{**cfg.__dict__, "H": 16})
    cap = cfg.cap()
    ref = oracle.plan(cfg, ids, want_M=False)
    hidden = _bits(rng, (cfg.P, cfg.S, cfg.H))
    whole = np.full((cfg.P, cap, cfg.H), SENTINEL, np.uint16)
    oracle.dispatch(cfg, ref["dst_row"], hidden, whole)
    bufs = [np.full((cap, cfg.H), SENTINEL, np.uint16) for _ in range(cfg.P)]
    for r in range(cfg.P):
        oracle.dispatch_ranks(cfg, ref["dst_row"][r], hidden[r], bufs)
    # numpy scatter of the definition: bufs[d // cap][d % cap] = hidden[r, s]
    want = [np.full((cap, cfg.H), SENTINEL, np.uint16) for _ in range(cfg.P)]
    for r in range(cfg.P):
        d = ref["dst_row"][r].reshape(-1)
        s = np.repeat(np.arange(cfg.S), cfg.K)
        for j in range(cfg.P):
            sel = (d // cap) == j
            want[j][d[sel] % cap] = hidden[r, s[sel]]
    for j in range(cfg.P):
        np.testing.assert_array_equal(bufs[j], want[j])
        np.testing.assert_array_equal(bufs[j], whole[j])


@pytest.mark.parametrize("seed", range(4))
def test_combine_ranks_is_the_fold(seed):
    rng = np.random.default_rng(70 + seed)
    cfg, ids, _ = _random_case(rng, 4, 1, policy=0, relax=0, repair=0, placed=False)
    cfg = oracle.Config(**{**cfg.__dict__, "H": 8, "S": max(cfg.S, 3)})
    ids = rng.integers(0, cfg.E, (cfg.P, cfg.S, cfg.K)).astype(np.int32)
    cap = cfg.cap()
    ref = oracle.plan(cfg, ids, want_M=False)
    ys = [_torch_bf16_bits(rng.standard_normal((cap, cfg.H))) for _ in range(cfg.P)]
    w = rng.dirichlet(np.ones(cfg.K), size=(cfg.P, cfg.S)).astype(np.float32)
    whole = oracle.combine(cfg, ref["dst_row"], np.concatenate(ys), w)
    for r in range(cfg.P):
        got = oracle.combine_ranks(cfg, ref["dst_row"][r], ys, w[r])
        np.testing.assert_array_equal(got, whole[r])
        for s in range(min(cfg.S, 3)):  # the exact-rational fold on a few tokens
            d = ref["dst_row"][r, s]
            for h in (0, cfg.H - 1):
                yk = [ys[x // cap][x % cap, h] for x in d]
                assert got[s, h] == _model(w[r, s], yk)


def test_combine_ranks_k1_returns_rows():
    rng = np.random.default_rng(9)
    cfg = oracle.Config(P=3, E=6, K=1, S=20, H=16, R=1, cap_rows=60)
    ids = rng.integers(0, 6, (3, 20, 1)).astype(np.int32)
    ref = oracle.plan(cfg, ids, want_M=False)
    ys = [_bits(rng, (60, 16)) for _ in range(3)]
    for r in range(3):
        got = oracle.combine_ranks(cfg, ref["dst_row"][r], ys, np.ones((20, 1), np.float32))
        d = ref["dst_row"][r, :, 0]
        np.testing.assert_array_equal(got, np.stack([ys[x // 60][x % 60] for x in d]))
