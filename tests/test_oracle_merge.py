"""Pins of the oracle's merged dispatch layout (Zepp 4.2, merge: a token's
experts served by the same rank share one copy of its row there)."""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")


def test_hand_example():
    ex = json.load(open(GOLDEN))["merge_examples"][0]
    d = ex["cfg"]
    cfg = oracle.Config(P=d["P"], E=d["E"], K=d["K"], S=d["S"], H=d["H"], R=d["R"])
    ids = np.array(ex["ids"], np.int32)
    p = oracle.plan(cfg, ids)
    assert p["status"] == oracle.OK
    np.testing.assert_array_equal(p["dst_row"], ex["expect"]["dst_row"])
    m = oracle.merge(cfg, p["dst_row"])
    for k in ("tok_row", "grp_tok", "tok_cnt"):
        np.testing.assert_array_equal(m[k], ex["expect"][k], err_msg=k)


def _cases(n=40, seed=31):
    rng = np.random.default_rng(seed)
    for _ in range(n):
        P = int(rng.choice([1, 2, 3, 4, 8]))
        Eh = int(rng.integers(1, 5))
        E = P * Eh
        K = int(rng.integers(1, 7))
        S = int(rng.integers(0, 40))
        R = int(rng.integers(0, P))
        ids = rng.integers(0, E, (P, S, K)).astype(np.int32)
        yield oracle.Config(P=P, E=E, K=K, S=S, H=8, R=R, cap_rows=P * S * K + 1), ids


@pytest.mark.parametrize("case", list(_cases()), ids=lambda c: "case")
def test_merge_properties(case):
    cfg, ids = case
    P, S, K, H, cap = cfg.P, cfg.S, cfg.K, cfg.H, cfg.cap()
    p = oracle.plan(cfg, ids)
    assert p["status"] in (oracle.OK, oracle.UNBALANCED)
    m = oracle.merge(cfg, p["dst_row"])
    dst = p["dst_row"].reshape(P * S, K)
    tok = m["tok_row"].reshape(P * S, K)
    # brute force: distinct tokens per rank, in token order, rows 0..n-1
    for j in range(P):
        toks = [t for t in range(P * S) if np.any(dst[t] // cap == j)]
        assert m["tok_cnt"][j] == len(toks) <= p["load_after"][j]
        for u, t in enumerate(toks):
            assert np.all(tok[t][dst[t] // cap == j] == j * cap + u)
    # each entry's merged row is on its own destination rank
    np.testing.assert_array_equal(tok // cap, dst // cap)
    # grp_tok inverts onto the grouped rows; unused rows -1
    gt = m["grp_tok"].ravel()
    np.testing.assert_array_equal(gt[dst.ravel()], tok.ravel())
    used = np.zeros(P * cap, bool)
    used[dst.ravel()] = True
    assert np.all(gt[~used] == -1)
    # gathering the merged buffer through grp_tok gives the plain dispatch
    rng = np.random.default_rng(0)
    hidden = rng.integers(0, 2 ** 16, (P, S, H), dtype=np.uint32).astype(np.uint16)
    buf = oracle.dispatch(cfg, p["dst_row"], hidden)
    tbuf = oracle.dispatch_merged(cfg, m["tok_row"], hidden)
    flat_b = buf.reshape(P * cap, H)
    flat_t = tbuf.reshape(P * cap, H)
    np.testing.assert_array_equal(flat_t[gt[used]], flat_b[used])
