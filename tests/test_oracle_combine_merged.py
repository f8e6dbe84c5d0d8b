"""Pins of the merged combine (Zepp 4.2 Merge: node-local pre-reduction).

Destination side: part[r] = bf16(fold of fmaf(w_k, y_k, acc) over the token's
k served by merged row r, k ascending, acc from +0.0f).  Source side:
out = bf16(acc + part[r] over the token's merged rows in order of first k,
acc from +0.0f).  The pins:
* when all of a token's experts sit on one rank, the single partial is the
  plain combine's fold, so out equals the plain combine bit for bit;
* when they sit on K different ranks, each partial is bf16(w*y) and out is a
  plain float32 sum of those, both recomputed here with torch CPU ops;
* in general, every partial equals the exact rational fold rounded to binary32
  at each step, then to bf16 (torch), and out is torch's float32 sum of them;
* on N(0,1) data, out lies within the rounding bound of the float64 sum.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from test_oracle_combine import _rn32


def _bf16_bits(x32) -> np.ndarray:
    return torch.from_numpy(np.asarray(x32, np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def _f32_of_bits(b) -> np.ndarray:
    return (np.asarray(b, np.uint32) << 16).view(np.float32)


def _plan(P, Eh, K, S, H, R, ids, seed):
    cfg = oracle.Config(P=P, E=P * Eh, K=K, S=S, H=H, R=R, cap_rows=P * S * K)
    p = oracle.plan(cfg, ids, want_M=False)
    assert p["status"] >= 0
    m = oracle.merge(cfg, p["dst_row"])
    rng = np.random.default_rng(seed)
    y = _bf16_bits(rng.standard_normal((P * cfg.cap(), H)).astype(np.float32))
    w = rng.dirichlet(np.ones(K), size=(P, S)).astype(np.float32)
    return cfg, p, m, y, w


def _merged(cfg, p, m, y, w):
    part = oracle.combine_reduce(cfg, p["dst_row"], m["tok_row"], y, w)
    return part, oracle.combine_merged(cfg, m["tok_row"], part)


@pytest.mark.parametrize("seed", range(4))
def test_fully_merged_equals_plain_combine(seed):
    rng = np.random.default_rng(seed)
    P, Eh, K, S, H = 4, 3, int(rng.integers(1, 9)), 33, 24
    # every token picks experts homed on its own rank; no slots
    ids = np.stack([rng.integers(i * Eh, (i + 1) * Eh, size=(S, K)) for i in range(P)]) \
        .astype(np.int32)
    cfg, p, m, y, w = _plan(P, Eh, K, S, H, 0, ids, seed)
    np.testing.assert_array_equal(m["tok_cnt"], [S] * P)
    _, out = _merged(cfg, p, m, y, w)
    np.testing.assert_array_equal(out, oracle.combine(cfg, p["dst_row"], y, w))


@pytest.mark.parametrize("seed", range(4))
def test_unmerged_is_rounded_products_summed(seed):
    rng = np.random.default_rng(10 + seed)
    K = int(rng.integers(1, 7))
    P, Eh, S, H = K, 2, 20, 16
    # the k-th expert of every token is homed on rank k: K distinct ranks
    ids = np.stack([np.stack([rng.integers(k * Eh, (k + 1) * Eh, size=S) for k in range(K)], 1)
                    for _ in range(P)]).astype(np.int32)
    cfg, p, m, y, w = _plan(P, Eh, K, S, H, 0, ids, seed)
    part, out = _merged(cfg, p, m, y, w)
    dst, tok = p["dst_row"].reshape(-1, K), m["tok_row"].reshape(-1, K)
    yf = torch.from_numpy(_f32_of_bits(y))
    wf = torch.from_numpy(w.reshape(-1, K))
    acc = torch.zeros((P * S, H), dtype=torch.float32)
    for k in range(K):
        pk = wf[:, k:k + 1] * yf[torch.from_numpy(dst[:, k].astype(np.int64))] + 0.0
        pk_bits = pk.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        np.testing.assert_array_equal(part.reshape(-1, H)[tok[:, k]], pk_bits)
        acc = acc + pk.to(torch.bfloat16).float()
    np.testing.assert_array_equal(out.reshape(-1, H),
                                  acc.to(torch.bfloat16).view(torch.int16).numpy()
                                  .view(np.uint16))


def test_general_matches_exact_fold():
    rng = np.random.default_rng(42)
    P, Eh, K, S, H, R = 4, 2, 5, 12, 8, 2
    pop = 1.0 / np.arange(1, P * Eh + 1) ** 1.2
    ids = rng.choice(P * Eh, size=(P, S, K), p=pop / pop.sum()).astype(np.int32)
    cfg, p, m, y, w = _plan(P, Eh, K, S, H, R, ids, 5)
    part, out = _merged(cfg, p, m, y, w)
    dst, tok = p["dst_row"].reshape(-1, K), m["tok_row"].reshape(-1, K)
    wk = w.reshape(-1, K)
    yf = _f32_of_bits(y)
    merged_rows = 0
    for t in range(P * S):
        acc_out = torch.zeros(H, dtype=torch.float32)
        seen = []
        for k0 in range(K):
            r = tok[t, k0]
            if r in seen:
                continue
            seen.append(r)
            ks = [k for k in range(k0, K) if tok[t, k] == r]
            merged_rows += len(ks) > 1
            acc = [np.float32(0.0)] * H
            for k in ks:
                acc = [_rn32(Fraction(float(wk[t, k])) * Fraction(float(yf[dst[t, k], h])) +
                             Fraction(float(acc[h]))) for h in range(H)]
            want = _bf16_bits(np.array(acc, np.float32))
            np.testing.assert_array_equal(part.reshape(-1, H)[r], want)
            acc_out = acc_out + torch.from_numpy(_f32_of_bits(want))
        np.testing.assert_array_equal(out.reshape(-1, H)[t], _bf16_bits(acc_out.numpy()))
    assert merged_rows > 20  # the case exercises real merging


def test_within_float64_bound():
    rng = np.random.default_rng(3)
    P, Eh, K, S, H, R = 8, 4, 6, 64, 64, 2
    ids = rng.integers(0, P * Eh, size=(P, S, K)).astype(np.int32)
    cfg, p, m, y, w = _plan(P, Eh, K, S, H, R, ids, 3)
    _, out = _merged(cfg, p, m, y, w)
    dst = p["dst_row"].reshape(-1, K)
    yf = _f32_of_bits(y).astype(np.float64)
    exact = np.einsum("tk,tkh->th", w.reshape(-1, K).astype(np.float64), yf[dst])
    absum = np.einsum("tk,tkh->th", np.abs(w.reshape(-1, K)).astype(np.float64),
                      np.abs(yf[dst]))
    # one bf16 rounding per partial and one at the end, fp32 terms negligible
    bound = 2.0 ** -8 * (np.abs(exact) + absum) + 1e-30
    got = _f32_of_bits(out.reshape(-1, H)).astype(np.float64)
    assert np.all(np.abs(got - exact) <= bound)
