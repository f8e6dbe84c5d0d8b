"""Pins of the oracle's dispatch (step 4) and combine (step 5).

The combine is fixed as: acc = +0.0f; acc = fmaf(w_k, y_k, acc) for k = 0..K-1
(one rounding per term, binary32), then bf16 round-to-nearest-even.  The pins:
* bf16 rounding against torch's CPU float32 -> bfloat16 conversion (a library
  routine) on random values and on the edge cases (ties, carries into the
  exponent, subnormals, overflow to infinity, NaN);
* the fold against exact rational arithmetic (fractions.Fraction) rounded to
  binary32 by nearest-even, on inputs chosen so that a separate multiply and
  add, or another summation order, would give a different answer;
* K = 1, w = 1 returns the expert row unchanged;
* on N(0,1) data, the result is within the rounding bound of the float64 sum;
* dispatch copies rows bit for bit and leaves unused rows untouched.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle


def _torch_bf16_bits(x32: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x32.astype(np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def _bits_f32(u: int) -> float:
    return float(np.array([u], np.uint32).view(np.float32)[0])


def test_bf16_rounding_matches_library():
    rng = np.random.default_rng(0)
    u = rng.integers(0, 2 ** 32, size=20000, dtype=np.uint64).astype(np.uint32)
    specials = [0x00000000, 0x80000000, 0x3F808000, 0x3F818000, 0x3F80FFFF, 0x3F7FFFFF,
                0x7F7FFFFF, 0x7F7F8000, 0x7F7F7FFF, 0xFF7FFFFF, 0x00000001, 0x00008000,
                0x00018000, 0x007FFFFF, 0x807FFFFF, 0x7F800000, 0xFF800000, 0x00800000]
    u = np.concatenate([u, np.array(specials, np.uint32)])
    x = u.view(np.float32)
    exp = _torch_bf16_bits(x)
    got = np.array([oracle.f32_to_bf16(float(v)) for v in x], np.uint16)
    nan = np.isnan(x)
    np.testing.assert_array_equal(got[~nan], exp[~nan])
    # NaN stays NaN
    g_nan = got[nan]
    assert np.all(((g_nan & 0x7F80) == 0x7F80) & ((g_nan & 0x007F) != 0))
    # widening is exact
    for b in [0x0000, 0x8000, 0x3F80, 0x0001, 0x7F7F, 0xFF80, 0x4049]:
        assert np.float32(oracle.bf16_to_f32(b)).view(np.uint32) == b << 16


def _rn32(q: Fraction) -> np.float32:
    """Round an exact rational to binary32, nearest, ties to even."""
    c = np.float32(float(q))
    cands = [np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))]
    best = None
    for v in cands:
        if not np.isfinite(v):
            continue
        d = abs(Fraction(float(v)) - q)
        key = (d, int(np.array([v], np.float32).view(np.uint32)[0]) & 1)
        if best is None or key < best[0]:
            best = (key, v)
    return best[1]


def _bf16_of(x: np.float32) -> int:
    return int(_torch_bf16_bits(np.array([x], np.float32))[0])


def _model(w, y_bits):
    acc = np.float32(0.0)
    for wk, yk in zip(w, y_bits):
        yv = np.float32(oracle.bf16_to_f32(int(yk)))
        acc = _rn32(Fraction(float(np.float32(wk))) * Fraction(float(yv)) + Fraction(float(acc)))
    return _bf16_of(acc)


def _unfused(w, y_bits, order):
    acc = np.float32(0.0)
    for k in order:
        prod = np.float32(np.float32(w[k]) * np.float32(oracle.bf16_to_f32(int(y_bits[k]))))
        acc = np.float32(acc + prod)
    return _bf16_of(acc)


def _combine_one(w, y_bits):
    K = len(w)
    H = 8
    cfg = oracle.Config(P=1, E=1, K=K, S=1, H=H, R=0, cap_rows=K)
    y = np.zeros((K, H), np.uint16)
    y[:, 0] = y_bits
    out = oracle.combine(cfg, np.arange(K, dtype=np.int32).reshape(1, 1, K), y,
                         np.asarray(w, np.float32).reshape(1, 1, K))
    return int(out[0, 0, 0])


def test_fold_matches_exact_rounding():
    rng = np.random.default_rng(5)
    for trial in range(3000):
        K = int(rng.integers(1, 5))
        # mixed magnitudes make the rounding of each step visible
        w = rng.standard_normal(K).astype(np.float32) * np.float32(10.0) ** rng.integers(-3, 4, K)
        y = _torch_bf16_bits(rng.standard_normal(K).astype(np.float32) *
                             np.float32(10.0) ** rng.integers(-3, 4, K))
        assert _combine_one(w, y) == _model(w, y), (w.tolist(), y.tolist())


def _f32(x):
    return np.float32(x)


def test_fold_is_fused():
    """A case where one rounding per term and a rounded product then a rounded
    add land on different sides of a bf16 tie.  Term 0 is 1 + 2^-8 (a bf16
    tie); term 1 is a product just above 2^-24 (half a binary32 ulp at 1), so
    the fused sum rounds up past the tie while the rounded product lands
    exactly on the binary32 tie and rounds to even (back onto the bf16 tie)."""
    y1 = 0x3C01  # bf16 1.0078125 * 2^-7
    m_y = Fraction(oracle.bf16_to_f32(y1))
    target = Fraction(1, 2 ** 24)
    w1 = np.float32(float(target / m_y))
    while Fraction(float(w1)) * m_y <= target:
        w1 = np.nextafter(w1, np.float32(np.inf))
    p = Fraction(float(w1)) * m_y
    assert target < p < target * (1 + Fraction(1, 2 ** 24))
    w = [_f32(1 + 2.0 ** -8), w1]
    y = [0x3F80, y1]
    fused = _model(w, y)
    assert fused == 0x3F81 and _unfused(w, y, [0, 1]) == 0x3F80
    assert _combine_one(w, y) == fused


def test_fold_order_is_k_ascending():
    """1 + 2^-8, then two terms of 2^-24: each add is a binary32 tie that
    rounds to even, leaving the bf16 tie (rounds down).  In reverse order the
    two small terms add exactly first and push the sum past the tie."""
    w = [_f32(1 + 2.0 ** -8), _f32(2.0 ** -24), _f32(2.0 ** -24)]
    y = [0x3F80, 0x3F80, 0x3F80]
    assert _model(w, y) == 0x3F80 and _model(w[::-1], y[::-1]) == 0x3F81
    assert _combine_one(w, y) == 0x3F80


def test_identity_expert_k1():
    rng = np.random.default_rng(1)
    P, S, H = 2, 5, 64
    y = _torch_bf16_bits(rng.standard_normal((P * S, H)).astype(np.float32))
    y[0, :4] = [0x0001, 0x8001, 0x7F7F, 0x8000]  # subnormal, -subnormal, max, -0
    cfg = oracle.Config(P=P, E=P, K=1, S=S, H=H, R=0, cap_rows=S)
    dst = np.arange(P * S, dtype=np.int32).reshape(P, S, 1)
    out = oracle.combine(cfg, dst, y, np.ones((P, S, 1), np.float32))
    exp = y.reshape(P, S, H).copy()
    exp[0, 0, 3] = 0x0000  # (+0.0) + 1 * (-0.0) = +0.0 under round-to-nearest
    np.testing.assert_array_equal(out, exp)


def test_combine_within_float64_bound():
    rng = np.random.default_rng(2)
    P, S, K, H = 2, 16, 6, 128
    rows = P * S * K
    y = _torch_bf16_bits(rng.standard_normal((rows, H)).astype(np.float32))
    w = rng.dirichlet(np.ones(K), size=(P, S)).astype(np.float32)
    dst = rng.permutation(rows).astype(np.int32).reshape(P, S, K)
    cfg = oracle.Config(P=P, E=P, K=K, S=S, H=H, R=0, cap_rows=S * K)
    out = oracle.combine(cfg, dst, y, w)
    yf = torch.from_numpy(y.view(np.int16)).view(torch.bfloat16).float().double().numpy()
    exact = np.einsum("psk,pskh->psh", w.astype(np.float64), yf[dst])
    absum = np.einsum("psk,pskh->psh", np.abs(w.astype(np.float64)), np.abs(yf[dst]))
    got = torch.from_numpy(out.view(np.int16)).view(torch.bfloat16).double().numpy()
    # bf16 rounding (half an ulp, 2^-9 relative) plus K binary32 roundings
    bound = np.abs(exact) * 2.0 ** -8 + absum * K * 2.0 ** -23 + 1e-40
    assert np.all(np.abs(got - exact) <= bound)


def test_dispatch_copies_rows_bit_for_bit():
    rng = np.random.default_rng(4)
    P, E, K, S, H, R = 4, 8, 2, 10, 16, 1
    ids = rng.integers(0, E, (P, S, K)).astype(np.int32)
    cfg = oracle.Config(P=P, E=E, K=K, S=S, H=H, R=R, cap_rows=P * S * K)
    p = oracle.plan(cfg, ids)
    hidden = rng.integers(0, 2 ** 16, (P, S, H), dtype=np.uint32).astype(np.uint16)
    sentinel = np.full((P, cfg.cap(), H), 0xABCD, np.uint16)
    buf = oracle.dispatch(cfg, p["dst_row"], hidden, sentinel.copy())
    flat = buf.reshape(P * cfg.cap(), H)
    touched = np.zeros(P * cfg.cap(), bool)
    for i in range(P):
        for s in range(S):
            for k in range(K):
                r = p["dst_row"][i, s, k]
                assert np.array_equal(flat[r], hidden[i, s])
                touched[r] = True
    assert np.all(flat[~touched] == 0xABCD)
    # y = buf with one-hot weights returns each token's row
    w = np.zeros((P, S, K), np.float32)
    w[:, :, 0] = 1.0
    out = oracle.combine(cfg, p["dst_row"], flat, w)
    finite = np.isfinite(torch.from_numpy(hidden.view(np.int16)).view(torch.bfloat16).float()
                         .numpy())
    nz = (hidden & 0x7FFF) != 0
    same = (out == hidden) | ~finite | ~nz
    assert np.all(same)
