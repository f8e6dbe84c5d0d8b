"""zb_place_by_demand (the library's host code, through the C ABI) against
the oracle's placement from historical demand: identical placements on
random shapes up to the largest (P = 32, E = 384, R = 31), every node size,
and demands with ties, zeros and large values.  Host only: no device."""
import numpy as np
import pytest

import oracle
from token_dispatch_top_b200 import build, zb


@pytest.fixture(scope="module", autouse=True)
def lib():
    build.build()
    zb.load()


def _cfgs(seed):
    rng = np.random.default_rng(seed)
    P = int(rng.choice([1, 2, 3, 4, 8, 16, 32]))
    Eh = int(rng.integers(1, min(12, 384 // P) + 1))
    R = int(rng.integers(0, P))
    gpn = int(rng.choice([g for g in (1, 2, 4, 8) if P % g == 0]))
    kind = seed % 4
    E = P * Eh
    if kind == 0:
        D = rng.integers(0, 10 ** 9, E)
    elif kind == 1:
        D = (10 ** 6 / np.arange(1, E + 1) ** rng.uniform(0.3, 2.0)).astype(np.int64)
        D = D[rng.permutation(E)]
    elif kind == 2:
        D = rng.integers(0, 4, E)  # many ties and zeros
    else:
        D = np.zeros(E, np.int64)
        D[rng.integers(0, E)] = 10 ** 12  # one dominant expert
    kw = dict(P=P, E=E, K=1, S=1, H=8, R=R, gpus_per_node=gpn)
    return zb.Config(**kw), oracle.Config(**kw), D.astype(np.int64)


@pytest.mark.parametrize("seed", range(80))
def test_matches_oracle(seed):
    zc, oc, D = _cfgs(seed)
    np.testing.assert_array_equal(zb.place_by_demand(zc, D), oracle.place_by_demand(oc, D))


def test_largest_shape():
    rng = np.random.default_rng(7)
    kw = dict(P=32, E=384, K=1, S=1, H=8, R=31, gpus_per_node=8)
    D = rng.integers(0, 10 ** 6, 384).astype(np.int64)
    np.testing.assert_array_equal(zb.place_by_demand(zb.Config(**kw), D),
                                  oracle.place_by_demand(oracle.Config(**kw), D))


def test_rejects_negative_or_too_large_demand():
    zc = zb.Config(P=2, E=4, K=1, S=1, H=8, R=1)
    oc = oracle.Config(P=2, E=4, K=1, S=1, H=8, R=1)
    for bad in ([1, -1, 0, 0], [0, 0, (1 << 57) + 1, 0]):
        with pytest.raises(zb.ZbError):
            zb.place_by_demand(zc, np.array(bad, np.int64))
        with pytest.raises(ValueError):
            oracle.place_by_demand(oc, np.array(bad, np.int64))
    big = np.array([1 << 57, 1 << 56, 3, 0], np.int64)  # the largest accepted demand
    np.testing.assert_array_equal(zb.place_by_demand(zc, big), oracle.place_by_demand(oc, big))
