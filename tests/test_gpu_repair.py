"""GPU parity of quota repair (ISER-MoE, HALO-Q stage 4, repair = 1) against
the oracle: plan tables and rows bit-exact on the every-pair construction,
random kept placements, hot-everywhere placements of the named workloads at
full size (with sampled dispatch and combine), the greedy's own placements,
and repair combined with eq. (1)'s band."""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_plan_equal, cfgs, plan_tables
from test_gpu_parity import SMALL, _rand_bits, full_parity, sampled_data_parity
from test_oracle_repair import CASES, _random_placed
from token_dispatch_top_b200 import build, synth, zb

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev(cuda_device):
    build.build()
    zb.load()
    return cuda_device


def _placed(zc, oc, ids, pl, dev, with_row_src=True):
    p = zb.Plan(zc, dev, with_row_src=with_row_src)
    zb.plan_placed(p, torch.from_numpy(np.ascontiguousarray(ids)).to(dev),
                   torch.from_numpy(np.ascontiguousarray(pl, np.int32)).to(dev))
    status, _ = zb.plan_status(p)
    o = oracle.plan(oc, ids, placement=pl, want_M=False)
    assert_plan_equal(plan_tables(p), o, status)
    return p, o, status


@pytest.mark.parametrize("P", [2, 3, 4, 7, 8, 9, 16])
def test_every_pair_is_visited_once(dev, P):
    Eh = P - 1

    def ex(i, j):
        return i * Eh + (j if j < i else j - 1)
    pl = np.full((P, P - 1), -1, np.int32)
    ids = []
    for i in range(P):
        others = [j for j in range(P) if j != i]
        pl[i] = [ex(j, i) for j in others]
        ids.append(sum(([ex(i, j)] * 3 + [ex(j, i)] for j in others), []))
    ids = np.array(ids, np.int32)[:, :, None]
    kw = dict(P=P, E=P * Eh, K=1, S=ids.shape[1], H=8, R=P - 1, repair=1)
    p, o, status = _placed(zb.Config(**kw), oracle.Config(**kw), ids, pl, dev)
    assert status == oracle.OK and o["repaired"] == P * (P - 1) // 2
    assert int(p.stats[zb.STAT_LOCALITY_COST]) == 0


@pytest.mark.parametrize("k", range(0, len(CASES), 2))
def test_random_placed(dev, k):
    P, R, E, ids, pl = CASES[k]
    S, K = ids.shape[1], ids.shape[2]
    gpn = 2 if P % 2 == 0 and k % 3 == 0 else 1
    kw = dict(P=P, E=E, K=K, S=S, H=8, R=R, gpus_per_node=gpn, cap_rows=P * S * K + 1,
              repair=1, relax=k % 4 == 2, C=0.25)
    _placed(zb.Config(**kw), oracle.Config(**kw), ids, pl, dev)


@pytest.mark.parametrize("k", range(3, len(SMALL), 4))
def test_greedy_then_repair_small(dev, k):
    kw, ids = SMALL[k]
    rng = np.random.default_rng(5000 + k)
    kw = dict(kw, repair=1, cap_rows=max(1, kw["P"] * kw["S"] * kw["K"]))
    zc, oc = zb.Config(**kw), oracle.Config(**kw)
    w = rng.dirichlet(np.ones(zc.K), size=(zc.P, zc.S)).astype(np.float32)
    full_parity(zc, oc, ids, w, _rand_bits(rng, (zc.P, zc.S, zc.H)),
                _rand_bits(rng, (zc.P * zc.cap, zc.H)), dev)


def _hot_everywhere(ids, E, P, R):
    """Every rank holds copies of the R hottest experts homed elsewhere."""
    Te = np.bincount(ids.ravel(), minlength=E)
    Eh = E // P
    pl = np.full((P, R), -1, np.int32)
    for j in range(P):
        order = [e for e in np.argsort(-Te, kind="stable") if e // Eh != j][:R]
        pl[j, :len(order)] = order
    return pl


@pytest.mark.parametrize("name,R,relax", [("mid", 4, 0), ("mid", 7, 0), ("mid", 7, 1),
                                          ("hot", 7, 0), ("hier", 8, 0)])
def test_hot_everywhere_full_size(dev, name, R, relax):
    wl = synth.WORKLOADS[name]
    ids, w = synth.routing(wl, 0)
    kw = dict(P=wl.P, E=wl.E, K=wl.K, S=wl.S, H=wl.H, R=R, C=0.1,
              gpus_per_node=wl.gpus_per_node, cap_rows=2 * wl.S * wl.K, repair=1, relax=relax)
    zc, oc = zb.Config(**kw), oracle.Config(**kw)
    pl = _hot_everywhere(ids, wl.E, wl.P, R)
    p, o, status = _placed(zc, oc, ids, pl, dev, with_row_src=False)
    assert o["repaired"] > 0
    if status >= 0 and name == "mid":
        sampled_data_parity(zc, oc, p, o, ids, w, synth.hidden_device(wl, 0, 0, dev), dev,
                            n=128)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["mid", "hier"])
def test_greedy_then_repair_workload(dev, name):
    wl = synth.WORKLOADS[name]
    zc, oc = cfgs(wl, cap_rows=2 * wl.S * wl.K, repair=1)
    ids, _ = synth.routing(wl, 1)
    p = zb.Plan(zc, dev, with_row_src=False)
    zb.plan(p, torch.from_numpy(ids).to(dev))
    status, _ = zb.plan_status(p)
    assert_plan_equal(plan_tables(p), oracle.plan(oc, ids, want_M=False), status)


def test_maximum_shape(dev):
    """P = 32, E = 384, R = 31 (every slot filled): the largest quota-index
    table and the most rounds (31)."""
    rng = np.random.default_rng(77)
    E, ids, pl = _random_placed(rng, 32, 12, 4, 40, 31, 0.8)
    for j in range(32):  # fill every slot
        held = set(pl[j][pl[j] >= 0].tolist())
        free = [e for e in range(E) if e // 12 != j and e not in held]
        for s_ in range(31):
            if pl[j, s_] < 0:
                pl[j, s_] = free.pop(int(rng.integers(0, len(free))))
    for relax in (0, 1):
        kw = dict(P=32, E=E, K=4, S=40, H=8, R=31, gpus_per_node=4, cap_rows=32 * 40 * 4,
                  repair=1, relax=relax, C=0.2)
        p, o, status = _placed(zb.Config(**kw), oracle.Config(**kw), ids, pl, dev)
        assert status >= 0 and o["repaired"] > 0
