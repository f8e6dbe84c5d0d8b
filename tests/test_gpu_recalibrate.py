"""GPU parity of placement recalibration (zb_recalibrate: ViBE incremental
slot changes, mode 0; Zepp eq. (4) intra-node swaps, mode 1) against the
oracle: the same steps, final placement and max load, on the hand example,
small random cases and the drift and hier workloads at full size."""
import numpy as np
import pytest
import torch

import oracle
from test_oracle_recalibrate import _case
from token_dispatch_top_b200 import build, synth, zb

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev(cuda_device):
    build.build()
    zb.load()
    return cuda_device


def _parity(ocfg, cnt, pl, mode, eps, max_swaps, dev):
    zcfg = zb.Config(P=ocfg.P, E=ocfg.E, K=ocfg.K, S=ocfg.S, H=ocfg.H, R=ocfg.R,
                     gpus_per_node=ocfg.gpus_per_node, cap_rows=ocfg.cap())
    want = oracle.recalibrate(ocfg, cnt, pl, mode, eps, max_swaps)
    pl_d = torch.from_numpy(np.ascontiguousarray(pl, np.int32)).to(dev)
    cnt_d = torch.from_numpy(np.ascontiguousarray(cnt, np.int32)).to(dev)
    got = zb.recalibrate(zcfg, cnt_d, pl_d, mode, eps, max_swaps)
    assert got == want[1:], (got, want[1:])
    np.testing.assert_array_equal(pl_d.cpu().numpy(), want[0])
    return want


def test_hand_example(dev):
    cfg = oracle.Config(P=2, E=2, K=1, S=4, H=8, R=1)
    cnt = np.array([[4, 0], [2, 2]], np.int32)
    pl, n, mx = _parity(cfg, cnt, np.full((2, 1), -1, np.int32), 0, 0.03, 10, dev)
    assert (n, mx) == (1, 4)


@pytest.mark.parametrize("seed", range(16))
def test_random_small(dev, seed):
    rng = np.random.default_rng(1500 + seed)
    mode = seed % 2
    P = int(rng.choice([4, 6, 8]))
    gpn = (2 if P != 6 else 3) if mode == 1 else int(rng.choice([1, 2]))
    cfg, ids, pl = _case(rng, P, int(rng.integers(1, 4)), int(rng.integers(1, 5)),
                         int(rng.integers(2, 40)), int(rng.integers(1, 4)), gpn,
                         float(rng.uniform(0.8, 2.5)))
    cnt = oracle.plan(cfg, ids, want_M=False, placement=pl)["cnt"]
    _parity(cfg, cnt, pl, mode, float(rng.choice([0.0, 0.03, 0.1])), 8, dev)


@pytest.mark.parametrize("step", [16, 32, 63])
def test_drift_incremental(dev, step):
    wl = synth.WORKLOADS["drift"]
    cfg = oracle.Config(P=wl.P, E=wl.E, K=wl.K, S=wl.S, H=wl.H, R=wl.R,
                        cap_rows=3 * wl.S * wl.K)
    pl0 = oracle.plan(cfg, synth.routing(wl, 0, 0)[0], want_M=False)["rep_expert"]
    ids, _ = synth.routing(wl, 0, step)
    cnt = oracle.plan(cfg, ids, want_M=False, placement=pl0)["cnt"]
    pl, n, mx = _parity(cfg, cnt, pl0, 0, 0.03, 64, dev)
    assert n >= 1


def test_hier_intra_node(dev):
    wl = synth.WORKLOADS["hier"]
    cfg = oracle.Config(P=wl.P, E=wl.E, K=wl.K, S=wl.S, H=wl.H, R=wl.R,
                        gpus_per_node=wl.gpus_per_node, cap_rows=3 * wl.S * wl.K)
    pl0 = oracle.plan(cfg, synth.routing(wl, 0)[0], want_M=False)["rep_expert"]
    ids, _ = synth.routing(wl, 1)  # another batch: the placement is stale
    cnt = oracle.plan(cfg, ids, want_M=False, placement=pl0)["cnt"]
    _parity(cfg, cnt, pl0, 1, 0.03, 16, dev)


def test_rejects_invalid(dev):
    zcfg = zb.Config(P=2, E=4, K=1, S=4, H=8, R=1)
    cnt = torch.zeros((2, 4), dtype=torch.int32, device=dev)
    bad = torch.tensor([[0], [3]], dtype=torch.int32, device=dev)  # expert 0 is homed on 0
    with pytest.raises(zb.ZbError):
        zb.recalibrate(zcfg, cnt, bad)
