"""The device plan decomposes by source rank, as the oracle's does: shuffling
other ranks' entries (same counts) leaves every plan table and the source's
dst_row unchanged on the GPU too, for each option of the planner."""
import numpy as np
import pytest
import torch

from parity import gpu_plan, plan_tables
from test_plan_decomposition import _case, _stand_in
from token_dispatch_top_b200 import build, zb

pytestmark = pytest.mark.gpu

TABLES = ("cnt", "rep_expert", "rep_quota", "home_quota", "load_before", "load_after",
          "cu_seqlens")


@pytest.fixture(scope="module")
def dev(cuda_device):
    build.build()
    zb.load()
    return cuda_device


@pytest.mark.parametrize("seed", range(8))
def test_rows_of_a_source_depend_on_counts_and_own_ids(dev, seed):
    ocfg, ids = _case(seed, P=8, Eh=4, K=4, S=300, policy=seed % 2, relax=(seed // 2) % 2,
                      repair=(seed // 4) % 2)
    zcfg = zb.Config(P=ocfg.P, E=ocfg.E, K=ocfg.K, S=ocfg.S, H=ocfg.H, R=ocfg.R, C=ocfg.C,
                     gpus_per_node=ocfg.gpus_per_node, cap_rows=ocfg.cap_rows,
                     policy=ocfg.policy, relax=ocfg.relax, repair=ocfg.repair)
    p, status, _ = gpu_plan(zcfg, ids, dev, with_row_src=False)
    assert status >= 0
    ref = plan_tables(p)
    rng = np.random.default_rng(200 + seed)
    for i in (0, 3, 7):
        other = ids.copy()
        for j in range(zcfg.P):
            if j != i:
                other[j] = _stand_in(rng, ref["cnt"][j], zcfg.S, zcfg.K)
        q, st2, _ = gpu_plan(zcfg, other, dev, with_row_src=False)
        got = plan_tables(q)
        assert st2 == status
        for k in TABLES:
            np.testing.assert_array_equal(got[k], ref[k], err_msg=k)
        np.testing.assert_array_equal(got["dst_row"][i], ref["dst_row"][i])
        assert got["stats"][zb.STAT_LOCALITY_COST] == ref["stats"][zb.STAT_LOCALITY_COST]
