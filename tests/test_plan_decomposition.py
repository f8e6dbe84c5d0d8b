"""The plan decomposes by source rank, which is what lets P real ranks plan
without exchanging their ids (the P-GPU form of the path).

* Property, on the oracle: the plan tables depend only on the route counts,
  and the rows of source i depend only on those counts and i's own ids.  Any
  shuffle of another rank's entries (same counts) leaves every table and
  every row of source i unchanged.
* Protocol, on CPU processes with gloo (world size 4 = P): each rank holds its
  own ids, all-gathers the count rows, fills the other ranks' entries with
  any ids of the same counts, plans, and gets exactly the global plan's rows
  for its own source.
* The same protocol through the library binding's count exchange
  (``zb.exchange_counts``) and the oracle's per-rank plan: each rank's
  tables and rows equal the global plan's, under every option.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import oracle

TABLES = ("cnt", "rep_expert", "rep_quota", "home_quota", "load_before", "load_after",
          "cu_seqlens")


def _case(seed, P=4, Eh=3, K=3, S=40, R=2, gpn=2, policy=0, relax=0, repair=0):
    rng = np.random.default_rng(seed)
    E = P * Eh
    pop = 1.0 / np.arange(1, E + 1) ** 1.3
    ids = rng.choice(E, size=(P, S, K), p=pop / pop.sum()).astype(np.int32)
    cfg = oracle.Config(P=P, E=E, K=K, S=S, H=8, R=R, C=0.25, gpus_per_node=gpn,
                        cap_rows=2 * S * K, policy=policy, relax=relax, repair=repair)
    return cfg, ids


def _stand_in(rng, cnt_row, S, K):
    """Ids of one rank with the given per-expert counts, in a random order."""
    flat = np.repeat(np.arange(len(cnt_row)), cnt_row).astype(np.int32)
    assert len(flat) == S * K
    return rng.permutation(flat).reshape(S, K)


@pytest.mark.parametrize("seed", range(12))
def test_rows_of_a_source_depend_on_counts_and_own_ids(seed):
    cfg, ids = _case(seed, policy=seed % 2, relax=(seed // 2) % 2, repair=(seed // 4) % 2)
    ref = oracle.plan(cfg, ids, want_M=False)
    assert ref["status"] >= 0
    rng = np.random.default_rng(100 + seed)
    for i in range(cfg.P):
        other = ids.copy()
        for j in range(cfg.P):
            if j != i:
                other[j] = _stand_in(rng, ref["cnt"][j], cfg.S, cfg.K)
        p = oracle.plan(cfg, other, want_M=False)
        for k in TABLES:
            np.testing.assert_array_equal(p[k], ref[k], err_msg=k)
        assert p["locality_cost"] == ref["locality_cost"]
        np.testing.assert_array_equal(p["dst_row"][i], ref["dst_row"][i])


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, seed, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg, ids = _case(seed, P=world)
        mine = ids[rank]  # a rank sees only its own ids
        row = torch.from_numpy(np.bincount(mine.ravel(), minlength=cfg.E).astype(np.int32))
        rows = [torch.empty_like(row) for _ in range(world)]
        dist.all_gather(rows, row)  # the count exchange
        cnt = torch.stack(rows).numpy()
        rng = np.random.default_rng(1000 + rank)
        local = np.stack([mine if j == rank else _stand_in(rng, cnt[j], cfg.S, cfg.K)
                          for j in range(world)])
        p = oracle.plan(cfg, local, want_M=False)
        q.put((rank, p["dst_row"][rank].copy(), p["cu_seqlens"].copy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("seed", [3, 8])
def test_count_exchange_protocol_gloo(seed):
    world = 4
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, seed, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict()
    for _ in range(world):
        r, rows, cu = q.get(timeout=120)
        got[r] = (rows, cu)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg, ids = _case(seed, P=world)
    ref = oracle.plan(cfg, ids, want_M=False)
    for r in range(world):
        np.testing.assert_array_equal(got[r][0], ref["dst_row"][r])
        np.testing.assert_array_equal(got[r][1], ref["cu_seqlens"])


def _rank_main_binding(rank, world, port, seed, opts, q):
    import torch
    import torch.distributed as dist
    from token_dispatch_top_b200 import zb
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg, ids = _case(seed, P=world, **opts)
        mine = torch.from_numpy(oracle.count(cfg, ids[rank]))  # only this rank's ids
        table = torch.empty((world, cfg.E + 1), dtype=torch.int32)
        zb.exchange_counts(mine, table)
        p = oracle.plan_rank(cfg, rank, table.numpy(), ids[rank])
        q.put((rank, p["status"], p["dst_row"].copy(), {k: p[k].copy() for k in TABLES}))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("seed,opts", [(5, {}), (6, dict(policy=1, relax=1)),
                                       (7, dict(repair=1, R=3))])
def test_binding_count_exchange_gloo(seed, opts):
    world = 4
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main_binding, args=(r, world, port, seed, opts, q))
             for r in range(world)]
    for p in procs:
        p.start()
    got = dict()
    for _ in range(world):
        r, st, rows, tables = q.get(timeout=120)
        got[r] = (st, rows, tables)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg, ids = _case(seed, P=world, **opts)
    ref = oracle.plan(cfg, ids, want_M=False)
    for r in range(world):
        st, rows, tables = got[r]
        assert st == ref["status"]
        np.testing.assert_array_equal(rows, ref["dst_row"][r])
        for k in TABLES:
            np.testing.assert_array_equal(tables[k], ref[k], err_msg=k)


def test_exchange_without_a_process_group():
    import torch
    from token_dispatch_top_b200 import zb
    row = torch.arange(5, dtype=torch.int32)
    table = torch.empty((1, 5), dtype=torch.int32)
    zb.exchange_counts(row, table)
    assert torch.equal(table[0], row)
    with pytest.raises(zb.ZbError):
        zb.exchange_counts(row, torch.empty((2, 5), dtype=torch.int32))
