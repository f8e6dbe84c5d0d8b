"""GPU parity of the per-rank form of the path (one rank of P GPUs) on one GPU.

Every rank's calls run in this one process: ``zb.count`` on the rank's own
ids, the count rows stacked in rank order (what the all-gather between P GPUs
produces), ``zb.plan_rank``, then ``zb.dispatch_rank`` / ``zb.combine_rank``
through a table of P buffer pointers -- P parts of one allocation, or P
separate allocations standing for the other GPUs' buffers.  Everything is
compared bit for bit with the whole-batch device path (``zb.plan``,
``zb.dispatch``, ``zb.combine``) and with the oracle's per-rank functions.
"""
import numpy as np
import pytest
import torch

import oracle
import parity
from parity import bf16_to_bits, bits_to_bf16, plan_tables, PLAN_KEYS
from token_dispatch_top_b200 import build, synth, zb

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev(cuda_device):
    build.build()
    zb.load()
    return cuda_device


def _rank_plans(zc, ids, dev, placement=None):
    """Count, exchange (stack on this GPU), plan every rank."""
    P = zc.P
    ids_d = [torch.from_numpy(np.ascontiguousarray(ids[r])).to(dev) for r in range(P)]
    rps = [zb.RankPlan(zc, r, dev) for r in range(P)]
    for r in range(P):
        zb.count(rps[r], ids_d[r])
    table = torch.stack([rp.counts for rp in rps])
    pl = None if placement is None else torch.from_numpy(placement).to(dev)
    for r in range(P):
        rps[r].table.copy_(table)
        zb.plan_rank(rps[r], ids_d[r], placement=pl)
    status = [zb.plan_status(rp)[0] for rp in rps]
    return rps, table.cpu().numpy(), status


def _whole_plan(zc, ids, dev, placement=None):
    p = zb.Plan(zc, dev, with_row_src=False)
    ids_d = torch.from_numpy(np.ascontiguousarray(ids)).to(dev)
    if placement is None:
        zb.plan(p, ids_d)
    else:
        zb.plan_placed(p, ids_d, torch.from_numpy(placement).to(dev))
    return p, zb.plan_status(p)[0]


def check_rank_plans(zc, oc, ids, dev, placement=None):
    rps, table, status = _rank_plans(zc, ids, dev, placement)
    whole, st = _whole_plan(zc, ids, dev, placement)
    g = plan_tables(whole)
    for r, rp in enumerate(rps):
        np.testing.assert_array_equal(table[r], oracle.count(oc, ids[r]))
        o = oracle.plan_rank(oc, r, table, ids[r], placement=placement)
        assert status[r] == st == o["status"], (r, status[r], st, o["status"])
        if st < 0 and st != oracle.ERR_CAPACITY:
            continue
        for k in PLAN_KEYS:
            got = getattr(rp, k).cpu().numpy()
            np.testing.assert_array_equal(got, g[k], err_msg=f"{k} rank {r}")
            np.testing.assert_array_equal(got, o[k], err_msg=f"{k} rank {r} (oracle)")
        sr, sw = rp.stats.cpu().numpy(), g["stats"]
        np.testing.assert_array_equal(sr, sw)
        if st >= 0:
            np.testing.assert_array_equal(rp.dst_row.cpu().numpy(), g["dst_row"][r])
            np.testing.assert_array_equal(rp.dst_row.cpu().numpy(), o["dst_row"])
    return rps, whole, st


def check_rank_rows(zc, oc, rps, whole, hidden_bits, y_bits, w, dev, separate):
    """dispatch_rank / combine_rank of every rank against zb.dispatch /
    zb.combine and the oracle."""
    P, S, K, H, cap = zc.P, zc.S, zc.K, zc.H, zc.cap
    hid = bits_to_bf16(hidden_bits, dev)
    flat = torch.full((P, cap, H), parity.SENTINEL, dtype=torch.int16, device=dev) \
        .view(torch.bfloat16)
    zb.dispatch(whole, hid, flat)
    if separate:
        bufs = [torch.full((cap, H), parity.SENTINEL, dtype=torch.int16, device=dev)
                .view(torch.bfloat16) for _ in range(P)]
    else:
        one = torch.full((P, cap, H), parity.SENTINEL, dtype=torch.int16, device=dev) \
            .view(torch.bfloat16)
        bufs = list(one.unbind(0))
    for r in range(P):
        zb.dispatch_rank(rps[r], hid[r], bufs)
    torch.cuda.synchronize()
    for j in range(P):
        assert torch.equal(bufs[j].view(torch.int16), flat[j].view(torch.int16)), f"buffer {j}"
    # the oracle's per-rank dispatch into P host buffers
    ob = [np.full((cap, H), parity.SENTINEL, np.uint16) for _ in range(P)]
    for r in range(P):
        oracle.dispatch_ranks(oc, rps[r].dst_row.cpu().numpy(), hidden_bits[r], ob)
    for j in range(P):
        np.testing.assert_array_equal(bf16_to_bits(bufs[j]), ob[j])
    # combine from the dispatched rows and from independent expert outputs
    w_d = torch.from_numpy(np.ascontiguousarray(w, np.float32)).to(dev)
    y_flat = bits_to_bf16(y_bits, dev).view(P, cap, H)
    if separate:
        ys = [y_flat[j].clone() for j in range(P)]
    else:
        ys = list(y_flat.unbind(0))
    for src, src_flat, host in ((bufs, flat, ob), (ys, y_flat, None)):
        want = torch.empty((P, S, H), dtype=torch.bfloat16, device=dev)
        zb.combine(whole, src_flat, w_d, want)
        got = torch.empty((P, S, H), dtype=torch.bfloat16, device=dev)
        for r in range(P):
            zb.combine_rank(rps[r], src, w_d[r], got[r])
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int16), want.view(torch.int16))
        hb = host if host is not None else [y_bits.reshape(P, cap, H)[j] for j in range(P)]
        for r in range(P):
            o = oracle.combine_ranks(oc, rps[r].dst_row.cpu().numpy(), hb, w[r])
            np.testing.assert_array_equal(bf16_to_bits(got[r]), o)


def _rand_bits(rng, shape):
    x = rng.standard_normal(shape, dtype=np.float32)
    return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("name,seed", [("tiny", 0), ("tiny", 1), ("mid", 0)])
def test_named_workloads(dev, name, seed):
    wl = synth.WORKLOADS[name]
    zc, oc = parity.cfgs(wl)
    ids, w = synth.routing(wl, seed)
    rps, whole, st = check_rank_plans(zc, oc, ids, dev)
    assert st == oracle.OK
    rng = np.random.default_rng(seed)
    hidden = synth.hidden_bits(wl, seed)
    y = _rand_bits(rng, (zc.P * zc.cap, zc.H))
    check_rank_rows(zc, oc, rps, whole, hidden, y, w, dev, separate=(seed == 1))


def _small(k):
    rng = np.random.default_rng(300 + k)
    P = int(rng.choice([1, 2, 3, 4, 8, 16]))
    gpn = int(rng.choice([g for g in (1, 2, 4) if P % g == 0]))
    Eh = int(rng.integers(1, 8))
    E, K, S = P * Eh, int(rng.integers(1, 9)), int(rng.integers(0, 400))
    R = int(rng.integers(0, min(P, 4)))
    pop = 1.0 / np.arange(1, E + 1) ** rng.uniform(0.3, 2.0)
    ids = rng.choice(E, size=(P, S, K), p=pop[rng.permutation(E)] / pop.sum()).astype(np.int32)
    kw = dict(P=P, E=E, K=K, S=S, H=int(rng.choice([8, 64, 136])), R=R, C=0.2,
              gpus_per_node=gpn, cap_rows=max(1, P * S * K), policy=k % 2,
              relax=(k // 2) % 2, repair=(k // 4) % 2)
    pl = None
    if (k // 8) % 2 and R > 0:
        pl = np.full((P, R), -1, np.int32)
        for j in range(P):
            foreign = [e for e in rng.permutation(E) if e // Eh != j][:R]
            pl[j, :len(foreign)] = foreign
    return kw, ids, pl, rng


@pytest.mark.parametrize("k", range(24))
def test_random_shapes_every_option(dev, k):
    kw, ids, pl, rng = _small(k)
    zc, oc = zb.Config(**kw), oracle.Config(**kw)
    rps, whole, st = check_rank_plans(zc, oc, ids, dev, placement=pl)
    if st < 0:
        return
    w = rng.dirichlet(np.ones(zc.K), size=(zc.P, zc.S)).astype(np.float32)
    check_rank_rows(zc, oc, rps, whole, _rand_bits(rng, (zc.P, zc.S, zc.H)),
                    _rand_bits(rng, (zc.P * zc.cap, zc.H)), w, dev, separate=bool(k % 3 == 0))


def _device_status(rp) -> int:
    """The plan's status as the planner recorded it (the binding's plan_status
    raises on ERR_INVALID, which is also its code for a bad argument)."""
    torch.cuda.synchronize()
    return int(rp.stats[zb.STAT_STATUS])


def test_inconsistent_counts_and_bad_ids(dev):
    rng = np.random.default_rng(11)
    zc = zb.Config(P=4, E=8, K=2, S=50, H=16, R=1, cap_rows=400)
    ids = rng.integers(0, 8, (4, 50, 2)).astype(np.int32)
    rps, table, status = _rank_plans(zc, ids, dev)
    assert all(s >= 0 for s in status)
    # another rank's counts in rank 1's row (same total): rank 1 refuses
    rp = rps[1]
    t = torch.from_numpy(table).to(dev)
    t[1] = t[2]
    if not torch.equal(t[1], torch.from_numpy(table[1]).to(dev)):
        rp.table.copy_(t)
        zb.plan_rank(rp, torch.from_numpy(ids[1]).to(dev))
        assert _device_status(rp) == zb.ERR_INVALID
        hid = torch.randn((50, 16), device=dev).to(torch.bfloat16)
        bufs = [torch.full((400, 16), parity.SENTINEL, dtype=torch.int16, device=dev)
                .view(torch.bfloat16) for _ in range(4)]
        zb.dispatch_rank(rp, hid, bufs)
        torch.cuda.synchronize()
        assert all(bool((b.view(torch.int16) == parity.SENTINEL).all()) for b in bufs)
    # a row that does not sum to S*K
    t = torch.from_numpy(table).to(dev)
    t[3, 0] += 1
    rps[0].table.copy_(t)
    zb.plan_rank(rps[0], torch.from_numpy(ids[0]).to(dev))
    assert _device_status(rps[0]) == zb.ERR_INVALID
    # an id out of range on rank 2 fails every rank alike
    ids2 = ids.copy()
    ids2[2, 7, 1] = -5
    _, _, status2 = _rank_plans(zc, ids2, dev)
    assert status2 == [zb.ERR_BAD_ID] * 4


def test_hot_full_size_separate_buffers(dev):
    """The benchmark shape of MoonEP (P=8, E=384, K=8, H=7168) in the per-rank
    form with 8 separate receive buffers: plans, buffers and both combines
    equal the whole-batch path (itself compared with the oracle element by
    element in test_gpu_fullsize), including the 32-byte combine."""
    wl = synth.WORKLOADS["hot"]
    zc, oc = parity.cfgs(wl, cap_rows=2 * wl.S * wl.K)
    ids, w = synth.routing(wl, 0)
    P, S, K, H, cap = zc.P, zc.S, zc.K, zc.H, zc.cap
    rps, _, status = _rank_plans(zc, ids, dev)
    whole, st = _whole_plan(zc, ids, dev)
    assert status == [st] * P and st >= 0
    for r in range(P):
        for k in PLAN_KEYS:
            assert torch.equal(getattr(rps[r], k), getattr(whole, k)), k
        assert torch.equal(rps[r].dst_row, whole.dst_row[r])
    hidden = synth.hidden_device(wl, 0, 0, dev)
    flat = torch.empty((P, cap, H), dtype=torch.bfloat16, device=dev)
    zb.dispatch(whole, hidden, flat)
    bufs = [torch.empty((cap, H), dtype=torch.bfloat16, device=dev) for _ in range(P)]
    for r in range(P):
        zb.dispatch_rank(rps[r], hidden[r], bufs)
    la = whole.load_after.cpu().numpy()
    for j in range(P):
        assert torch.equal(bufs[j][:la[j]].view(torch.int16), flat[j, :la[j]].view(torch.int16))
    w_d = torch.from_numpy(w).to(dev)
    want = torch.empty((P, S, H), dtype=torch.bfloat16, device=dev)
    got = torch.empty_like(want)
    zb.combine(whole, flat, w_d, want)
    for r in range(P):
        zb.combine_rank(rps[r], bufs, w_d[r], got[r])
    torch.cuda.synchronize()
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    del flat, bufs, want, got, hidden
    torch.cuda.empty_cache()


def _rank_group_main(port, q):
    """One process, one GPU, a one-rank NCCL group: the RankGroup plumbing
    (symmetric-memory buffers and their pointer tables, the count all-gather,
    the barriers) around the per-rank calls."""
    import os
    import torch.distributed as dist
    from token_dispatch_top_b200 import ranks
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=dev)
    try:
        zc = zb.Config(P=1, E=8, K=3, S=700, H=64, R=0)
        rng = np.random.default_rng(2)
        ids = torch.from_numpy(rng.integers(0, 8, (700, 3)).astype(np.int32)).to(dev)
        w = torch.from_numpy(rng.dirichlet(np.ones(3), 700).astype(np.float32)).to(dev)
        hidden = torch.randn((700, 64), device=dev).to(torch.bfloat16)
        g = ranks.RankGroup(zc, device=dev)
        g.plan_and_dispatch(ids, hidden)
        g.y.copy_(g.buf)  # identity experts
        out = torch.empty((700, 64), dtype=torch.bfloat16, device=dev)
        g.combine(w, out)
        whole = zb.Plan(zc, dev, with_row_src=False)
        zb.plan(whole, ids.view(1, 700, 3))
        buf = torch.empty((1, zc.cap, 64), dtype=torch.bfloat16, device=dev)
        zb.dispatch(whole, hidden.view(1, 700, 64), buf)
        want = torch.empty((1, 700, 64), dtype=torch.bfloat16, device=dev)
        zb.combine(whole, buf, w.view(1, 700, 3), want)
        torch.cuda.synchronize()
        ok = (torch.equal(g.plan.dst_row, whole.dst_row[0]) and
              torch.equal(g.buf.view(torch.int16), buf[0].view(torch.int16)) and
              torch.equal(out.view(torch.int16), want[0].view(torch.int16)) and
              zb.plan_status(g.plan)[0] == zb.OK)
        q.put(bool(ok))
        del g
    finally:
        dist.destroy_process_group()


def test_rank_group_one_gpu(dev):
    import socket
    import torch.multiprocessing as mp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_rank_group_main, args=(port, q))
    p.start()
    ok = q.get(timeout=300)
    p.join(timeout=120)
    assert p.exitcode == 0 and ok


def test_capacity_on_every_rank_writes_nothing(dev):
    """A plan whose rows do not fit cap_rows is ZB_ERR_CAPACITY on every rank
    alike (all ranks compute the same tables), and no rank writes a row."""
    ids = np.array([[0, 1, 2], [0, 1, 2]], np.int32).reshape(2, 3, 1)
    kw = dict(P=2, E=6, K=1, S=3, H=16, R=1, cap_rows=3)
    zc, oc = zb.Config(**kw), oracle.Config(**kw)
    rps, table, status = _rank_plans(zc, ids, dev)
    assert status == [zb.ERR_CAPACITY] * 2
    for r in range(2):
        assert oracle.plan_rank(oc, r, table, ids[r])["status"] == oracle.ERR_CAPACITY
    bufs = [torch.full((3, 16), parity.SENTINEL, dtype=torch.int16, device=dev)
            .view(torch.bfloat16) for _ in range(2)]
    out = torch.full((3, 16), parity.SENTINEL, dtype=torch.int16, device=dev).view(torch.bfloat16)
    for r in range(2):
        zb.dispatch_rank(rps[r], torch.randn((3, 16), device=dev).to(torch.bfloat16), bufs)
        zb.combine_rank(rps[r], bufs, torch.ones((3, 1), device=dev), out)
    torch.cuda.synchronize()
    assert all(bool((b.view(torch.int16) == parity.SENTINEL).all()) for b in bufs)
    assert bool((out.view(torch.int16) == parity.SENTINEL).all())
