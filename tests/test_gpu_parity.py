"""GPU parity: the sm_100a path through the C ABI against the CPU oracle.

Bit-exact for the histogram, plan tables, cu_seqlens, dst_row/row_src, the
dispatched rows and the combined output (the combine's summation order is
fixed, so no tolerance is taken).  Small cases compare every element; the
full-size workloads compare the whole plan and sampled rows of dispatch and
combine, plus properties that hold at any size.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import parity
from parity import bf16_to_bits, bits_to_bf16, cfgs, gpu_plan, plan_tables, assert_plan_equal
from token_dispatch_top_b200 import build, synth, zb

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")


@pytest.fixture(scope="module")
def dev(cuda_device):
    build.build()
    zb.load()
    return cuda_device


def _rand_bits(rng, shape):
    x = rng.standard_normal(shape, dtype=np.float32)
    return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def full_parity(zc, oc, ids, w, hidden_bits, y_bits, dev, with_row_src=True, stream=None):
    """Plan, dispatch and combine on both sides; compare every element."""
    ctx = torch.cuda.stream(stream) if stream is not None else torch.cuda.stream(
        torch.cuda.current_stream())
    with ctx:
        p, status, max_load = gpu_plan(zc, ids, dev, with_row_src)
        g = plan_tables(p)
    o = oracle.plan(oc, ids)
    assert_plan_equal(g, o, status)
    if status < 0:
        return p, status
    P, S, K, H, cap = zc.P, zc.S, zc.K, zc.H, zc.cap
    with ctx:
        hid = bits_to_bf16(hidden_bits, dev)
        buf = torch.full((P, cap, H), 0, dtype=torch.int16, device=dev)
        buf.fill_(parity.SENTINEL)
        buf = buf.view(torch.bfloat16)
        zb.dispatch(p, hid, buf)
        w_d = torch.from_numpy(np.ascontiguousarray(w, np.float32)).to(dev)
        out_a = torch.empty((P, S, H), dtype=torch.bfloat16, device=dev)
        zb.combine(p, buf, w_d, out_a)
        y_d = bits_to_bf16(y_bits, dev).view(P, cap, H)
        out_b = torch.empty((P, S, H), dtype=torch.bfloat16, device=dev)
        zb.combine(p, y_d, w_d, out_b)
        torch.cuda.current_stream().synchronize()
    ob = np.full((P, cap, H), parity.SENTINEL, np.uint16)
    oracle.dispatch(oc, o["dst_row"], hidden_bits, ob)
    gb = bf16_to_bits(buf)
    np.testing.assert_array_equal(gb, ob)  # rows past the load keep the sentinel too
    oa = oracle.combine(oc, o["dst_row"], ob.reshape(P * cap, H), w)
    np.testing.assert_array_equal(bf16_to_bits(out_a), oa)
    oy = oracle.combine(oc, o["dst_row"], y_bits.reshape(P * cap, H), w)
    np.testing.assert_array_equal(bf16_to_bits(out_b), oy)
    return p, status


# ------------------------------------------------------------- hand examples

@pytest.mark.parametrize("ex", json.load(open(GOLDEN))["examples"], ids=lambda e: e["name"])
def test_hand_examples(dev, ex):
    d = ex["cfg"]
    kw = dict(P=d["P"], E=d["E"], K=d["K"], S=d["S"], H=d["H"], R=d["R"], C=d.get("C", 0.0),
              gpus_per_node=d.get("gpus_per_node", 1), cap_rows=d.get("cap_rows"),
              policy=d.get("policy", 0), relax=d.get("relax", 0), repair=d.get("repair", 0))
    zc, oc = zb.Config(**kw), oracle.Config(**kw)
    ids = np.array(ex["ids"], np.int32).reshape(zc.P, zc.S, zc.K)
    if "placement" in ex:  # a kept placement: the plan tables through zb_plan_placed
        pl = np.array(ex["placement"], np.int32)
        p = zb.Plan(zc, dev)
        zb.plan_placed(p, torch.from_numpy(ids).to(dev), torch.from_numpy(pl).to(dev))
        status, _ = zb.plan_status(p)
        assert_plan_equal(plan_tables(p), oracle.plan(oc, ids, placement=pl), status)
        return
    rng = np.random.default_rng(0)
    w = rng.dirichlet(np.ones(zc.K), size=(zc.P, zc.S)).astype(np.float32)
    full_parity(zc, oc, ids, w, _rand_bits(rng, (zc.P, zc.S, zc.H)),
                _rand_bits(rng, (zc.P * zc.cap, zc.H)), dev)


# ------------------------------------------------------------- random small

def _small_cases(n=60, seed=21):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        P = int(rng.choice([1, 2, 3, 4, 6, 8, 16, 32]))
        gpn = int(rng.choice([g for g in (1, 2, 4, 8) if P % g == 0]))
        Eh = int(rng.integers(1, min(12, 384 // P) + 1))
        E = P * Eh
        K = int(rng.integers(1, 9))
        S = int(rng.integers(0, 300))
        R = int(rng.integers(0, min(P, 4)))
        H = int(rng.choice([8, 16, 64, 136]))
        p = 1.0 / np.arange(1, E + 1) ** rng.uniform(0, 2)
        p = p[rng.permutation(E)] / p.sum()
        ids = rng.choice(E, size=(P, S, K), p=p).astype(np.int32)
        out.append((dict(P=P, E=E, K=K, S=S, H=H, R=R, C=0.1, gpus_per_node=gpn,
                         policy=len(out) % 2), ids))
    return out


SMALL = _small_cases()


@pytest.mark.parametrize("k", range(len(SMALL)))
def test_random_small(dev, k):
    kw, ids = SMALL[k]
    rng = np.random.default_rng(1000 + k)
    # cap large enough for an unbalanced plan: the sum of all entries
    kw = dict(kw, cap_rows=max(1, kw["P"] * kw["S"] * kw["K"]))
    zc, oc = zb.Config(**kw), oracle.Config(**kw)
    w = rng.dirichlet(np.ones(zc.K), size=(zc.P, zc.S)).astype(np.float32)
    full_parity(zc, oc, ids, w, _rand_bits(rng, (zc.P, zc.S, zc.H)),
                _rand_bits(rng, (zc.P * zc.cap, zc.H)), dev)


# ------------------------------------------------------------- named workloads

@pytest.mark.parametrize("name,seed", [("tiny", 0), ("tiny", 1), ("mid", 0), ("mid", 1)])
def test_workload_full(dev, name, seed):
    """tiny and mid (the benchmark workload, same launch configuration) compared
    element by element, including the receive buffers."""
    wl = synth.WORKLOADS[name]
    zc, oc = cfgs(wl)
    ids, w = synth.routing(wl, seed)
    hidden = synth.hidden_bits(wl, seed)
    y = synth.y_bits(wl, zc.P * zc.cap, seed)
    p, status = full_parity(zc, oc, ids, w, hidden, y, dev, with_row_src=(name == "tiny"))
    assert status == oracle.OK  # both balance to T = S*K


@pytest.mark.parametrize("seed", [2, 3, 4, 5])
def test_mid_seed_sweep_plan(dev, seed):
    wl = synth.WORKLOADS["mid"]
    zc, oc = cfgs(wl)
    ids, _ = synth.routing(wl, seed)
    p, status, _ = gpu_plan(zc, ids, dev)
    assert_plan_equal(plan_tables(p), oracle.plan(oc, ids), status)


def sampled_data_parity(zc, oc, p, o, ids, w, hidden_d, dev, n=384, seed=0):
    """Dispatch and combine on the device at full size; compare sampled token
    rows with the oracle computed one token at a time."""
    P, S, K, H, cap = zc.P, zc.S, zc.K, zc.H, zc.cap
    rng = np.random.default_rng(seed)
    tok = np.unique(np.concatenate([[0, P * S - 1], rng.integers(0, P * S, n)]))
    buf = torch.empty((P, cap, H), dtype=torch.int16, device=dev)
    buf.fill_(parity.SENTINEL)
    buf = buf.view(torch.bfloat16)
    zb.dispatch(p, hidden_d, buf)
    # sampled rows: every destination row of a sampled token holds its hidden row
    dst = o["dst_row"].reshape(P * S, K)
    rows = torch.from_numpy(dst[tok].ravel().astype(np.int64)).to(dev)
    got = buf.view(P * cap, H).index_select(0, rows).view(len(tok), K, H)
    want = hidden_d.view(P * S, H).index_select(0, torch.from_numpy(tok).to(dev))
    assert torch.equal(got.view(torch.int16), want.view(torch.int16)[:, None, :].expand_as(
        got.view(torch.int16)))
    # rows past each rank's load are untouched
    la = o["load_after"]
    spare = [(j, r) for j in range(P) for r in rng.integers(la[j], cap, 8) if la[j] < cap]
    if spare:
        idx = torch.tensor([j * cap + r for j, r in spare], device=dev)
        assert bool((buf.view(P * cap, H).index_select(0, idx).view(torch.int16) ==
                     parity.SENTINEL).all())
    # property at full size: y = buf and weights summing to 1 give back each
    # token's row within one bf16 ulp
    w_d = torch.from_numpy(np.ascontiguousarray(w)).to(dev)
    out = torch.empty((P, S, H), dtype=torch.bfloat16, device=dev)
    zb.combine(p, buf, w_d, out)
    diff = (out.float() - hidden_d.float()).abs()
    ulp = torch.where(hidden_d.float() == 0, torch.full_like(diff, 1e-38),
                      hidden_d.float().abs() * 2.0 ** -7)
    assert bool((diff <= ulp).all())
    # independent expert outputs: exact against the oracle on sampled tokens
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234 + seed)
    y = torch.randn((P, cap, H), generator=gen, device=dev, dtype=torch.bfloat16)
    zb.combine(p, y, w_d, out)
    yk = bf16_to_bits(y.view(P * cap, H).index_select(0, rows))
    n_t = len(tok)
    ocfg = oracle.Config(P=1, E=1, K=K, S=n_t, H=H, R=0, cap_rows=n_t * K)
    want_o = oracle.combine(ocfg, np.arange(n_t * K, dtype=np.int32).reshape(1, n_t, K), yk,
                            w.reshape(P * S, K)[tok].reshape(1, n_t, K))
    got_o = bf16_to_bits(out.view(P * S, H).index_select(0, torch.from_numpy(tok).to(dev)))
    np.testing.assert_array_equal(got_o, want_o[0])
    del buf, y, out


@pytest.mark.parametrize("name,seed", [("mid", 0), ("mid", 3), ("hot", 0), ("hot", 1),
                                       ("hier", 0), ("hier", 2)])
def test_locality_policy_plan(dev, name, seed):
    """The locality-aware receiver policy, full-size plans bit-exact."""
    wl = synth.WORKLOADS[name]
    zc, oc = cfgs(wl, cap_rows=2 * wl.S * wl.K, policy=zb.POLICY_LOCAL)
    ids, _ = synth.routing(wl, seed)
    p, status, _ = gpu_plan(zc, ids, dev, with_row_src=False)
    assert_plan_equal(plan_tables(p), oracle.plan(oc, ids, want_M=False), status)


@pytest.mark.parametrize("name", ["hot", "hier"])
def test_workload_full_size(dev, name):
    """Full-size plan bit-exact; dispatch/combine sampled (same launch path)."""
    wl = synth.WORKLOADS[name]
    zc, oc = cfgs(wl, cap_rows=2 * wl.S * wl.K)
    ids, w = synth.routing(wl, 0)
    p, status, _ = gpu_plan(zc, ids, dev)
    o = oracle.plan(oc, ids)
    assert_plan_equal(plan_tables(p), o, status)
    assert status in (oracle.OK, oracle.UNBALANCED)
    hidden = synth.hidden_device(wl, 0, 0, dev)
    sampled_data_parity(zc, oc, p, o, ids, w, hidden, dev)
    # at the water level the plan refuses to fit in S*K rows when unbalanced
    if status == oracle.UNBALANCED:
        zc2, oc2 = cfgs(wl)
        p2, st2, _ = gpu_plan(zc2, ids, dev)
        assert st2 == oracle.ERR_CAPACITY == oracle.plan(oc2, ids, want_M=False)["status"]
    torch.cuda.empty_cache()


def test_drift_all_steps(dev):
    """64 re-planned invocations of the drifting workload: every plan bit-exact,
    dispatch/combine sampled on a few steps."""
    wl = synth.WORKLOADS["drift"]
    zc, oc = cfgs(wl, cap_rows=2 * wl.S * wl.K)
    data_steps = {0, 1, 32, 63}
    for step in range(wl.steps):
        ids, w = synth.routing(wl, 0, step)
        p, status, _ = gpu_plan(zc, ids, dev, with_row_src=False)
        o = oracle.plan(oc, ids, want_M=False)
        assert_plan_equal(plan_tables(p), o, status)
        if step in data_steps:
            hidden = synth.hidden_device(wl, 0, step, dev)
            sampled_data_parity(zc, oc, p, o, ids, w, hidden, dev, n=128, seed=step)
            del hidden
            torch.cuda.empty_cache()


# ------------------------------------------------------------- edge cases

def _run_small(dev, ids, K=None, H=16, R=1, P=None, E=None, cap_rows=None, gpn=1, seed=0,
               with_row_src=True, stream=None):
    P = P or ids.shape[0]
    S = ids.shape[1]
    K = K or ids.shape[2]
    kw = dict(P=P, E=E, K=K, S=S, H=H, R=R, C=0.0, gpus_per_node=gpn, cap_rows=cap_rows)
    zc, oc = zb.Config(**kw), oracle.Config(**kw)
    rng = np.random.default_rng(seed)
    w = rng.dirichlet(np.ones(K), size=(P, S)).astype(np.float32)
    return full_parity(zc, oc, ids, w, _rand_bits(rng, (P, S, H)),
                       _rand_bits(rng, (P * zc.cap, H)), dev, with_row_src, stream)


def test_empty_input(dev):
    p, status = _run_small(dev, np.zeros((4, 0, 2), np.int32), E=8)
    assert status == oracle.OK


def test_single_rank_and_no_slots(dev):
    rng = np.random.default_rng(2)
    _run_small(dev, rng.integers(0, 8, (1, 100, 3)).astype(np.int32), E=8, R=0)
    _run_small(dev, rng.integers(0, 8, (4, 100, 3)).astype(np.int32), E=8, R=0,
               cap_rows=1200)


def test_ragged_chunks_and_k1(dev):
    rng = np.random.default_rng(3)
    # S*K = 3000: one full chunk of 2048 entries and a ragged tail
    _run_small(dev, rng.integers(0, 9, (3, 1000, 3)).astype(np.int32), E=9, R=2,
               cap_rows=9000)
    _run_small(dev, rng.integers(0, 12, (4, 2049, 1)).astype(np.int32), E=12, R=3, H=8,
               cap_rows=8196)


def test_maximum_shape(dev):
    """P = 32 ranks, E = 384 experts, K = 16, R = 31 slots, two-level cost."""
    rng = np.random.default_rng(4)
    P, E, K, S = 32, 384, 16, 96
    p = 1.0 / np.arange(1, E + 1) ** 1.2
    ids = np.stack([np.stack([rng.choice(E, K, replace=False, p=p / p.sum())
                              for _ in range(S)]) for _ in range(P)]).astype(np.int32)
    _run_small(dev, ids, E=E, R=31, H=64, gpn=8, cap_rows=S * K * 2)
    _run_small(dev, ids, E=E, R=2, H=64, gpn=1, cap_rows=S * K * P)


@pytest.mark.parametrize("K,H", [(7, 1032), (9, 1032), (12, 1032), (13, 1032), (14, 1032),
                                 (16, 1032), (8, 1040), (16, 1040), (7, 4112), (8, 4112)])
def test_large_k_two_vectors_in_flight(dev, K, H):
    """K = 7..16 combine.  H = 1032 and 1040: 16-byte vectors, two per row in
    flight, with a ragged last chunk.  H = 4112 at K = 7 and 8: the 32-byte
    kernel, 257 vectors per row, also ragged."""
    rng = np.random.default_rng(40 + K)
    P, E, S = 4, 32, 70
    ids = rng.integers(0, E, (P, S, K)).astype(np.int32)
    kw = dict(P=P, E=E, K=K, S=S, H=H, R=2, cap_rows=P * S * K)
    zc, oc = zb.Config(**kw), oracle.Config(**kw)
    w = rng.dirichlet(np.ones(K), size=(P, S)).astype(np.float32)
    full_parity(zc, oc, ids, w, _rand_bits(rng, (P, S, H)), _rand_bits(rng, (P * zc.cap, H)),
                dev, with_row_src=False)


def test_combine_on_16_byte_aligned_buffers(dev):
    """y and out 16- but not 32-byte aligned: K = 8 takes the 16-byte kernel,
    bit for bit the same as the 32-byte one on aligned copies."""
    rng = np.random.default_rng(8)
    P, E, K, S, H = 4, 32, 8, 50, 4096
    ids = rng.integers(0, E, (P, S, K)).astype(np.int32)
    zc = zb.Config(P=P, E=E, K=K, S=S, H=H, R=1, cap_rows=P * S * K)
    p, status, _ = gpu_plan(zc, ids, dev, with_row_src=False)
    assert status >= 0
    w = torch.from_numpy(rng.dirichlet(np.ones(K), size=(P, S)).astype(np.float32)).to(dev)
    y_a = bits_to_bf16(_rand_bits(rng, (P, zc.cap, H)), dev)
    y_raw = torch.empty(y_a.numel() + 8, dtype=torch.bfloat16, device=dev)
    y_u = y_raw[8:].view(P, zc.cap, H)  # 16-byte offset
    y_u.copy_(y_a)
    out_raw = torch.empty(P * S * H + 8, dtype=torch.bfloat16, device=dev)
    out_u = out_raw[8:].view(P, S, H)
    out_a = torch.empty((P, S, H), dtype=torch.bfloat16, device=dev)
    assert y_u.data_ptr() % 32 == 16 and out_u.data_ptr() % 32 == 16
    zb.combine(p, y_a, w, out_a)
    zb.combine(p, y_u, w, out_u)
    torch.cuda.synchronize()
    assert torch.equal(out_a.view(torch.int16), out_u.view(torch.int16))


def test_all_rows_on_one_expert_and_duplicates(dev):
    _run_small(dev, np.zeros((8, 64, 4), np.int32), E=16, R=7)
    rng = np.random.default_rng(5)
    ids = rng.integers(0, 2, (4, 50, 6)).astype(np.int32)  # many duplicates per token
    _run_small(dev, ids, E=8, R=3, cap_rows=1200)


def test_bad_ids_write_nothing(dev):
    ids = np.zeros((2, 4, 2), np.int32)
    ids[0, 1, 1] = -1
    ids[1, 3, 0] = 4
    zc = zb.Config(P=2, E=4, K=2, S=4, H=16, R=1)
    p, status, _ = gpu_plan(zc, ids, dev)
    assert status == oracle.ERR_BAD_ID == oracle.plan(oracle.Config(P=2, E=4, K=2, S=4, H=16,
                                                                      R=1), ids)["status"]
    assert int(p.stats[zb.STAT_BAD_IDS]) == 2
    hid = torch.randn((2, 4, 16), device=dev).to(torch.bfloat16)
    buf = torch.full((2, 8, 16), parity.SENTINEL, dtype=torch.int16, device=dev) \
        .view(torch.bfloat16)
    zb.dispatch(p, hid, buf)
    out = torch.full((2, 4, 16), parity.SENTINEL, dtype=torch.int16, device=dev) \
        .view(torch.bfloat16)
    zb.combine(p, buf, torch.ones((2, 4, 2), device=dev), out)
    torch.cuda.synchronize()
    assert bool((buf.view(torch.int16) == parity.SENTINEL).all())
    assert bool((out.view(torch.int16) == parity.SENTINEL).all())


@pytest.mark.parametrize("P,E,K,S", [(8, 32, 2, 39000), (4, 16, 8, 298000)])
def test_assign_several_chunks_per_cta(dev, P, E, K, S):
    """Batches whose assignment grid would not fit the device at once, so each
    assignment CTA takes 2 (P=8: 39 chunks per source) or 4 consecutive chunks
    (P=4: 1165 chunks per source), the last CTA fewer, the last chunk ragged:
    the whole plan, dst_row and row_src bit-exact."""
    rng = np.random.default_rng(P)
    pop = 1.0 / np.arange(1, E + 1) ** 1.1
    ids = rng.choice(E, size=(P, S, K), p=pop[rng.permutation(E)] / pop.sum()).astype(np.int32)
    kw = dict(P=P, E=E, K=K, S=S, H=8, R=2, C=0.0, cap_rows=2 * S * K)
    zc, oc = zb.Config(**kw), oracle.Config(**kw)
    p, status, _ = gpu_plan(zc, ids, dev)
    assert_plan_equal(plan_tables(p), oracle.plan(oc, ids, want_M=False), status)
    del p
    torch.cuda.empty_cache()


def test_ids_far_out_of_range(dev):
    """Ids far outside [0, E) (beyond every table an id indexes) are counted
    and stop the plan like any bad id; the same on the per-rank entry points.
    A ragged chunk tail follows the bad ids."""
    rng = np.random.default_rng(11)
    P, E, K, S = 3, 12, 4, 700
    ids = rng.integers(0, E, (P, S, K)).astype(np.int32)
    bad = [(0, 5, 1, 1 << 30), (1, 699, 3, 4096), (2, 0, 0, -7), (2, 321, 2, -(1 << 31)),
           (1, 100, 0, 384), (0, 600, 2, 2**31 - 1)]
    for r, t, k, v in bad:
        ids[r, t, k] = v
    kw = dict(P=P, E=E, K=K, S=S, H=16, R=1)
    zc, oc = zb.Config(**kw), oracle.Config(**kw)
    o = oracle.plan(oc, ids, want_M=False)
    assert o["status"] == oracle.ERR_BAD_ID
    p, status, _ = gpu_plan(zc, ids, dev)
    assert status == oracle.ERR_BAD_ID
    assert int(p.stats[zb.STAT_BAD_IDS]) == len(bad)
    rps = [zb.RankPlan(zc, r, dev) for r in range(P)]
    ids_d = [torch.from_numpy(np.ascontiguousarray(ids[r])).to(dev) for r in range(P)]
    for r in range(P):
        zb.count(rps[r], ids_d[r])
    table = torch.stack([rp.counts for rp in rps])
    np.testing.assert_array_equal(table.cpu().numpy(),
                                  np.stack([oracle.count(oc, ids[r]) for r in range(P)]))
    for r in range(P):
        rps[r].table.copy_(table)
        zb.plan_rank(rps[r], ids_d[r])
        assert int(rps[r].stats[zb.STAT_STATUS]) == oracle.ERR_BAD_ID


def test_capacity_then_unbalanced(dev):
    ids = np.array([[0, 1, 2], [0, 1, 2]], np.int32).reshape(2, 3, 1)
    zc = zb.Config(P=2, E=6, K=1, S=3, H=16, R=1, cap_rows=3)
    p, status, max_load = gpu_plan(zc, ids, dev)
    assert status == oracle.ERR_CAPACITY and max_load == 4
    buf = torch.full((2, 3, 16), parity.SENTINEL, dtype=torch.int16, device=dev) \
        .view(torch.bfloat16)
    zb.dispatch(p, torch.randn((2, 3, 16), device=dev).to(torch.bfloat16), buf)
    torch.cuda.synchronize()
    assert bool((buf.view(torch.int16) == parity.SENTINEL).all())
    p, status = _run_small(dev, ids, E=6, R=1, cap_rows=4)
    assert status == oracle.UNBALANCED


def test_without_row_src_and_on_a_side_stream(dev):
    rng = np.random.default_rng(6)
    ids = rng.integers(0, 16, (4, 300, 2)).astype(np.int32)
    side = torch.cuda.Stream()
    _run_small(dev, ids, E=16, R=2, cap_rows=2400, with_row_src=False, stream=side)


def test_plan_buffers_are_reusable(dev):
    """A second plan into the same buffers leaves no trace of the first."""
    wl = synth.WORKLOADS["tiny"]
    zc, oc = cfgs(wl)
    p = zb.Plan(zc, dev)
    for seed in (0, 1, 2):
        ids, _ = synth.routing(wl, seed)
        zb.plan(p, torch.from_numpy(ids).to(dev))
        status, _ = zb.plan_status(p)
        assert_plan_equal(plan_tables(p), oracle.plan(oc, ids), status)


def test_combine_special_values(dev):
    """Infinities, subnormals and signed zeros follow IEEE through the fold;
    NaN stays NaN (its payload is not compared)."""
    P, S, K, H = 2, 8, 3, 64
    rng = np.random.default_rng(7)
    ids = rng.integers(0, 4, (P, S, K)).astype(np.int32)
    kw = dict(P=P, E=4, K=K, S=S, H=H, R=1, cap_rows=P * S * K)
    zc, oc = zb.Config(**kw), oracle.Config(**kw)
    p, status, _ = gpu_plan(zc, ids, dev)
    o = oracle.plan(oc, ids)
    assert status >= 0
    y = _rand_bits(rng, (P * zc.cap, H))
    specials = np.array([0x7F80, 0xFF80, 0x7FC0, 0x0001, 0x8001, 0x8000, 0x0000, 0x7F7F],
                        np.uint16)
    y.ravel()[rng.integers(0, y.size, 400)] = rng.choice(specials, 400)
    w = rng.standard_normal((P, S, K)).astype(np.float32)
    w.ravel()[:5] = [0.0, -0.0, 1e-40, 3e38, -3e38]
    out = torch.empty((P, S, H), dtype=torch.bfloat16, device=dev)
    zb.combine(p, bits_to_bf16(y, dev).view(P, zc.cap, H),
               torch.from_numpy(w).to(dev), out)
    got = bf16_to_bits(out)
    want = oracle.combine(oc, o["dst_row"], y, w)
    nan_g = ((got & 0x7F80) == 0x7F80) & ((got & 0x7F) != 0)
    nan_w = ((want & 0x7F80) == 0x7F80) & ((want & 0x7F) != 0)
    np.testing.assert_array_equal(nan_g, nan_w)
    np.testing.assert_array_equal(got[~nan_w], want[~nan_w])


# ------------------------------------------------------------- kept placement

def _random_placement(rng, P, E, R):
    Eh = E // P
    pl = np.full((P, R), -1, np.int32)
    for j in range(P):
        others = [e for e in range(E) if e // Eh != j]
        n = int(rng.integers(0, min(R, len(others)) + 1))
        if n:
            pl[j, :n] = rng.choice(others, size=n, replace=False)
    return pl


@pytest.mark.parametrize("k", range(0, len(SMALL), 2))
def test_placed_random_small(dev, k):
    """zb_plan_placed against the oracle's plan with the same placement."""
    kw, ids = SMALL[k]
    if kw["R"] == 0:
        pytest.skip("no slots to place")
    rng = np.random.default_rng(2000 + k)
    kw = dict(kw, cap_rows=max(1, kw["P"] * kw["S"] * kw["K"]))
    zc, oc = zb.Config(**kw), oracle.Config(**kw)
    pl = _random_placement(rng, zc.P, zc.E, zc.R)
    p = zb.Plan(zc, dev)
    zb.plan_placed(p, torch.from_numpy(ids).to(dev), torch.from_numpy(pl).to(dev))
    status, _ = zb.plan_status(p)
    assert_plan_equal(plan_tables(p), oracle.plan(oc, ids, placement=pl), status)


def test_placed_drift_and_aliasing(dev):
    """The drifting workload at full size: step 0's placement kept for later
    steps, passed as the plan's own rep_expert (aliasing is allowed)."""
    wl = synth.WORKLOADS["drift"]
    zc, oc = cfgs(wl, cap_rows=3 * wl.S * wl.K)
    ids0, _ = synth.routing(wl, 0, 0)
    p = zb.Plan(zc, dev, with_row_src=False)
    zb.plan(p, torch.from_numpy(ids0).to(dev))
    zb.plan_status(p)
    o0 = oracle.plan(oc, ids0, want_M=False)
    for step in (1, 31, 63):
        ids, _ = synth.routing(wl, 0, step)
        zb.plan_placed(p, torch.from_numpy(ids).to(dev), p.rep_expert)
        status, _ = zb.plan_status(p)
        assert_plan_equal(plan_tables(p), oracle.plan(oc, ids, want_M=False,
                                                      placement=o0["rep_expert"]), status)


def test_placed_invalid(dev):
    zc = zb.Config(P=3, E=6, K=1, S=2, H=8, R=2, cap_rows=6)
    ids = torch.zeros((3, 2, 1), dtype=torch.int32, device=dev)
    p = zb.Plan(zc, dev)
    for bad in ([[0, -1], [-1, -1], [-1, -1]], [[2, 2], [-1, -1], [-1, -1]],
                [[6, -1], [-1, -1], [-1, -1]], [[-2, -1], [-1, -1], [-1, -1]]):
        zb.plan_placed(p, ids, torch.tensor(bad, dtype=torch.int32, device=dev))
        with pytest.raises(zb.ZbError) as err:
            zb.plan_status(p)
        assert err.value.status == zb.ERR_INVALID
    zb.plan_placed(p, ids, torch.tensor([[2, 4], [0, -1], [-1, 1]], dtype=torch.int32,
                                        device=dev))
    assert zb.plan_status(p)[0] in (zb.OK, zb.WARN_UNBALANCED)
