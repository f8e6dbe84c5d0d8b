"""GPU parity of the merged combine (Zepp 4.2 merge: node-local
pre-reduction) against the oracle: the destination-side partials and the
source-side output bit for bit, on small random cases, the mid workload
(every element) and the hot workload (sampled tokens, checked against the
oracle one token at a time)."""
import numpy as np
import pytest
import torch

import oracle
import parity
from parity import bf16_to_bits, bits_to_bf16, cfgs, gpu_plan
from test_gpu_parity import _rand_bits
from token_dispatch_top_b200 import build, synth, zb

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev(cuda_device):
    build.build()
    zb.load()
    return cuda_device


def merged_combine_parity(zc, oc, ids, y_bits, w, dev):
    p, status, _ = gpu_plan(zc, ids, dev, with_row_src=False)
    assert status >= 0
    m = zb.Merge(zc, dev)
    zb.merge(p, m)
    P, S, cap, H = zc.P, zc.S, zc.cap, zc.H
    y = bits_to_bf16(y_bits, dev).view(P, cap, H)
    w_d = torch.from_numpy(np.ascontiguousarray(w, np.float32)).to(dev)
    part = torch.full((P, cap, H), parity.SENTINEL, dtype=torch.int16, device=dev) \
        .view(torch.bfloat16)
    out = torch.empty((P, S, H), dtype=torch.bfloat16, device=dev)
    zb.combine_reduce(p, m, y, w_d, part)
    zb.combine_merged(p, m, part, out)
    torch.cuda.synchronize()
    o = oracle.plan(oc, ids, want_M=False)
    om = oracle.merge(oc, o["dst_row"])
    opart = np.full((P, cap, H), parity.SENTINEL, np.uint16)
    oracle.combine_reduce(oc, o["dst_row"], om["tok_row"], y_bits.reshape(P * cap, H), w, opart)
    np.testing.assert_array_equal(bf16_to_bits(part), opart)  # unused rows untouched
    oout = oracle.combine_merged(oc, om["tok_row"], opart)
    np.testing.assert_array_equal(bf16_to_bits(out), oout)
    return p, m, part, out


@pytest.mark.parametrize("seed", range(24))
def test_random_small(dev, seed):
    rng = np.random.default_rng(700 + seed)
    P = int(rng.choice([1, 2, 3, 4, 8, 16, 32]))
    Eh = int(rng.integers(1, min(8, 384 // P) + 1))
    K = int(rng.integers(1, 17)) if seed % 4 == 0 else int(rng.integers(1, 9))
    S = int(rng.integers(0, 300))
    R = int(rng.integers(0, min(P, 3)))
    H = int(rng.choice([8, 64, 264, 1032]))
    kw = dict(P=P, E=P * Eh, K=K, S=S, H=H, R=R, cap_rows=max(1, P * S * K))
    zc, oc = zb.Config(**kw), oracle.Config(**kw)
    ids = rng.integers(0, P * Eh, (P, S, K)).astype(np.int32)
    w = rng.dirichlet(np.ones(K), size=(P, S)).astype(np.float32)
    merged_combine_parity(zc, oc, ids, _rand_bits(rng, (P * zc.cap, H)), w, dev)


def test_mid_every_element_and_fully_merged(dev):
    wl = synth.WORKLOADS["mid"]
    zc, oc = cfgs(wl)
    ids, w = synth.routing(wl, 0)
    y = synth.y_bits(wl, zc.P * zc.cap, 0)
    merged_combine_parity(zc, oc, ids, y, w, dev)
    # a single rank: every token fully merged, so the merged combine is the
    # plain combine bit for bit
    kw = dict(P=1, E=8, K=4, S=2048, H=512, R=0)
    zc1 = zb.Config(**kw)
    rng = np.random.default_rng(3)
    ids1 = rng.integers(0, 8, (1, 2048, 4)).astype(np.int32)
    w1 = torch.from_numpy(rng.dirichlet(np.ones(4), size=(1, 2048)).astype(np.float32)).to(dev)
    p, status, _ = gpu_plan(zc1, ids1, dev, with_row_src=False)
    m = zb.Merge(zc1, dev)
    zb.merge(p, m)
    y1 = bits_to_bf16(_rand_bits(rng, (zc1.cap, 512)), dev).view(1, zc1.cap, 512)
    part = torch.empty_like(y1)
    a = torch.empty((1, 2048, 512), dtype=torch.bfloat16, device=dev)
    b = torch.empty_like(a)
    zb.combine_reduce(p, m, y1, w1, part)
    zb.combine_merged(p, m, part, a)
    zb.combine(p, y1, w1, b)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_hot_sampled_tokens(dev):
    wl = synth.WORKLOADS["hot"]
    zc, oc = cfgs(wl, cap_rows=2 * wl.S * wl.K)
    ids, w = synth.routing(wl, 0)
    p, status, _ = gpu_plan(zc, ids, dev, with_row_src=False)
    assert status >= 0
    m = zb.Merge(zc, dev)
    zb.merge(p, m)
    P, S, K, cap, H = zc.P, zc.S, zc.K, zc.cap, zc.H
    gen = torch.Generator(device=dev)
    gen.manual_seed(5)
    y = torch.randn((P, cap, H), generator=gen, device=dev, dtype=torch.bfloat16)
    w_d = torch.from_numpy(w).to(dev)
    part = torch.empty_like(y)
    out = torch.empty((P, S, H), dtype=torch.bfloat16, device=dev)
    zb.combine_reduce(p, m, y, w_d, part)
    zb.combine_merged(p, m, part, out)
    torch.cuda.synchronize()
    rng = np.random.default_rng(9)
    tok = np.unique(np.concatenate([[0, P * S - 1], rng.integers(0, P * S, 256)]))
    dst = p.dst_row.view(-1, K).cpu().numpy()[tok]
    trow = m.tok_row.view(-1, K).cpu().numpy()[tok]
    n = len(tok)
    # the same tokens as a one-rank problem: entry (i, k) at row i*K + k, and
    # merged rows named by the first k of each group
    first = np.array([[i * K + list(trow[i]).index(trow[i, k]) for k in range(K)]
                      for i in range(n)], np.int32)
    yk = bf16_to_bits(y.view(-1, H).index_select(0, torch.from_numpy(
        dst.ravel().astype(np.int64)).to(dev)))
    mini = oracle.Config(P=1, E=1, K=K, S=n, H=H, R=0, cap_rows=n * K)
    opart = oracle.combine_reduce(mini, np.arange(n * K, dtype=np.int32).reshape(1, n, K),
                                  first.reshape(1, n, K), yk,
                                  w.reshape(-1, K)[tok].reshape(1, n, K))
    oout = oracle.combine_merged(mini, first.reshape(1, n, K), opart)
    lead = first.ravel()[np.unique(first.ravel(), return_index=True)[1]]
    gpart = bf16_to_bits(part.view(-1, H).index_select(0, torch.from_numpy(
        trow.ravel()[np.unique(first.ravel(), return_index=True)[1]].astype(np.int64)).to(dev)))
    np.testing.assert_array_equal(gpart, opart.reshape(-1, H)[lead])
    gout = bf16_to_bits(out.view(-1, H).index_select(0, torch.from_numpy(tok).to(dev)))
    np.testing.assert_array_equal(gout, oout[0])
    del y, part, out
    torch.cuda.empty_cache()


def test_error_status_writes_nothing(dev):
    kw = dict(P=2, E=4, K=2, S=16, H=16, R=1)
    zc = zb.Config(**kw)
    ids = np.zeros((2, 16, 2), np.int32)
    ids[1, 3, 1] = 99  # an id outside [0, E)
    p, status, _ = gpu_plan(zc, ids, dev)
    assert status == zb.ERR_BAD_ID
    m = zb.Merge(zc, dev)
    part = torch.full((2, zc.cap, 16), parity.SENTINEL, dtype=torch.int16, device=dev) \
        .view(torch.bfloat16)
    out = torch.full((2, 16, 16), parity.SENTINEL, dtype=torch.int16, device=dev) \
        .view(torch.bfloat16)
    y = torch.zeros((2, zc.cap, 16), dtype=torch.bfloat16, device=dev)
    w = torch.ones((2, 16, 2), dtype=torch.float32, device=dev)
    zb.combine_reduce(p, m, y, w, part)
    zb.combine_merged(p, m, part, out)
    torch.cuda.synchronize()
    assert bool((part.view(torch.int16) == parity.SENTINEL).all())
    assert bool((out.view(torch.int16) == parity.SENTINEL).all())
