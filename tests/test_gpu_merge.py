"""GPU parity of the merged dispatch layout and scatter against the oracle
(Zepp 4.2 merge: one row per (token, destination rank))."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import parity
from parity import bf16_to_bits, bits_to_bf16, cfgs, gpu_plan
from token_dispatch_top_b200 import build, synth, zb

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")


@pytest.fixture(scope="module")
def dev(cuda_device):
    build.build()
    zb.load()
    return cuda_device


def merge_parity(zc, oc, ids, hidden_bits, dev):
    p, status, _ = gpu_plan(zc, ids, dev, with_row_src=False)
    assert status >= 0
    m = zb.Merge(zc, dev)
    zb.merge(p, m)
    P, cap, H = zc.P, zc.cap, zc.H
    tbuf = torch.full((P, cap, H), parity.SENTINEL, dtype=torch.int16, device=dev) \
        .view(torch.bfloat16)
    zb.dispatch_merged(p, m, bits_to_bf16(hidden_bits, dev), tbuf)
    torch.cuda.synchronize()
    o = oracle.plan(oc, ids, want_M=False)
    om = oracle.merge(oc, o["dst_row"])
    for k in ("tok_row", "grp_tok", "tok_cnt"):
        np.testing.assert_array_equal(getattr(m, k).cpu().numpy(), om[k], err_msg=k)
    ot = np.full((P, cap, H), parity.SENTINEL, np.uint16)
    oracle.dispatch_merged(oc, om["tok_row"], hidden_bits, ot)
    np.testing.assert_array_equal(bf16_to_bits(tbuf), ot)
    return p, m, tbuf


def test_hand_example(dev):
    ex = json.load(open(GOLDEN))["merge_examples"][0]
    d = ex["cfg"]
    kw = dict(P=d["P"], E=d["E"], K=d["K"], S=d["S"], H=d["H"], R=d["R"])
    zc, oc = zb.Config(**kw), oracle.Config(**kw)
    ids = np.array(ex["ids"], np.int32)
    hidden = np.arange(zc.P * zc.S * zc.H, dtype=np.uint16).reshape(zc.P, zc.S, zc.H)
    merge_parity(zc, oc, ids, hidden, dev)


@pytest.mark.parametrize("seed", range(30))
def test_random_small(dev, seed):
    rng = np.random.default_rng(400 + seed)
    P = int(rng.choice([1, 2, 3, 4, 8, 16, 32]))
    Eh = int(rng.integers(1, min(8, 384 // P) + 1))
    K = int(rng.integers(1, 9))
    S = int(rng.integers(0, 600))
    R = int(rng.integers(0, min(P, 3)))
    H = int(rng.choice([8, 64, 264]))
    kw = dict(P=P, E=P * Eh, K=K, S=S, H=H, R=R, cap_rows=max(1, P * S * K))
    zc, oc = zb.Config(**kw), oracle.Config(**kw)
    ids = rng.integers(0, P * Eh, (P, S, K)).astype(np.int32)
    hidden = rng.integers(0, 2 ** 16, (P, S, H), dtype=np.uint32).astype(np.uint16)
    merge_parity(zc, oc, ids, hidden, dev)


def test_mid_full_and_gather(dev):
    """mid workload: everything bit-exact, and the expert-grouped rows the
    plain dispatch writes are the grp_tok-gathers of the merged buffer."""
    wl = synth.WORKLOADS["mid"]
    zc, oc = cfgs(wl)
    ids, _ = synth.routing(wl, 0)
    hidden = synth.hidden_bits(wl, 0)
    p, m, tbuf = merge_parity(zc, oc, ids, hidden, dev)
    buf = torch.empty_like(tbuf)
    zb.dispatch(p, bits_to_bf16(hidden, dev), buf)
    gt = m.grp_tok.view(-1)
    used = gt >= 0
    flat_t = tbuf.view(-1, zc.H).view(torch.int16)
    flat_b = buf.view(-1, zc.H).view(torch.int16)
    assert torch.equal(flat_t[gt[used].long()], flat_b[used])
    assert int(m.tok_cnt.sum()) < zc.P * zc.S * zc.K  # the merge saved rows


def test_hot_full_size_gather(dev):
    wl = synth.WORKLOADS["hot"]
    zc, oc = cfgs(wl, cap_rows=2 * wl.S * wl.K)
    ids, _ = synth.routing(wl, 0)
    p, status, _ = gpu_plan(zc, ids, dev, with_row_src=False)
    m = zb.Merge(zc, dev)
    zb.merge(p, m)
    o = oracle.plan(oc, ids, want_M=False)
    om = oracle.merge(oc, o["dst_row"])
    for k in ("tok_row", "grp_tok", "tok_cnt"):
        np.testing.assert_array_equal(getattr(m, k).cpu().numpy(), om[k], err_msg=k)
    hid = synth.hidden_device(wl, 0, 0, dev)
    tbuf = torch.empty((zc.P, zc.cap, zc.H), dtype=torch.bfloat16, device=dev)
    zb.dispatch_merged(p, m, hid, tbuf)
    rng = np.random.default_rng(1)
    ent = torch.from_numpy(rng.integers(0, zc.P * zc.S * zc.K, 2048)).to(dev)
    tok = ent // zc.K
    rows = m.tok_row.view(-1)[ent].long()
    got = tbuf.view(-1, zc.H).index_select(0, rows).view(torch.int16)
    want = hid.view(-1, zc.H).index_select(0, tok).view(torch.int16)
    assert torch.equal(got, want)
    del tbuf, hid
    torch.cuda.empty_cache()
