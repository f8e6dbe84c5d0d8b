"""A plan whose rows were overwritten after planning (a caller's bug, or memory
gone bad): dispatch, combine and the merged layout skip every row outside
[0, P*cap) and write nothing else.  Under ZB_DEBUG=1 (the bounds-checked
library, libzb_debug.so) the skipped accesses are also recorded, with site,
index and bound, and read back through zb_debug_read.

Everything else in the plan is valid; every receive buffer has slack rows
past P*cap whose sentinel must survive.
"""
import numpy as np
import pytest
import torch

import oracle
import parity
from parity import bf16_to_bits, bits_to_bf16
from token_dispatch_top_b200 import build, zb

pytestmark = pytest.mark.gpu

SLACK = 16


@pytest.fixture(scope="module")
def dev(cuda_device):
    build.build(debug=zb.DEBUG)
    zb.load()
    return cuda_device


def _corrupt_plan(dev):
    rng = np.random.default_rng(17)
    kw = dict(P=4, E=16, K=2, S=64, H=128, R=1, cap_rows=256)
    zc, oc = zb.Config(**kw), oracle.Config(**kw)
    ids = rng.integers(0, 16, (4, 64, 2)).astype(np.int32)
    p = zb.Plan(zc, dev)
    zb.plan(p, torch.from_numpy(ids).to(dev))
    status, _ = zb.plan_status(p)
    assert status == oracle.plan(oc, ids, want_M=False)["status"] >= 0
    if zb.DEBUG:  # planning a valid batch fails no check
        assert zb.debug_read(reset=True)["count"] == 0
    good = p.dst_row.cpu().numpy()
    nrows = zc.P * zc.cap
    bad = {(0, 3, 1): nrows + 3, (2, 10, 0): 1 << 30, (3, 63, 1): -5}
    for (i, s, k), v in bad.items():
        p.dst_row[i, s, k] = v
    return zc, oc, p, good, bad, nrows


def _check_record(site, bad, nrows, count):
    if not zb.DEBUG:
        return
    rec = zb.debug_read(reset=True)
    assert rec["count"] == count, rec
    assert rec["site"] == site and rec["index"] in set(bad.values()) and rec["bound"] == nrows


def test_corrupt_rows_are_skipped_and_recorded(dev):
    zc, oc, p, good, bad, nrows = _corrupt_plan(dev)
    P, S, K, H, cap = zc.P, zc.S, zc.K, zc.H, zc.cap
    rng = np.random.default_rng(18)
    hidden_bits = rng.integers(0, 0x7F00, (P, S, H)).astype(np.uint16)
    buf = torch.full((nrows + SLACK, H), parity.SENTINEL, dtype=torch.int16, device=dev)
    rows = buf[:nrows].view(torch.bfloat16).view(P, cap, H)
    zb.dispatch(p, bits_to_bf16(hidden_bits, dev), rows)
    torch.cuda.synchronize()
    got = buf.cpu().numpy().view(np.uint16)
    assert (got[nrows:] == parity.SENTINEL).all()  # nothing past the buffers
    want = np.full((nrows, H), parity.SENTINEL, np.uint16)
    for i in range(P):
        for s in range(S):
            for k in range(K):
                if (i, s, k) not in bad:
                    want[good[i, s, k]] = hidden_bits[i, s]
    np.testing.assert_array_equal(got[:nrows], want)  # the corrupt entries' rows: untouched
    _check_record("dispatch: row", bad, nrows, len(bad))

    # combine: tokens with a corrupt row keep their output row as it was
    w = rng.dirichlet(np.ones(K), size=(P, S)).astype(np.float32)
    out = torch.full((P, S, H), parity.SENTINEL, dtype=torch.int16, device=dev)
    zb.combine(p, rows, torch.from_numpy(w).to(dev), out.view(torch.bfloat16))
    got_out = bf16_to_bits(out.view(torch.bfloat16))
    ref = oracle.combine(oc, good, got[:nrows], w)
    hit = {(i, s) for (i, s, _k) in bad}
    for i in range(P):
        for s in range(S):
            if (i, s) in hit:
                assert (got_out[i, s] == parity.SENTINEL).all()
            else:
                np.testing.assert_array_equal(got_out[i, s], ref[i, s])
    _check_record("combine: row", bad, nrows, len(bad))


def test_corrupt_rows_in_the_merged_layout(dev):
    zc, oc, p, good, bad, nrows = _corrupt_plan(dev)
    m = zb.Merge(zc, dev)
    zb.merge(p, m)
    torch.cuda.synchronize()
    tok_cnt = m.tok_cnt.cpu().numpy()
    # the merged rows per rank count only the valid entries' (token, rank) pairs
    want = np.zeros(zc.P, np.int64)
    for i in range(zc.P):
        for s in range(zc.S):
            ranks = {good[i, s, k] // zc.cap for k in range(zc.K) if (i, s, k) not in bad}
            for j in ranks:
                want[j] += 1
    np.testing.assert_array_equal(tok_cnt, want)
    # each bad row is refused once counting and once placing
    _check_record("merge: row", bad, nrows, 2 * len(bad))
