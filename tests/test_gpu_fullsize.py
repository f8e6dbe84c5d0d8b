"""Full-size parity on the hot, hier and drift workloads: every element.

The plan tables, dst_row and row_src are compared whole.  Every (token, k)
row of the receive buffer is compared with the oracle's dispatch, every row
past a rank's load must still hold the sentinel, and both combined outputs
(y = the dispatched rows, and y = independent seeded rows, which runs the
32-byte combine kernel at K = 8, H = 7168 on every token) are compared bit
for bit with the oracle's combine.

The oracle runs on blocks of tokens so that host memory stays bounded: for a
block, the device gathers the rows the oracle's dst_row names, and the
oracle's dispatch and combine run on exactly those rows (a block is a
one-rank problem whose rows are numbered in (token, k) order).  Its combine
is about 3.8 G fused multiply-adds per output on hot and hier and 7.5 G per
drift step; the blocks run on the host's cores in threads (the oracle is
plain C called through ctypes, which releases the interpreter lock), so this
file takes about a minute on an 8-core host.
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
import parity
from parity import assert_plan_equal, bf16_to_bits, cfgs, gpu_plan, plan_tables
from token_dispatch_top_b200 import build, synth, zb

pytestmark = pytest.mark.gpu

BLOCK = 1024  # tokens per oracle call


@pytest.fixture(scope="module")
def dev(cuda_device):
    build.build()
    zb.load()
    return cuda_device


def _threads() -> int:
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(16, n))


def _block_cfg(n: int, K: int, H: int) -> oracle.Config:
    """A one-rank problem of n tokens whose K rows each are numbered t*K + k."""
    return oracle.Config(P=1, E=1, K=K, S=n, H=H, R=0, cap_rows=max(1, n * K))


def _local_rows(n: int, K: int) -> np.ndarray:
    return np.arange(n * K, dtype=np.int32).reshape(1, n, K)


def check_dispatch(zc, o, hidden_d, buf, dev):
    """buf[dst_row[t, k]] against the oracle's dispatch of token t, for every
    (t, k); rows past each rank's load still hold the sentinel."""
    P, S, K, H, cap = zc.P, zc.S, zc.K, zc.H, zc.cap
    ntok = P * S
    dst = o["dst_row"].reshape(ntok, K)
    hid = bf16_to_bits(hidden_d).reshape(ntok, H)
    flat = buf.view(P * cap, H)
    for t0 in range(0, ntok, BLOCK):
        t1 = min(ntok, t0 + BLOCK)
        n = t1 - t0
        want = oracle.dispatch(_block_cfg(n, K, H), _local_rows(n, K), hid[t0:t1])
        rows = torch.from_numpy(dst[t0:t1].ravel().astype(np.int64)).to(dev)
        got = bf16_to_bits(flat.index_select(0, rows))
        np.testing.assert_array_equal(got, want.reshape(n * K, H),
                                      err_msg=f"dispatch, tokens {t0}..{t1}")
    for j in range(P):
        la = int(o["load_after"][j])
        tail = flat[j * cap + la:(j + 1) * cap].view(torch.int16)
        assert bool((tail == parity.SENTINEL).all()), f"rank {j}: a row past the load was written"


def check_combine(zc, o, y, w, out, dev, pool):
    """out[t] against the oracle's combine of the K rows y[dst_row[t, :]] with
    the gates w[t, :], for every token t."""
    P, S, K, H, cap = zc.P, zc.S, zc.K, zc.H, zc.cap
    ntok = P * S
    dst = o["dst_row"].reshape(ntok, K)
    wf = np.ascontiguousarray(w.reshape(ntok, K))
    flat_y = y.view(P * cap, H)
    flat_out = out.view(ntok, H)
    limit = 2 * pool._max_workers

    def oracle_block(t0, t1, yk):
        n = t1 - t0
        return oracle.combine(_block_cfg(n, K, H), _local_rows(n, K), yk,
                              wf[t0:t1].reshape(1, n, K))[0]

    pending = []

    def drain(keep):
        while len(pending) > keep:
            fut, got, t0 = pending.pop(0)
            np.testing.assert_array_equal(got, fut.result(),
                                          err_msg=f"combine, tokens {t0}..{t0 + len(got)}")

    for t0 in range(0, ntok, BLOCK):
        t1 = min(ntok, t0 + BLOCK)
        rows = torch.from_numpy(dst[t0:t1].ravel().astype(np.int64)).to(dev)
        yk = bf16_to_bits(flat_y.index_select(0, rows))
        got = bf16_to_bits(flat_out[t0:t1])
        pending.append((pool.submit(oracle_block, t0, t1, yk), got, t0))
        drain(limit)
    drain(0)


def full_size_parity(wl, seed, step, dev):
    zc, oc = cfgs(wl, cap_rows=2 * wl.S * wl.K)
    P, S, H, cap = zc.P, zc.S, zc.H, zc.cap
    ids, w = synth.routing(wl, seed, step)
    p, status, _ = gpu_plan(zc, ids, dev, with_row_src=True)
    o = oracle.plan(oc, ids, want_M=False)
    assert_plan_equal(plan_tables(p), o, status)
    assert status in (oracle.OK, oracle.UNBALANCED)

    hidden = synth.hidden_device(wl, seed, step, dev)
    buf = torch.full((P, cap, H), parity.SENTINEL, dtype=torch.int16, device=dev) \
        .view(torch.bfloat16)
    zb.dispatch(p, hidden, buf)
    w_d = torch.from_numpy(np.ascontiguousarray(w)).to(dev)
    out = torch.empty((P, S, H), dtype=torch.bfloat16, device=dev)
    zb.combine(p, buf, w_d, out)
    torch.cuda.synchronize()
    with ThreadPoolExecutor(max_workers=_threads()) as pool:
        check_dispatch(zc, o, hidden, buf, dev)
        check_combine(zc, o, buf, w, out, dev, pool)   # y = the dispatched rows
        del buf
        gen = torch.Generator(device=dev)
        gen.manual_seed(77 + 1000 * seed + step)
        y = torch.randn((P, cap, H), generator=gen, device=dev, dtype=torch.bfloat16)
        zb.combine(p, y, w_d, out)
        torch.cuda.synchronize()
        check_combine(zc, o, y, w, out, dev, pool)     # independent expert outputs
    del y, out, hidden, p
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["hot", "hier"])
def test_full_size_every_element(dev, name):
    full_size_parity(synth.WORKLOADS[name], 0, 0, dev)


@pytest.mark.parametrize("step", [0, 31, 63])
def test_drift_step_every_element(dev, step):
    full_size_parity(synth.WORKLOADS["drift"], 0, step, dev)
