"""The multi-rank plumbing of bench.py on CPU with gloo (world size 2).

On this pool each GPU call has one GPU, so ``bench.py --gpus N`` runs N
independent replicas (no data-path collective).  What needs more than one rank
is the timing plumbing: every rank's time is reduced with a max, and the job's
throughput is all ranks' tokens over the slowest rank's time.  These tests run
two gloo ranks as processes on CPU.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        vals = bench.max_over_ranks([10.0 + rank, 5.0 - rank, 7.0], dist, torch.device("cpu"))
        q.put((rank, vals))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got[0] == got[1] == [11.0, 5.0, 7.0]


def test_single_rank_is_identity():
    assert bench.max_over_ranks([1.0, 2.0], None, None) == [1.0, 2.0]


def test_weak_scaling_value():
    # 32768 tokens per rank per step, 10 steps in 4 ms on the slowest rank
    assert bench.weak_scaling_value(32768, 1, 4.0, 10) == pytest.approx(32768 / 0.0004)
    assert bench.weak_scaling_value(32768, 4, 4.0, 10) == pytest.approx(4 * 32768 / 0.0004)


def test_reference_arm_other_ranks_do_nothing(capsys):
    class A:
        steps, warmup, gpus = 1, 0, 2
    from token_dispatch_top_b200 import synth
    assert bench.run_reference(A, synth.WORKLOADS["tiny"], rank=1) is None
    assert capsys.readouterr().out == ""
