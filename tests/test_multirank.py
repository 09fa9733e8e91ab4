"""The N > 1 path of bench.py on CPU: two gloo ranks.

bench.py runs one process per GPU; attention is independent per (batch, head),
so every rank runs its own layer on its own inputs (weak scaling) and the only
collectives are on timing: a barrier around the timed region and the slowest
rank's time (all_reduce MAX).  These tests run that host logic with world size 2
on the gloo backend: distinct inputs per rank, the max over ranks, the whole-job
throughput, and a reference arm that only rank 0 runs.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from workloads import CONFIGS, make_qkv  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = bench.rank_workload(CONFIGS["tiny_sol"], rank, world)
        q, _, _ = make_qkv(w, "cpu")
        dist.barrier()
        ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        slowest = bench.max_over_ranks(ms, dist, "cpu")
        tput = bench.job_throughput(w, world, slowest)
        dist.barrier()
        out.put((rank, w.seed, float(q.float().sum()), slowest, tput))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.SimpleQueue()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    res = sorted(out.get() for _ in range(world))
    (r0, seed0, sum0, slow0, tp0), (r1, seed1, sum1, slow1, tp1) = res
    assert (r0, r1) == (0, 1)
    assert seed0 != seed1 and sum0 != sum1          # each rank draws its own inputs
    assert slow0 == slow1 == 15.0                   # both see the slowest rank's time
    w = CONFIGS["tiny_sol"]
    expect = world * bench.dense_equiv_flops(w) / (15.0e-3) / 1e12
    assert tp0 == pytest.approx(expect) and tp1 == pytest.approx(expect)


def test_single_rank_helpers_are_identities():
    w = CONFIGS["sol_mid"]
    assert bench.rank_workload(w, 0, 1) == w
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
    assert bench.job_throughput(w, 1, 1000.0) == pytest.approx(bench.dense_equiv_flops(w) / 1e12)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    class Args:
        steps, warmup = 1, 0
    bench.run_reference(Args(), CONFIGS["tiny_sol"], rank=1, world=2)
    assert capsys.readouterr().out == ""
