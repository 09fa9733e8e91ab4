"""The N > 1 path of bench.py on CPU: two gloo ranks.

bench.py runs one process per GPU.  Attention is independent per (batch, head),
so by default the ranks share one layer's heads (--split heads: rank r takes a
contiguous head range, reads a strided view of the layer's Q/K/V, and no data
crosses between ranks), or each runs a whole layer on its own inputs (--split
replicas).  The only collectives are on timing: a barrier around the timed
region and the slowest rank's time (all_reduce MAX).  These tests run that host
logic with world size 2 on the gloo backend: the head ranges tile [0, H), the
two ranks' oracle outputs on their views put together equal the single-rank
output of the whole layer, distinct inputs per replica, the max over ranks,
the whole-job throughput, and a reference arm that only rank 0 runs.
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
        launches = bench.sum_over_ranks(100 + rank, dist, "cpu")
        dist.barrier()
        out.put((rank, w.seed, float(q.float().sum()), slowest, tput, launches))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.SimpleQueue()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    res = sorted(out.get() for _ in range(world))
    (r0, seed0, sum0, slow0, tp0, n0), (r1, seed1, sum1, slow1, tp1, n1) = res
    assert (r0, r1) == (0, 1)
    assert seed0 != seed1 and sum0 != sum1          # each rank draws its own inputs
    assert slow0 == slow1 == 15.0                   # both see the slowest rank's time
    assert n0 == n1 == 201                          # launch counts add up over the job
    w = CONFIGS["tiny_sol"]
    expect = world * bench.dense_equiv_flops(w) / (15.0e-3) / 1e12
    assert tp0 == pytest.approx(expect) and tp1 == pytest.approx(expect)


def _heads_rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import numpy as np

    import oracle
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = HEADS_CASE
        h0, h1 = bench.head_range(w.H, rank, world)
        q, k, v = make_qkv(w, "cpu")                      # the same layer on every rank
        qs, ks, vs = (t[:, :, h0:h1] for t in (q, k, v))  # this rank's heads, strided view
        wr = w.replace(H=h1 - h0)
        raw = [oracle.as_raw(t) for t in (qs, ks, vs)]
        res = oracle.routing(wr, *raw)
        o, lse = oracle.layer_rows(wr, *raw, res, oracle.all_tokens(wr))
        slowest = bench.max_over_ranks(4.0 + rank, dist, "cpu")
        out.put((rank, h0, h1, o.reshape(wr.H, w.N, w.d), lse.reshape(wr.H, w.N), slowest,
                 bench.job_throughput(w, world, slowest, "heads")))
    finally:
        dist.destroy_process_group()


HEADS_CASE = CONFIGS["tiny_sol"].replace(name="heads_split", H=5, N=640)


def test_two_gloo_ranks_head_split_tiles_the_layer():
    import numpy as np

    import oracle
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.SimpleQueue()
    procs = mp.start_processes(_heads_rank_main, args=(world, _free_port(), out), nprocs=world, join=False,
                               start_method="spawn")
    # read before joining: a rank blocks in put() until its (large) result is taken
    res = sorted((out.get() for _ in range(world)), key=lambda r: r[0])
    while not procs.join(timeout=60):
        pass
    w = HEADS_CASE
    assert [(r[1], r[2]) for r in res] == [(0, 3), (3, 5)]          # contiguous, covering [0, H)
    q, k, v = make_qkv(w, "cpu")
    raw = [oracle.as_raw(t) for t in (q, k, v)]
    full = oracle.routing(w, *raw)
    o, lse = oracle.layer_rows(w, *raw, full, oracle.all_tokens(w))
    got_o = np.concatenate([r[3] for r in res], axis=0)
    got_l = np.concatenate([r[4] for r in res], axis=0)
    assert np.array_equal(got_o, o.reshape(w.H, w.N, w.d))
    assert np.array_equal(got_l, lse.reshape(w.H, w.N))
    assert res[0][5] == res[1][5] == 5.0
    # strong scaling: the job is one layer, whatever the rank count
    assert res[0][6] == pytest.approx(bench.dense_equiv_flops(w) / 5.0e-3 / 1e12)


def test_head_range_balance():
    for H in (1, 5, 40):
        for world in range(1, min(H, 8) + 1):
            rs = [bench.head_range(H, r, world) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
            sizes = [b - a for a, b in rs]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        bench.head_range(2, 0, 3)


def test_single_rank_helpers_are_identities():
    w = CONFIGS["sol_mid"]
    assert bench.rank_workload(w, 0, 1) == w
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
    assert bench.sum_over_ranks(7, None, "cpu") == 7
    assert bench.job_throughput(w, 1, 1000.0) == pytest.approx(bench.dense_equiv_flops(w) / 1e12)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    class Args:
        steps, warmup = 1, 0
    bench.run_reference(Args(), CONFIGS["tiny_sol"], rank=1, world=2)
    assert capsys.readouterr().out == ""
