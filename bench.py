"""Benchmark: one layer of block-sparse "sol-attn" attention per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
                    [--split heads|replicas] [--impl reference]

A step is the whole hot path on one batch of synthetic inputs already resident
in HBM: bsa_pool -> bsa_select -> bsa_attention (sparse + centroid + dense
rows), the last as bsa_attention_prepare + bsa_attention_run so that the fine
pass kernel is timed alone.  Rank 0 prints one JSON line.  Metric:
sparse-attention ms per layer and dense-equivalent TFLOP/s (4*B*H*N^2*d /
layer time).  The roofline block reports the fine pass (bsa_attention_run)
against the measured bf16 tensor peak on the FLOPs it really has to do (kept
FLOPs, counted from the CSR of the run); roofline_select reports pooling and
selection against the measured HBM copy bandwidth.

Multi-GPU (torchrun): attention is independent per (batch, head).  The default
split gives each of the N ranks a contiguous range of the same layer's heads
(strong scaling: the job is one layer, no collective on the data path; the
step time is the max over ranks).  --split replicas runs one whole layer per
rank on its own inputs instead (weak scaling).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import CONFIGS, make_qkv  # noqa: E402

DEFAULT_CONFIG = "long"
METRIC = "sparse-attn ms/layer & dense-equiv TFLOP/s at N tokens; % roofline (kept FLOPs)"
UNIT = "TFLOP/s (dense-equivalent)"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def attn_traffic(w):
    """DRAM bytes per fine-pass launch from the committed ncu capture of this
    workload (a few heads, scaled to all heads), or None when the kernel source
    changed since the capture or no capture covers the workload."""
    import hashlib
    try:
        recs = json.load(open(os.path.join(ROOT, "profiles", "attn_traffic.json")))
    except (OSError, ValueError):
        return None
    for rec in recs.get("captures", []):
        if rec.get("workload") != w.name or int(rec.get("heads_full", -1)) != w.H:
            continue
        try:
            src = open(os.path.join(ROOT, rec["source"]), "rb").read()
        except (OSError, KeyError):
            return None
        if hashlib.sha256(src).hexdigest() != rec.get("source_sha256"):
            return None
        return float(rec["dram_bytes_per_launch"])
    return None


def rank_workload(w, rank: int, world: int):
    """--split replicas: every rank runs its own layer of the same shape on its
    own inputs (heads are independent; no collective on the data path)."""
    return w.replace(seed=w.seed + 17 * rank) if world > 1 else w


def head_range(H: int, rank: int, world: int):
    """--split heads: rank's contiguous share [h0, h1) of the layer's H heads
    (the first H % world ranks take one head more)."""
    if world > H:
        raise ValueError(f"{world} ranks for {H} heads: every rank needs at least one head")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, pg, device) -> float:
    """The job's time is the slowest rank's (all_reduce MAX); identity on one rank."""
    if pg is None:
        return float(value)
    t = torch.tensor([float(value)], device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t)


def sum_over_ranks(value: int, pg, device) -> int:
    """A count over the whole job (all_reduce SUM); identity on one rank."""
    if pg is None:
        return int(value)
    t = torch.tensor([int(value)], dtype=torch.int64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.SUM)
    return int(t)


def job_throughput(w, world: int, ms_per_step: float, split: str = "replicas") -> float:
    """Whole-job dense-equivalent TFLOP/s over the slowest rank's time: all
    ranks' layers (replicas), or the one layer whose heads the ranks share."""
    layers = world if split == "replicas" else 1
    return layers * dense_equiv_flops(w) / (ms_per_step * 1e-3) / 1e12


def pool_bytes(w) -> float:
    """Algorithmic HBM bytes of bsa_pool: Q, K and V read once, the f32 means
    and the block sizes written once."""
    s_in = 2 if w.dtype == "bf16" else 4
    read = 3.0 * w.B * w.N * w.H * w.d * s_in
    write = (w.nQB + 2 * w.nKB) * w.B * w.H * w.d * 4 + 4 * w.nKB
    return read + write


def select_flops(w) -> float:
    """Block-score FLOPs of bsa_select: 2*d per (row, key block)."""
    return 2.0 * w.rows * w.nKB * w.d


def dense_equiv_flops(w) -> float:
    return 4.0 * w.B * w.H * float(w.N) * w.N * w.d


def kept_flops(w, row_ptr: torch.Tensor, col: torch.Tensor, extra_count=None) -> float:
    """FLOPs of the fine pass actually required: 4*d per (query row, key) pair over
    the exact keys (kept blocks and extra tokens) and centroids of every sparse
    row, plus 4*d*N per dense row.  A block that gave extra tokens still counts
    one (modified) centroid; the rare block whose every token became an extra
    token is counted too (an overcount below 1 %)."""
    rp = row_ptr.to(torch.int64)
    cnt = (rp[1:] - rp[:-1]).view(w.B, w.H, w.nQB)
    nnz = int(rp[-1])
    c = col[:nnz].to(torch.int64)
    last_n = w.N - (w.nKB - 1) * w.k_block
    # exact keys per row: kept blocks x 64, minus the short last block where kept
    row_of = torch.repeat_interleave(torch.arange(cnt.numel(), device=c.device), cnt.reshape(-1))
    short = torch.zeros(cnt.numel(), dtype=torch.int64, device=c.device)
    short.index_add_(0, row_of, (c == w.nKB - 1).to(torch.int64))
    exact_keys = cnt.reshape(-1) * w.k_block - short * (w.k_block - last_n)
    if extra_count is not None:
        exact_keys = exact_keys + extra_count.to(torch.int64).reshape(-1)
    cent = (w.nKB - cnt.reshape(-1)) if w.centroid else torch.zeros_like(exact_keys)
    per_row_keys = (exact_keys + cent).view(w.B, w.H, w.nQB).double()
    # query rows per query block (the last one may be short)
    qrows = torch.full((w.nQB,), float(w.q_block), dtype=torch.float64, device=c.device)
    qrows[-1] = w.N - (w.nQB - 1) * w.q_block
    r0, r1 = w.dense_rows
    if r1 > r0:
        # rows in the dense range are computed by the dense pass instead
        for i in range(w.nQB):
            lo, hi = i * w.q_block, min(w.N, (i + 1) * w.q_block)
            ov = max(0, min(hi, r1) - max(lo, r0))
            qrows[i] -= ov
    sparse = float((per_row_keys * qrows.view(1, 1, -1)).sum())
    dense = float(w.B * w.H * (r1 - r0) * w.N) if r1 > r0 else 0.0
    return 4.0 * w.d * (sparse + dense)


def issued_flops(w, row_ptr: torch.Tensor, col: torch.Tensor, extra_count=None) -> float:
    """Tensor-core FLOPs the fine pass issues: every 128-key tile costs
    4 * 128 * 128 * d (S = Q K^T and P V at M = 128), whatever its masks.  A sparse
    item (128 query rows: two 64-row query blocks, or one 128-row block) runs
    ceil(|union of its blocks' kept key blocks| / 2) exact tiles, ceil(ceil(nKB /
    64) / 2) centroid tiles with centroids, and with extra tokens at least
    ceil(their count / 128) gathered tiles (both blocks' lists counted in full;
    the modified centroids beside them are left out); items whose rows all lie in
    the dense range are skipped; the dense rows' 128-row tiles each run
    ceil(nKB / 2) tiles.  Against kept_flops this is the pairing's overwork."""
    rp = row_ptr.to(torch.int64)
    rows = w.B * w.H * w.nQB
    nnz = int(rp[-1])
    cnt = rp[1:] - rp[:-1]
    row_of = torch.repeat_interleave(torch.arange(rows, device=col.device), cnt)
    mask = torch.zeros((rows, w.nKB), dtype=torch.bool, device=col.device)
    mask[row_of, col[:nnz].to(torch.int64)] = True
    mask = mask.view(w.B * w.H, w.nQB, w.nKB)
    per = 128 // w.q_block                        # query blocks per item
    n_items = -(-w.N // 128)
    if w.nQB % per:
        mask = torch.cat([mask, torch.zeros((w.B * w.H, per - w.nQB % per, w.nKB), dtype=torch.bool,
                                              device=mask.device)], 1)
    union = mask.view(w.B * w.H, n_items, per, w.nKB).any(2).sum(2)          # [BH, items]
    tiles = (union + 1) // 2
    if w.centroid:
        tiles = tiles + (-(-w.nKB // 64) + 1) // 2
    if extra_count is not None and w.extra_tokens > 0:
        ec = extra_count.to(torch.int64).view(w.B * w.H, w.nQB)
        if w.nQB % per:
            ec = torch.cat([ec, torch.zeros((w.B * w.H, per - w.nQB % per), dtype=torch.int64, device=ec.device)], 1)
        tiles = tiles + (ec.view(w.B * w.H, n_items, per).sum(2) + 127) // 128
    r0, r1 = w.dense_rows
    live = torch.ones(n_items, dtype=torch.bool, device=tiles.device)
    if r1 > r0:
        for it in range(n_items):
            if it * 128 >= r0 and min(it * 128 + 128, w.N) <= r1:
                live[it] = False
    total = int((tiles * live.view(1, -1)).sum())
    if r1 > r0:
        total += w.B * w.H * (-(-(r1 - r0) // 128)) * ((w.nKB + 1) // 2)
    return 4.0 * 128 * 128 * w.d * total


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        except OSError:
            pass
        finally:
            try:
                os.unlink(self.path)
            except OSError:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}

        def mhz(s):
            try:
                return float(s.split()[0])
            except (ValueError, IndexError):
                return None
        sm = [mhz(r[1]) for r in rows if mhz(r[1]) is not None]
        smax = max((mhz(r[2]) for r in rows if mhz(r[2]) is not None), default=None)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [x for x in sm if smax and x > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": reasons, "samples": len(rows)}


def cpu_baseline(w, q, k, v, budget_s: float = 20.0):
    """The CPU oracle, as it stands, on a bounded sample of the workload.

    Sample: one head (b=0, h=0): pooling of Q, K and V, block scores and
    selection for all of that head's query blocks, then exact/centroid attention
    for a seeded sample of that head's query rows.  The layer time is
    extrapolated: H*B x (pool + select of one head) + (B*H*N / rows) x attention.
    """
    import numpy as np

    import oracle

    w1 = w.replace(B=1, H=1)
    qc, kc, vc = (t[:1, :, :1].cpu() for t in (q, k, v))
    qr, kr, vr = oracle.as_raw(qc), oracle.as_raw(kc), oracle.as_raw(vc)
    t0 = time.perf_counter()
    res = oracle.routing(w1, qr, kr, vr, extra_rows=[], with_extra=False)
    t_route = time.perf_counter() - t0
    t_extra = 0.0
    n_extra = 0
    if w.extra_tokens > 0:
        rows = list(range(0, w1.nQB, max(1, w1.nQB // 8)))[:8]
        t0 = time.perf_counter()
        ex, ec, rr = oracle.extra_tokens(res.qbar, kr, res.keep, w.q_block, w.k_block, w.extra_tokens, rows)
        t_extra = time.perf_counter() - t0
        n_extra = len(rows)
        res.extra = np.full((w1.rows, w.extra_tokens), -1, np.int32)
        res.ecnt = np.zeros((w1.rows,), np.int32)
        res.extra[rr] = ex
        res.ecnt[rr] = ec
    # attention rows: grow the sample until about a quarter of the budget is used
    g = np.random.default_rng(0)
    m = 64
    t_attn, done = 0.0, 0
    while True:
        toks = np.stack([np.zeros(m, np.int64), np.zeros(m, np.int64),
                         g.integers(0, w.N, m).astype(np.int64)], axis=1)
        if w.extra_tokens > 0:
            # keep to query blocks whose extra tokens were computed
            allowed = np.array(sorted(set(int(r) for r in range(0, w1.nQB, max(1, w1.nQB // 8)))))[:8]
            toks[:, 2] = (allowed[g.integers(0, len(allowed), m)] * w.q_block +
                          g.integers(0, w.q_block, m)).clip(max=w.N - 1)
        t0 = time.perf_counter()
        oracle.layer_rows(w1, qr, kr, vr, res, toks)
        t_attn += time.perf_counter() - t0
        done += m
        if t_attn > budget_s / 4 or done >= 65536:
            break
        m *= 2
    per_row = t_attn / done
    layer_s = w.B * w.H * (t_route + (t_extra / max(n_extra, 1)) * w1.nQB) + w.B * w.H * w.N * per_row
    sample = (f"1 head of {w.B * w.H}: pool + select of all {w1.nQB} query blocks "
              f"({t_route:.2f} s), attention for {done} sampled query rows ({t_attn:.2f} s)"
              + (f", extra tokens for {n_extra} query blocks ({t_extra:.2f} s)" if n_extra else "")
              + "; layer time extrapolated linearly")
    return {"value": dense_equiv_flops(w) / layer_s / 1e12, "unit": UNIT, "cores": oracle.threads(),
            "kind": "oracle", "sample": sample, "layer_s_extrapolated": layer_s}


def run_reference(args, w, rank, world):
    """--impl reference: the CPU oracle timed as it stands (rank 0 only)."""
    if rank != 0:
        return
    dev = "cpu"
    q, k, v = make_qkv(w.replace(B=1, H=1), dev)
    per_step = []
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(w, q, k, v, budget_s=max(4.0, 60.0 / (args.warmup + args.steps)))
        if i >= args.warmup:
            per_step.append(cb["layer_s_extrapolated"])
    layer_s = statistics.median(per_step)
    val = dense_equiv_flops(w) / layer_s / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": layer_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": _config_json(w, world, "heads" if world > 1 else "replicas", [0, w.H]),
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": cb["cores"], "kind": "oracle",
                             "sample": cb["sample"]},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _config_json(w, world, split="replicas", heads=None):
    par = (f"heads split over {world} ranks (ranges {heads}; no collective)" if split == "heads" and world > 1
           else f"replicas x{world} (heads independent, no collective)")
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "dtype": w.dtype,
            "method": w.method, "q_block": w.q_block, "k_block": w.k_block,
            "tau": w.tau if w.method == "sol" else None,
            "keep_percent": w.keep_percent if w.method == "sla" else None,
            "prefix_len": w.prefix_len, "dense_rows": list(w.dense_rows), "extra_tokens": w.extra_tokens,
            "centroid": w.centroid, "grid": list(w.grid) if w.grid else None,
            "qk_fp8": bool(getattr(w, "qk_fp8", False)),
            "pv_fp8": bool(getattr(w, "pv_fp8", False)),
            "parallelism": par,
            "l2": "inputs larger than L2 (126 MB); no flush" if 3 * w.B * w.N * w.H * w.d * 2 > 126e6
            else "L2 flushed between steps"}


def run_producer(args, w, dev):
    """--producer: the QKV projection with pooling in its epilogue
    (bsa_qkv_pool) against the same work unfused: cuBLAS (torch.matmul) for
    X W^T, then bsa_pool reading Q, K and V back.  d_model = H * d."""
    import block_sparse_attention_26_b200 as bsa
    dm = w.H * w.d
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed + 9)
    x = torch.randn((w.B, w.N, dm), generator=g, device=dev).to(torch.bfloat16)
    W = (torch.randn((3 * w.H * w.d, dm), generator=g, device=dev) / dm ** 0.5).to(torch.bfloat16)
    q, k, v = (torch.empty((w.B, w.N, w.H, w.d), dtype=torch.bfloat16, device=dev) for _ in range(3))
    p = bsa.params_for(w, q)
    nQB, nKB, _ = bsa.dims(p)
    qbar = torch.empty((w.B, w.H, nQB, w.d), dtype=torch.float32, device=dev)
    kbar = torch.empty((w.B, w.H, nKB, w.d), dtype=torch.float32, device=dev)
    vbar = torch.empty_like(kbar)
    cnt = torch.empty((nKB,), dtype=torch.int32, device=dev)
    ws = torch.zeros(4096, dtype=torch.uint8, device=dev)
    y = torch.empty((w.B, w.N, 3, w.H, w.d), dtype=torch.bfloat16, device=dev)
    yq, yk, yv = y[:, :, 0], y[:, :, 1], y[:, :, 2]
    py = bsa.params_for(w, yq)
    stream = torch.cuda.current_stream(dev)

    def fused():
        bsa.bsa_qkv_pool(p, x, W, q, k, v, qbar, kbar, vbar, cnt, ws, stream)

    def unfused(ev=None):
        torch.matmul(x, W.t(), out=y.view(w.B, w.N, 3 * w.H * w.d))
        if ev:
            ev.record(stream)
        bsa.bsa_pool(py, yq, yk, yv, qbar, kbar, vbar, cnt, stream)

    def timed(fn, mid=False):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        em = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        e0.record(stream)
        for i in range(args.steps):
            starts[i].record(stream)
            fn(em[i]) if mid else fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        total = e0.elapsed_time(e1) / args.steps
        part = statistics.mean(s.elapsed_time(m) for s, m in zip(starts, em)) if mid else None
        return total, part

    with ClockSampler(int(str(dev).split(":")[-1]) if ":" in str(dev) else 0) as clocks:
        t_fused, _ = timed(fused)
        t_unf, t_gemm = timed(unfused, mid=True)
    assert bsa.bsa_device_status(ws) == 0
    flop = 2.0 * w.B * w.N * dm * 3 * w.H * w.d
    peaks, src = _peaks()
    line = {"metric": "qkv projection + pooling ms (producer)", "workload": w.name, "d_model": dm,
            "fused_ms": t_fused, "unfused_ms": t_unf, "unfused_gemm_ms": t_gemm, "unfused_pool_ms": t_unf - t_gemm,
            "fused_tflops": flop / (t_fused * 1e-3) / 1e12, "cublas_tflops": flop / (t_gemm * 1e-3) / 1e12,
            "fused_frac_of_bf16_peak": flop / (t_fused * 1e-3) / 1e12 / float(peaks["bf16_tflops"]),
            "peak_source": f"{src} bf16_tflops", "steps": args.steps, "warmup": args.warmup,
            "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--split", default="heads", choices=["heads", "replicas"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--heads", type=int, default=0, help="override H (profiling a smaller case)")
    ap.add_argument("--qk-fp8", action="store_true", help="fine pass with S = Q K^T in fp8 (e4m3)")
    ap.add_argument("--pv-fp8", action="store_true", help="with --qk-fp8: P V in fp8 (e4m3) as well")
    ap.add_argument("--producer", action="store_true",
                    help="time the QKV projection with pooling in its epilogue against cuBLAS + bsa_pool")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w_job = CONFIGS[args.config]
    if args.heads > 0:
        w_job = w_job.replace(H=args.heads)
    if args.qk_fp8:
        w_job = w_job.replace(qk_fp8=True, pv_fp8=bool(args.pv_fp8))
    elif args.pv_fp8:
        raise SystemExit("--pv-fp8 needs --qk-fp8")
    split = args.split if world > 1 else "replicas"
    if split == "replicas":
        w_job = rank_workload(w_job, rank, world)
        h0, h1 = 0, w_job.H
    else:
        h0, h1 = head_range(w_job.H, rank, world)
    w = w_job.replace(H=h1 - h0)              # this rank's share of the work

    if args.impl == "reference":
        run_reference(args, w_job, rank, world)
        return

    import block_sparse_attention_26_b200 as bsa
    from block_sparse_attention_26_b200 import params_for

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.producer:
        run_producer(args, w, dev)
        return
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist

    qf, kf, vf = make_qkv(w_job, dev)
    # this rank's heads: a strided view of the layer's tensors (same strides)
    q, k, v = (t[:, :, h0:h1] for t in (qf, kf, vf))
    p = params_for(w, q)
    buf = bsa.Buffers(p, dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)
    l2_flush = None
    if 3 * q.numel() * q.element_size() <= 126e6:
        l2_flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def step(ev=None):
        if l2_flush is not None:
            l2_flush.zero_()
        if ev:
            ev[0].record(stream)
        bsa.bsa_pool(p, q, k, v, buf.qbar, buf.kbar, buf.vbar, buf.blk_count, stream)
        if ev:
            ev[1].record(stream)
        bsa.bsa_select(p, buf.qbar, buf.kbar, k, buf.row_ptr, buf.col_idx, buf.kept_count, buf.extra_idx,
                       buf.extra_count, buf.ws, stream)
        if ev:
            ev[2].record(stream)
        att = (p, q, k, v, buf.kbar, buf.vbar, buf.blk_count, buf.row_ptr, buf.col_idx, buf.extra_idx,
               buf.extra_count, out, buf.lse, buf.ws, stream)
        bsa.bsa_attention_prepare(*att)
        if ev:
            ev[3].record(stream)
        bsa.bsa_attention_run(*att)
        if ev:
            ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    status = bsa.bsa_device_status(buf.ws, stream)
    if status != 0:
        raise SystemExit(f"device status {status} after warm-up")
    flops_kept = kept_flops(w, buf.row_ptr, buf.col_idx, buf.extra_count)
    flops_issued = issued_flops(w, buf.row_ptr, buf.col_idx, buf.extra_count)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        launches0 = bsa.bsa_launch_count()
        start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        stop.record(stream)
        torch.cuda.synchronize(dev)
        launches = bsa.bsa_launch_count() - launches0   # the library's own kernels, as it counted them
    if pg:
        pg.barrier()
    total_ms = max_over_ranks(start.elapsed_time(stop), pg, dev)
    launches = sum_over_ranks(launches, pg, dev)
    status = bsa.bsa_device_status(buf.ws, stream)
    if status != 0:
        raise SystemExit(f"device status {status} after the timed steps")
    names = ["pool", "select", "attention_prepare", "attention_fine_pass"]
    ph = {n: [e[i].elapsed_time(e[i + 1]) for e in evs] for i, n in enumerate(names)}
    ph_ms = {n: statistics.mean(x) for n, x in ph.items()}
    ph_ms["attention"] = ph_ms["attention_prepare"] + ph_ms["attention_fine_pass"]
    ms_step = total_ms / args.steps

    # end to end through the public API with host buffers: every step, H2D of this
    # rank's Q/K/V heads, the layer, D2H of the output -- bsa_layer_host, which
    # takes the heads in chunks so that one chunk's copies overlap another's kernels
    e2e = None
    if args.e2e_steps > 0:
        hq, hk, hv = (t.contiguous().cpu().pin_memory() for t in (q, k, v))
        hout = torch.empty(hq.shape, dtype=hq.dtype, pin_memory=True)
        pe = params_for(w, hq)
        hl = bsa.HostLayer(pe, dev)
        cin, cout = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if pg:
            pg.barrier()
        for i in range(args.e2e_steps + 1):
            if i == 1:
                torch.cuda.synchronize(dev)
                s0.record(stream)
            bsa.bsa_layer_host(pe, hq, hk, hv, hout, hl, stream, cin, cout)
        s1.record(stream)   # the call leaves `stream` waiting for its last copy back
        torch.cuda.synchronize(dev)
        if bsa.bsa_device_status(hl.buf.ws, stream) != 0:
            raise SystemExit("device status after the end-to-end steps")
        e2e_ms = max_over_ranks(s0.elapsed_time(s1) / args.e2e_steps, pg, dev)
        nbytes = q.numel() * q.element_size()
        e2e = {"value": job_throughput(w_job, world, e2e_ms, split), "unit": UNIT,
               "h2d_bytes_per_step": 3 * nbytes, "d2h_bytes_per_step": nbytes, "ms_per_step": e2e_ms,
               "heads_per_chunk": hl.hc}
        dq = dk = dv = None
        del hq, hk, hv, hout, dq, dk, dv, hl

    peaks, peak_src = _peaks()
    # the fine pass's own dtype: half its FLOP (S = Q K^T) at the fp8 rate with
    # qk_fp8, all of it with pv_fp8 too; fp8 runs at twice the dense bf16 rate
    # (nominal 4.5 against 2.25 PFLOP/s), applied to the measured bf16 peak
    ratio = 2.0 if w.pv_fp8 else (4.0 / 3.0 if w.qk_fp8 else 1.0)
    peak = float(peaks.get("bf16_tflops")) * ratio
    peak_sus = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))) * ratio
    hbm = float(peaks.get("hbm_gbs"))
    fine_ms = ph_ms["attention_fine_pass"]
    achieved = flops_kept / (fine_ms * 1e-3) / 1e12
    pool_gbs = pool_bytes(w) / (ph_ms["pool"] * 1e-3) / 1e9
    ps_gbs = pool_bytes(w) / ((ph_ms["pool"] + ph_ms["select"]) * 1e-3) / 1e9
    line = {
        "metric": METRIC,
        "value": job_throughput(w_job, world, ms_step, split),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "strong" if split == "heads" and world > 1 else "weak",
        "vs_baseline": None,
        "dtype": (("bf16 (Q K^T and P V in e4m3)" if w.pv_fp8 else "bf16 (Q K^T in e4m3)") if w.qk_fp8 else "bf16")
        if w.dtype == "bf16" else "f32",
        "data": "synthetic (smooth Gaussian-filtered fields + noise, seeded)",
        "config": _config_json(w_job, world, split, [h0, h1]),
        "ms_per_layer": ms_step,
        "phases_ms": ph_ms,
        "kept_tflop": flops_kept / 1e12,
        "dense_equiv_tflop": dense_equiv_flops(w) / 1e12,
        "kept_fraction_of_dense": flops_kept / dense_equiv_flops(w),
        "roofline": {"bound": "tensor", "kernel": "attn_kernel (bsa_attention_run: sparse + centroid + dense rows)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{peak_src} bf16_tflops (burst: the kernel runs inside a sub-second step)"
                     + ("" if ratio == 1.0 else f" x {ratio:.3f} for the e4m3 products (fp8 = 2 x bf16, nominal)"),
                     "frac_of_sustained": achieved / peak_sus,
                     "issued_tflop": flops_issued / 1e12,
                     "issued_achieved": flops_issued / (fine_ms * 1e-3) / 1e12,
                     "frac_issued": flops_issued / (fine_ms * 1e-3) / 1e12 / peak,
                     "traffic": attn_traffic(w),
                     "traffic_unit": "bytes per launch (ncu dram read+write, scaled from a 4-head capture)"},
        "roofline_select": {"bound": "hbm", "peak": hbm, "unit": "GB/s", "peak_source": f"{peak_src} hbm_gbs",
                            "pool_bytes": pool_bytes(w), "pool_achieved": pool_gbs, "pool_frac": pool_gbs / hbm,
                            "pool_plus_select_achieved": ps_gbs, "pool_plus_select_frac": ps_gbs / hbm,
                            "select_flop": select_flops(w),
                            "select_tflops": select_flops(w) / (ph_ms["select"] * 1e-3) / 1e12},
        "extra_tokens_per_row": (float(buf.extra_count.float().mean()) if buf.extra_count is not None else 0.0),
        "gpu_launches": launches,
        "workspace_bytes": int(buf.ws.numel() * buf.ws.element_size()),
        "clocks": clocks.summary(),
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = {k2: v2 for k2, v2 in cpu_baseline(w, q, k, v).items()
                                if k2 != "layer_s_extrapolated"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
