"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle,
element by element, on seeded inputs that span several tiles and ragged tails.
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_26_b200 as bsa
import oracle
from tests.gpu_helpers import (compare_masks, compare_outputs, csr_to_mask, gpu_layer, params_for,
                               to_cpu_raw)
from workloads import TINY_SOL, Workload, make_qkv

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny_sol": TINY_SOL,
    "sol_grid": Workload("sol_grid", B=1, H=3, N=3000, d=128, dtype="bf16", method="sol", q_block=64,
                         k_block=64, tau=1.3, grid=(3, 20, 50), seed=11),
    "sla_grid": Workload("sla_grid", B=1, H=2, N=2880, d=128, dtype="bf16", method="sla", q_block=128,
                         k_block=64, keep_percent=15.0, centroid=0, grid=(4, 24, 30), seed=12),
    "sol_sinks": Workload("sol_sinks", B=1, H=2, N=2120, d=128, dtype="bf16", method="sol", q_block=64,
                          k_block=64, tau=1.3, prefix_len=200, dense_rows=(72, 200), grid=(3, 16, 40),
                          seed=13),
    "sol_b2_d64": Workload("sol_b2_d64", B=2, H=2, N=1500, d=64, dtype="bf16", method="sol", q_block=64,
                           k_block=64, tau=0.8, grid=(3, 10, 50), seed=14),
    "sol_dense_tau": Workload("sol_dense_tau", B=1, H=2, N=1100, d=128, dtype="bf16", method="sol",
                              q_block=64, k_block=64, tau=-math.inf, grid=(2, 10, 55), seed=15),
    "sla_keep_all": Workload("sla_keep_all", B=1, H=2, N=1000, d=128, dtype="bf16", method="sla",
                             q_block=128, k_block=64, keep_percent=100.0, centroid=0, grid=(2, 10, 50),
                             seed=16),
    "single_block": Workload("single_block", B=1, H=2, N=40, d=128, dtype="bf16", method="sol", q_block=64,
                             k_block=64, tau=1.0, grid=(1, 5, 8), seed=17),
    "dense_split": Workload("dense_split", B=1, H=1, N=20032, d=128, dtype="bf16", method="sol", q_block=64,
                            k_block=64, tau=1.5, prefix_len=256, dense_rows=(100, 300), grid=(4, 24, 206),
                            seed=20),
    "sol_extra64": Workload("sol_extra64", B=1, H=2, N=2120, d=128, dtype="bf16", method="sol", q_block=64,
                            k_block=64, tau=1.3, prefix_len=200, dense_rows=(72, 200), extra_tokens=64,
                            grid=(3, 16, 40), seed=21),
    "sol_extra256": Workload("sol_extra256", B=1, H=2, N=3000, d=128, dtype="bf16", method="sol", q_block=64,
                             k_block=64, tau=1.0, extra_tokens=256, grid=(3, 20, 50), seed=22),
    # extra tokens with d = 64 and two batches: the modified-centroid build's
    # 64-channel form and its (batch, head) indexing; a ragged last block
    "sol_extra_b2_d64": Workload("sol_extra_b2_d64", B=2, H=2, N=1500, d=64, dtype="bf16", method="sol",
                                 q_block=64, k_block=64, tau=1.0, extra_tokens=64, grid=(3, 10, 50), seed=23),
    "no_diag_no_sink": Workload("no_diag_no_sink", B=1, H=2, N=1300, d=128, dtype="bf16", method="sol",
                                q_block=64, k_block=64, tau=1.0, sink_blocks=0, keep_diag=0,
                                grid=(2, 13, 50), seed=18),
}


def _inputs(w, layout="bnhd"):
    q, k, v = make_qkv(w, "cpu", layout)
    return q, k, v, q.cuda(), k.cuda(), v.cuda()


def _to_cuda_like(t):
    """Copy a (possibly strided) CPU tensor to the GPU keeping its strides."""
    out = torch.empty_strided(t.shape, t.stride(), dtype=t.dtype, device="cuda")
    out.copy_(t)
    return out


@pytest.fixture(scope="module")
def runs():
    cache = {}

    def get(name, layout="bnhd"):
        key = (name, layout)
        if key not in cache:
            w = SMALL[name]
            qc, kc, vc = make_qkv(w, "cpu", layout)
            q, k, v = (_to_cuda_like(t) for t in (qc, kc, vc))
            p, buf, out, status = gpu_layer(w, q, k, v)
            res = oracle.routing(w, oracle.as_raw(qc), oracle.as_raw(kc), oracle.as_raw(vc))
            cache[key] = (w, (qc, kc, vc), (q, k, v), p, buf, out, status, res)
        return cache[key]

    return get


@pytest.mark.parametrize("name", list(SMALL))
def test_pool_bit_exact(runs, name):
    w, _, _, p, buf, _, status, res = runs(name)
    assert status == 0
    assert np.array_equal(buf.qbar.cpu().numpy(), res.qbar)
    assert np.array_equal(buf.kbar.cpu().numpy(), res.kbar)
    assert np.array_equal(buf.vbar.cpu().numpy(), res.vbar)
    assert np.array_equal(buf.blk_count.cpu().numpy(), res.count)


@pytest.mark.parametrize("name", list(SMALL))
def test_select_masks_match(runs, name):
    w, _, _, p, buf, _, status, res = runs(name)
    assert status == 0
    mask = csr_to_mask(buf.row_ptr, buf.col_idx, w.rows, w.nKB)
    exempt = compare_masks(mask, res, w)
    assert exempt <= max(1, w.rows // 1000), exempt
    kc = buf.kept_count.cpu().numpy()
    assert np.array_equal(kc, mask.sum(axis=1))


@pytest.mark.parametrize("name", list(SMALL))
def test_attention_matches_oracle(runs, name):
    w, (qc, kc, vc), _, p, buf, out, status, res = runs(name)
    assert status == 0
    tokens = oracle.all_tokens(w)
    ref, ref_lse = oracle.layer_rows(w, oracle.as_raw(qc), oracle.as_raw(kc), oracle.as_raw(vc), res, tokens)
    got = out.float().cpu().permute(0, 2, 1, 3).reshape(-1, w.d).numpy()   # (b, h, n) order
    compare_outputs(got, ref, f"{name} out")
    lse = buf.lse.cpu().numpy().reshape(-1)
    err = np.abs(lse - ref_lse)
    assert err.max() < 2e-2, err.max()


def test_strided_layout_matches_contiguous(runs):
    """[B, H, N, d] storage (head-major) gives the same result as [B, N, H, d]."""
    a = runs("sol_grid", "bnhd")
    b = runs("sol_grid", "bhnd")
    assert np.array_equal(a[4].qbar.cpu().numpy(), b[4].qbar.cpu().numpy())
    assert torch.equal(a[4].row_ptr.cpu(), b[4].row_ptr.cpu())
    assert torch.equal(a[5].cpu(), b[5].cpu())


def test_dense_ref_rows_matches_dense_attention():
    w = SMALL["sol_grid"]
    qc, kc, vc = make_qkv(w, "cpu")
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    p = params_for(w, q)
    buf = bsa.Buffers(p, q.device)
    out = torch.zeros_like(q)
    lse = torch.zeros((w.B, w.H, w.N), dtype=torch.float32, device="cuda")
    r0, r1 = 100, 333
    bsa.bsa_dense_ref_rows(p, q, k, v, r0, r1, out, lse, buf.ws)
    assert bsa.bsa_device_status(buf.ws) == 0
    tokens = np.array([(0, h, n) for h in range(w.H) for n in range(r0, r1)], np.int64)
    wd = w.replace(dense_rows=(r0, r1))
    res = oracle.routing(wd, oracle.as_raw(qc), oracle.as_raw(kc), oracle.as_raw(vc))
    ref, ref_lse = oracle.layer_rows(wd, oracle.as_raw(qc), oracle.as_raw(kc), oracle.as_raw(vc), res, tokens)
    got = out[0, r0:r1].float().cpu().permute(1, 0, 2).reshape(-1, w.d).numpy()
    compare_outputs(got, ref, "dense rows")
    assert torch.count_nonzero(out[0, :r0]) == 0 and torch.count_nonzero(out[0, r1:]) == 0
    got_lse = lse[0, :, r0:r1].cpu().numpy().reshape(-1)
    assert np.abs(got_lse - ref_lse).max() < 2e-2


def test_capacity_overflow_reported_on_device():
    w = SMALL["sol_grid"]
    qc, kc, vc = make_qkv(w, "cpu")
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    p = params_for(w, q)
    buf = bsa.Buffers(p, q.device, capacity=10)
    bsa.bsa_pool(p, q, k, v, buf.qbar, buf.kbar, buf.vbar, buf.blk_count)
    bsa.bsa_select(p, buf.qbar, buf.kbar, k, buf.row_ptr, buf.col_idx, buf.kept_count, None, None, buf.ws)
    assert bsa.bsa_device_status(buf.ws) == 3          # BSA_ERR_CAPACITY
    assert bsa.bsa_device_status(buf.ws) == 0          # cleared by the read
    assert int(buf.row_ptr[-1]) > 10                   # counts and offsets are still complete


def test_sigma_zero_rows_keep_only_forced():
    """Block-constant Q and K make every pooled score of a row equal (sigma = 0)."""
    w = Workload("flat", B=1, H=2, N=640, d=128, dtype="bf16", method="sol", q_block=64, k_block=64,
                 tau=1.0, grid=None, seed=19)
    q = torch.ones((1, w.N, w.H, w.d), dtype=torch.bfloat16, device="cuda")
    k = torch.ones_like(q)
    v = torch.randn(q.shape, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).cuda()
    p, buf, out, status = gpu_layer(w, q, k, v)
    assert status == 0
    kc = buf.kept_count.cpu().numpy()
    # sink block 0 plus the diagonal block (the same block for query block 0)
    assert kc[0] == 1 and (kc[1:w.nQB] == 2).all()


# Sol with a finite tau takes the certified route: its masks equal the
# definition's bit for bit, with no near-threshold exemption.  The cases below
# also push rows onto the route's exact paths: keys that are nearly identical
# (every block undecided by the tensor-core scores: list overflow, exact
# fallback rows), pooled values scaled far up or down (bounds near the ends of
# the f32 range), and one enormous key block (rows sent to the exact path, with
# scores whose fp64 sum depends on its order).
ROUTE = {
    "near_identical_keys": Workload("near_identical_keys", B=1, H=2, N=3000, d=128, dtype="bf16", method="sol",
                                    q_block=64, k_block=64, tau=1.0, grid=(3, 20, 50), seed=31),
    "large_scale": Workload("large_scale", B=1, H=2, N=2500, d=128, dtype="bf16", method="sol", q_block=64,
                            k_block=64, tau=1.3, grid=(2, 25, 50), seed=32),
    "tiny_scale": Workload("tiny_scale", B=1, H=2, N=2500, d=64, dtype="bf16", method="sol", q_block=64,
                           k_block=64, tau=0.7, grid=(2, 25, 50), seed=33),
    "huge_block": Workload("huge_block", B=1, H=2, N=2500, d=128, dtype="bf16", method="sol", q_block=64,
                           k_block=64, tau=1.3, grid=(2, 25, 50), seed=35),
    "negative_tau": Workload("negative_tau", B=1, H=2, N=2970, d=128, dtype="bf16", method="sol", q_block=64,
                             k_block=64, tau=-0.6, prefix_len=130, grid=(2, 20, 71), seed=34),
}


def _route_inputs(name, w):
    q, k, v = make_qkv(w, "cpu")
    if name == "near_identical_keys":
        # one key row for the whole sequence plus a perturbation of a few ulps
        base = k[:, :1].float()
        k = (base + 1e-3 * (k.float() - base)).to(k.dtype)
    elif name == "large_scale":
        q = q * 2.0 ** 60
    elif name == "tiny_scale":
        q = q * 2.0 ** -120
        k = k * 2.0 ** -4
    elif name == "huge_block":
        # one key block of head 0 at 2^110: the tensor-core products could
        # overflow, so every row of that head takes the exact path, whose scores
        # then span far more than fp64 can sum exactly in any order
        k = k.clone()
        k[:, 640:704, 0] = k[:, 640:704, 0] * 2.0 ** 110
    return q.contiguous(), k.contiguous(), v


@pytest.mark.parametrize("name", list(ROUTE))
def test_certified_route_masks_exact(name):
    w = ROUTE[name]
    q, k, v = _route_inputs(name, w)
    p, buf, out, status = gpu_layer(w, q.cuda(), k.cuda(), v.cuda())
    assert status == 0
    res = oracle.routing(w, oracle.as_raw(q), oracle.as_raw(k), oracle.as_raw(v))
    assert np.array_equal(buf.qbar.cpu().numpy(), res.qbar)
    mask = csr_to_mask(buf.row_ptr, buf.col_idx, w.rows, w.nKB)
    ora = res.keep.reshape(w.rows, w.nKB)
    diff = np.argwhere(mask != ora)
    assert len(diff) == 0, f"{len(diff)} mask differences, e.g. {diff[:5].tolist()}"
    assert np.array_equal(buf.kept_count.cpu().numpy(), ora.sum(axis=1).astype(np.int32))


@pytest.mark.parametrize("name", [n for n, w in SMALL.items() if w.method == "sol" and math.isfinite(w.tau)])
def test_certified_route_no_exemptions(runs, name):
    w, _, _, p, buf, _, status, res = runs(name)
    assert status == 0
    mask = csr_to_mask(buf.row_ptr, buf.col_idx, w.rows, w.nKB)
    assert np.array_equal(mask, res.keep.reshape(w.rows, w.nKB))


# Row maxima that rise steeply along the keys: key block b is scaled by 1 + 4 b,
# so a row's largest score grows by about 20 (natural units) from one tile to
# the next -- more than a tile's sum bound on P allows, which sends those tiles
# through the online softmax's rescale -- on exact and centroid tiles alike
# (with sla, no centroids: kept blocks only).
RISING = {
    "rising_sol": Workload("rising_sol", B=1, H=2, N=2085, d=128, dtype="bf16", method="sol", q_block=64,
                           k_block=64, tau=0.8, grid=(3, 5, 139), seed=41),
    "rising_sla": Workload("rising_sla", B=1, H=2, N=2085, d=128, dtype="bf16", method="sla", q_block=128,
                           k_block=64, keep_percent=40.0, centroid=0, grid=(3, 5, 139), seed=42),
}


@pytest.mark.parametrize("name", list(RISING))
def test_rising_row_maxima(name):
    w = RISING[name]
    q, k, v = make_qkv(w, "cpu")
    ramp = 1.0 + 4.0 * (torch.arange(w.N) // 64).double()
    k = (k.double() * ramp[None, :, None, None]).to(k.dtype)
    p, buf, out, status = gpu_layer(w, q.cuda(), k.cuda(), v.cuda())
    assert status == 0
    raw = [oracle.as_raw(t) for t in (q, k, v)]
    res = oracle.routing(w, *raw)
    ref, ref_lse = oracle.layer_rows(w, *raw, res, oracle.all_tokens(w))
    got = out.float().cpu().permute(0, 2, 1, 3).reshape(-1, w.d).numpy()
    compare_outputs(got, ref, f"{name} out")
    assert np.abs(buf.lse.cpu().numpy().reshape(-1) - ref_lse).max() < 2e-2
