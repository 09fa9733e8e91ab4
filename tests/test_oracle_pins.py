"""Pins for the CPU oracle: facts fixed by the pages or by mathematics.

Each test checks the oracle against something other than its own formulas:
a library routine (numpy dense softmax attention, numpy means, scipy's normal
tail), a closed-form identity, a property that must hold, the pages' own
figures, or an independent pure-Python brute force.
"""
import math
import os

import numpy as np
import pytest
import torch
from scipy.stats import norm

import oracle
from tests import brute
from workloads import Workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, dtype, seed, layout="bnhd"):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(shape, generator=g)
    if layout == "bhnd":
        B, N, H, d = shape
        x = x.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
    return x.to(dtype)


def _dense_numpy(q, k, v, keys=None):
    """Dense softmax attention in float64 via numpy (a library reference).

    q, k, v: torch [B, N, H, d]; keys: optional index array restricting keys.
    Returns out [B, H, N, d], lse [B, H, N].
    """
    Q = q.double().permute(0, 2, 1, 3).numpy()
    K = k.double().permute(0, 2, 1, 3).numpy()
    V = v.double().permute(0, 2, 1, 3).numpy()
    if keys is not None:
        K, V = K[:, :, keys], V[:, :, keys]
    d = Q.shape[-1]
    L = Q @ np.swapaxes(K, -1, -2) / math.sqrt(d)
    m = L.max(axis=-1, keepdims=True)
    P = np.exp(L - m)
    den = P.sum(axis=-1, keepdims=True)
    return (P @ V) / den, (m + np.log(den))[..., 0]


def _oracle_full(w, q, k, v):
    """Oracle outputs for every token, shaped [B, H, N, d] and [B, H, N]."""
    qr, kr, vr = oracle.as_raw(q), oracle.as_raw(k), oracle.as_raw(v)
    res = oracle.routing(w, qr, kr, vr)
    out, lse = oracle.layer_rows(w, qr, kr, vr, res, oracle.all_tokens(w))
    return (out.reshape(w.B, w.H, w.N, w.d), lse.reshape(w.B, w.H, w.N), res)


def _wl(**kw):
    base = dict(name="t", B=1, H=2, N=200, d=16, dtype="bf16", method="sol", q_block=64,
                k_block=64, tau=1.0, sink_blocks=1, keep_diag=1, centroid=1)
    base.update(kw)
    return Workload(**base)


# ---------------------------------------------------------------- pooling

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("layout", ["bnhd", "bhnd"])
def test_block_means_match_numpy(dtype, layout):
    x = _rand((2, 203, 3, 24), dtype, 1, layout)
    mean, cnt = oracle.block_means(oracle.as_raw(x), 64)
    X = x.double().numpy()
    assert list(cnt) == [64, 64, 64, 11]
    for i, s in enumerate(range(0, 203, 64)):
        ref = X[:, s:s + 64].mean(axis=1).astype(np.float32)      # [B, H, d]
        np.testing.assert_allclose(mean[:, :, i], ref, rtol=2e-7, atol=0)


# ---------------------------------------------------------------- dense limits

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("method", ["sol", "sla"])
def test_keep_everything_is_dense_attention(dtype, method):
    """tau = -inf (Sol) or keep_percent = 100 (SLA) keeps every block: dense."""
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    w = _wl(dtype=dtype, method=method, tau=-math.inf, keep_percent=100.0,
            q_block=64 if method == "sol" else 128, centroid=1 if method == "sol" else 0)
    q, k, v = (_rand((1, w.N, w.H, w.d), tdt, s) for s in (2, 3, 4))
    out, lse, res = _oracle_full(w, q, k, v)
    ref, ref_lse = _dense_numpy(q, k, v)
    assert res.keep.all()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("N", [256, 200])
@pytest.mark.parametrize("tau", [0.5, 1.3, math.inf])
def test_block_constant_kv_centroids_are_exact(N, tau):
    """K and V constant within each key block: n_b copies of the centroid are the
    block itself, so the centroid term (with its ln n_b bias, partial last block
    included) reproduces dense attention for every tau."""
    w = _wl(N=N, tau=tau)
    g = torch.Generator().manual_seed(5)
    nKB = w.nKB
    kb = torch.randn((1, nKB, w.H, w.d), generator=g)
    vb = torch.randn((1, nKB, w.H, w.d), generator=g)
    idx = torch.arange(N) // w.k_block
    k = kb[:, idx].to(torch.bfloat16)
    v = vb[:, idx].to(torch.bfloat16)
    q = _rand((1, N, w.H, w.d), torch.bfloat16, 6) * 2
    out, lse, res = _oracle_full(w, q, k, v)
    ref, ref_lse = _dense_numpy(q, k, v)
    if tau != math.inf:
        assert not res.keep.all()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_block_constant_kv_with_extra_tokens_is_exact():
    """Same identity with extra tokens taken out of their blocks' centroids."""
    w = _wl(N=200, tau=1.0, extra_tokens=16)
    g = torch.Generator().manual_seed(15)
    kb = torch.randn((1, w.nKB, w.H, w.d), generator=g)
    vb = torch.randn((1, w.nKB, w.H, w.d), generator=g)
    idx = torch.arange(w.N) // w.k_block
    k, v = kb[:, idx].to(torch.bfloat16), vb[:, idx].to(torch.bfloat16)
    q = _rand((1, w.N, w.H, w.d), torch.bfloat16, 16)
    out, _, res = _oracle_full(w, q, k, v)
    assert res.ecnt.sum() > 0
    ref, _ = _dense_numpy(q, k, v)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_extra_tokens_covering_everything_is_dense():
    """E >= the number of candidate tokens: every key is exact, every centroid
    drops, the result is dense attention."""
    w = _wl(N=320, tau=1.0, extra_tokens=320)
    q, k, v = (_rand((1, w.N, w.H, w.d), torch.bfloat16, s) for s in (7, 8, 9))
    out, lse, res = _oracle_full(w, q, k, v)
    ref, ref_lse = _dense_numpy(q, k, v)
    assert not res.keep.all()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_prefix_only_selection_is_dense_over_prefix_blocks():
    """tau = +inf with no sink, no diagonal and no centroid keeps only the blocks
    of the packed prefix: dense attention restricted to those keys."""
    P = 100                                          # blocks 0 and 1 overlap [0, 100)
    w = _wl(N=320, tau=math.inf, sink_blocks=0, keep_diag=0, centroid=0, prefix_len=P)
    q, k, v = (_rand((1, w.N, w.H, w.d), torch.bfloat16, s) for s in (10, 11, 12))
    out, lse, _ = _oracle_full(w, q, k, v)
    ref, ref_lse = _dense_numpy(q, k, v, keys=np.arange(128))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_dense_rows_override():
    """Rows in the dense range equal dense attention whatever the selection."""
    w = _wl(N=320, tau=2.0, dense_rows=(70, 150))
    q, k, v = (_rand((1, w.N, w.H, w.d), torch.bfloat16, s) for s in (13, 14, 15))
    out, lse, _ = _oracle_full(w, q, k, v)
    ref, ref_lse = _dense_numpy(q, k, v)
    np.testing.assert_allclose(out[:, :, 70:150], ref[:, :, 70:150], rtol=0, atol=1e-12)
    assert np.abs(out[:, :, :64] - ref[:, :, :64]).max() > 1e-3   # the others are sparse


def test_centroid_only_equals_attention_over_centroids():
    """No kept block at all (tau = +inf, no sink, no diagonal): the output is
    softmax attention over the block centroids, each weighted by its size."""
    w = _wl(N=256, tau=math.inf, sink_blocks=0, keep_diag=0)
    q, k, v = (_rand((1, w.N, w.H, w.d), torch.bfloat16, s) for s in (17, 18, 19))
    out, _, res = _oracle_full(w, q, k, v)
    assert not res.keep.any()
    kc = k.double().reshape(1, 4, 64, w.H, w.d).mean(2)             # equal-size blocks
    vc = v.double().reshape(1, 4, 64, w.H, w.d).mean(2)
    kc, vc = kc.float().double(), vc.float().double()               # centroids stored fp32
    ref, _ = _dense_numpy(q, kc, vc)                                # ln 64 cancels
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-10)


# ---------------------------------------------------------------- V == 1

@pytest.mark.parametrize("cfg", [
    dict(method="sol", tau=1.0),
    dict(method="sol", tau=0.3, extra_tokens=32, prefix_len=70, dense_rows=(64, 128)),
    dict(method="sla", q_block=128, keep_percent=30.0, centroid=0),
])
def test_unit_values_give_unit_output(cfg):
    w = _wl(N=300, **cfg)
    q, k = (_rand((1, w.N, w.H, w.d), torch.bfloat16, s) for s in (20, 21))
    v = torch.ones((1, w.N, w.H, w.d), dtype=torch.bfloat16)
    out, lse, _ = _oracle_full(w, q, k, v)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-13)
    assert np.isfinite(lse).all()


# ---------------------------------------------------------------- selection

@pytest.mark.parametrize("tau", [0.5, 1.0, 1.5, 2.0])
def test_gaussian_scores_kept_fraction(tau):
    """Scores i.i.d. normal (shifted and scaled so that a missing mean or a
    variance used in place of the standard deviation would show): the
    threshold keeps a fraction 1 - Phi(tau) of the blocks."""
    rows, nKB = 64, 4096
    S = (5.0 + 3.0 * np.random.default_rng(0).standard_normal((rows, nKB))).astype(np.float32)
    keep, thr = oracle.select(S, N=nKB * 64, Bq=64, Bk=64, method="sol", tau=tau,
                              sink_blocks=0, prefix_len=0, keep_diag=0)
    p = norm.sf(tau)
    frac = keep.mean()
    band = 4 * math.sqrt(p * (1 - p) / (rows * nKB)) + 4 * math.sqrt(p * (1 - p) / nKB) / math.sqrt(rows) + 2.0 / nKB
    assert abs(frac - p) < band, (frac, p, band)


def test_threshold_is_shift_and_scale_invariant():
    rng = np.random.default_rng(1)
    S = rng.standard_normal((8, 512)).astype(np.float32)
    a, _ = oracle.select(S, N=512 * 64, Bq=64, Bk=64, method="sol", tau=1.3, sink_blocks=0,
                         keep_diag=0)
    b, _ = oracle.select((S * 4 + 16).astype(np.float32), N=512 * 64, Bq=64, Bk=64, method="sol",
                         tau=1.3, sink_blocks=0, keep_diag=0)
    assert (a == b).mean() > 0.999


def test_pages_tau_to_kept_fraction_figures():
    """The pages' figures (about 16 / 7 / 2.7 % kept at tau = 1 / 1.5 / 2) on
    normal scores, with the sink and diagonal blocks kept in addition."""
    table = np.loadtxt(os.path.join(GOLDEN, "tau_kept_fraction.txt"))
    nQB = nKB = 1024
    S = np.random.default_rng(2).standard_normal((nQB, nKB)).astype(np.float32)
    for tau, pct in table:
        keep, _ = oracle.select(S, N=nKB * 64, Bq=64, Bk=64, method="sol", tau=float(tau),
                                sink_blocks=1, keep_diag=1)
        assert abs(100.0 * keep.mean() - pct) < 0.6, (tau, 100.0 * keep.mean(), pct)


def test_sigma_zero_keeps_only_forced():
    S = np.full((4, 64), 3.25, np.float32)
    keep, _ = oracle.select(S, N=64 * 64, Bq=64, Bk=64, method="sol", tau=-0.5, sink_blocks=1,
                            keep_diag=1)
    for i in range(4):
        exp = np.zeros(64, np.uint8)
        exp[0] = 1
        exp[i] = 1
        assert (keep[i] == exp).all()


def test_sla_topk_matches_stable_sort_with_ties():
    rng = np.random.default_rng(3)
    S = rng.integers(0, 6, size=(16, 90)).astype(np.float32)        # many ties
    keep, thr = oracle.select(S, N=90 * 64, Bq=128, Bk=64, method="sla", keep_percent=15.0,
                              sink_blocks=0, keep_diag=0)
    k = int(math.floor(15.0 * 90 / 100 + 0.5))                       # 14
    for r in range(16):
        order = np.argsort(-S[r], kind="stable")
        exp = np.zeros(90, np.uint8)
        exp[order[:k]] = 1
        assert (keep[r] == exp).all()
        assert thr[r] == S[r, order[k - 1]]


def test_forced_blocks_q128_diagonal_is_two_blocks():
    f = oracle.forced_blocks(3, nKB=20, N=20 * 64, Bq=128, Bk=64, sink_blocks=1, prefix_len=0,
                             keep_diag=1)
    assert list(np.nonzero(f)[0]) == [0, 6, 7]
    f = oracle.forced_blocks(9, nKB=20, N=20 * 64 - 10, Bq=128, Bk=64, sink_blocks=0,
                             prefix_len=130, keep_diag=1)
    assert list(np.nonzero(f)[0]) == [0, 1, 2, 18, 19]


def test_extra_tokens_match_numpy_bruteforce():
    w = _wl(N=320, H=2, d=16, tau=1.0, extra_tokens=24)
    q, k, v = (_rand((1, w.N, w.H, w.d), torch.bfloat16, s) for s in (22, 23, 24))
    kr = oracle.as_raw(k)
    res = oracle.routing(w, oracle.as_raw(q), kr, oracle.as_raw(v))
    K = k.double().numpy()[0]                                    # [N, H, d]
    keep = res.keep.reshape(w.rows, w.nKB)
    for r in range(w.rows):
        h, i = (r // w.nQB) % w.H, r % w.nQB
        qt = torch.from_numpy(res.qbar[0, h, i]).to(torch.bfloat16).double().numpy()
        t = (K[:, h] @ qt / math.sqrt(w.d)).astype(np.float32)
        cand = np.array([n for n in range(w.N) if not keep[r, n // 64]])
        order = sorted(cand, key=lambda n: (-t[n], n))
        exp = sorted(order[:w.extra_tokens])
        assert res.ecnt[r] == len(exp)
        assert list(res.extra[r, :res.ecnt[r]]) == exp


def test_mask_to_csr_roundtrip():
    keep = (np.random.default_rng(4).random((5, 7, 33)) < 0.3).astype(np.uint8)
    rp, col, cnt = oracle.mask_to_csr(keep)
    flat = keep.reshape(-1, 33)
    for r in range(flat.shape[0]):
        assert list(col[rp[r]:rp[r + 1]]) == list(np.nonzero(flat[r])[0])
        assert cnt[r] == flat[r].sum()


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("cfg", [
    dict(method="sol", tau=0.7, N=200),
    dict(method="sol", tau=0.2, N=256, extra_tokens=8, prefix_len=20, dense_rows=(10, 30)),
    dict(method="sla", q_block=128, keep_percent=40.0, centroid=0, N=250),
    dict(method="sol", tau=1.0, N=150, dtype="f32", extra_tokens=5),
])
def test_tiny_cases_match_pure_python_bruteforce(cfg):
    w = _wl(H=2, d=8, **cfg)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    g = torch.Generator().manual_seed(30)
    base = torch.randn((1, w.N // 8 + 1, w.H, w.d), generator=g)
    # smooth-ish keys so that selections differ between blocks
    idx = torch.arange(w.N) // 8
    q = (base[:, idx] + 0.5 * torch.randn((1, w.N, w.H, w.d), generator=g)).to(tdt)
    k = (base[:, idx] + 0.5 * torch.randn((1, w.N, w.H, w.d), generator=g)).to(tdt)
    v = torch.randn((1, w.N, w.H, w.d), generator=g).to(tdt)
    out, lse, res = _oracle_full(w, q, k, v)
    Q, K, V = (t[0].double().tolist() for t in (q, k, v))
    p = dict(method=w.method, tau=w.tau, keep_percent=w.keep_percent, q_block=w.q_block,
             k_block=w.k_block, sink_blocks=w.sink_blocks, prefix_len=w.prefix_len,
             keep_diag=w.keep_diag, extra_tokens=w.extra_tokens, centroid=w.centroid,
             dense_rows=w.dense_rows, dtype=w.dtype)
    keep_b, out_b, lse_b = brute.run(Q, K, V, w.N, w.H, w.d, p)
    assert (res.keep[0].astype(bool) == np.array(keep_b)).all()
    np.testing.assert_allclose(out[0], np.array(out_b), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0], np.array(lse_b), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- cube tiling (vsa)

def _vsa(**kw):
    base = dict(name="v", B=1, H=2, d=16, dtype="bf16", method="vsa", q_block=64, k_block=64,
                keep_percent=30.0, centroid=0)
    base.update(kw)
    return Workload(**base)


def test_cube_order_blocks_are_the_grid_cubes():
    """Every block of the cube order is one 4 x 4 x 4 box of the latent grid
    (its tokens' (t, y, x) span 4 consecutive values on each axis, aligned to
    4), the prefix keeps its order, and every token appears once."""
    w = _vsa(N=64 + 8 * 12 * 16, prefix_len=64, grid=(8, 12, 16))
    order = oracle.cube_order(w)
    assert sorted(order.tolist()) == list(range(w.N))
    assert order[:64].tolist() == list(range(64))
    T, Hs, Ws = w.grid
    for blk in range(1, w.N // 64):
        toks = order[64 * blk:64 * blk + 64] - w.prefix_len
        t, y, x = toks // (Hs * Ws), (toks // Ws) % Hs, toks % Ws
        for axis in (t, y, x):
            assert axis.min() % 4 == 0 and axis.max() - axis.min() == 3
        assert len({(a, b, c) for a, b, c in zip(t, y, x)}) == 64
        # t-major inside the cube: slot s = 16 dt + 4 dy + dx
        s = 16 * (t - t.min()) + 4 * (y - y.min()) + (x - x.min())
        assert s.tolist() == list(range(64))


def test_vsa_on_column_cubes_is_sla_with_64_token_blocks():
    """With a 4 x 4 frame every cube is 64 consecutive tokens, so cube tiling is
    the identity order and vsa must give exactly SLA with Q64/K64 blocks."""
    w = _vsa(N=64 * 12, grid=(48, 4, 4), keep_percent=25.0)
    assert oracle.cube_order(w).tolist() == list(range(w.N))
    q, k, v = (_rand((1, w.N, w.H, w.d), torch.bfloat16, s) for s in (41, 42, 43))
    out_v, lse_v, res_v = _oracle_full(w, q, k, v)
    out_s, lse_s, res_s = _oracle_full(w.replace(method="sla"), q, k, v)
    assert np.array_equal(res_v.keep, res_s.keep)
    assert np.array_equal(out_v, out_s) and np.array_equal(lse_v, lse_s)


def test_vsa_keep_all_is_dense_attention():
    w = _vsa(N=64 + 4 * 8 * 8, prefix_len=64, grid=(4, 8, 8), keep_percent=100.0)
    q, k, v = (_rand((1, w.N, w.H, w.d), torch.bfloat16, s) for s in (44, 45, 46))
    out, lse, res = _oracle_full(w, q, k, v)
    ref, ref_lse = _dense_numpy(q, k, v)
    assert res.keep.all()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_vsa_cube_means_are_means_over_the_cube():
    w = _vsa(N=8 * 8 * 8, grid=(8, 8, 8))
    k = _rand((1, w.N, w.H, w.d), torch.float32, 47)
    res = oracle.routing(w, *(oracle.as_raw(k) for _ in range(3)))
    K = k.double().numpy().reshape(8, 8, 8, w.H, w.d)          # (t, y, x, h, c)
    c = 0
    for t0 in range(0, 8, 4):
        for y0 in range(0, 8, 4):
            for x0 in range(0, 8, 4):
                ref = K[t0:t0 + 4, y0:y0 + 4, x0:x0 + 4].mean(axis=(0, 1, 2)).astype(np.float32)
                np.testing.assert_allclose(res.kbar[0, :, c], ref, rtol=2e-7, atol=0)
                c += 1
