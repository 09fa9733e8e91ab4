"""GPU parity of the extra-token selection ("BlockSparseAttention - ComfyUI
Built-in Node Documentation", general inputs, extra_tokens) against the CPU
oracle.

Both sides score token j of query block i as qt_i . k_j / sqrt(d) with qt_i the
pooled query rounded to bf16, so every product qt_c * k_jc is exact in fp32.
The GPU sums the 128 products on the tensor cores in fp32 (order and rounding
of the hardware's accumulation unspecified), the oracle in fp64 and rounds the
scaled sum to fp32.  With A_j = sum_c |qt_c k_jc|, the two scores of a token
differ by at most

    delta_j = gamma_128 * A_j / sqrt(d) + 2^-24 * |t_j|,
    gamma_n = n u / (1 - n u),  u = 2^-23

(u = 2^-23 rather than 2^-24 allows the accumulation to truncate instead of
rounding to nearest; the second term is the oracle's rounding to fp32).  Two
tokens can therefore trade places only if their oracle scores lie within the
sum of their deltas: a token in one set and not the other is exempt iff its
oracle score is within delta_j + delta_max of the row's E-th oracle score t_E,
delta_max being the largest delta of the row's differing and E-th tokens.
Exempted tokens are counted and reported.

Query blocks whose rows all run dense get no extra tokens (the design's
reading R14): bsa_attention replaces those rows by dense attention, which
never reads the list.
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_26_b200 as bsa
import oracle
from workloads import CONFIGS, Workload, make_qkv, sample_heads, sample_query_blocks

pytestmark = pytest.mark.gpu

U_ACC = 2.0 ** -23


def gamma(n: int) -> float:
    return n * U_ACC / (1.0 - n * U_ACC)


def _gpu_select(w, q, k, v):
    p = bsa.params_for(w, q)
    buf = bsa.Buffers(p, q.device)
    bsa.bsa_pool(p, q, k, v, buf.qbar, buf.kbar, buf.vbar, buf.blk_count)
    bsa.bsa_select(p, buf.qbar, buf.kbar, k, buf.row_ptr, buf.col_idx, buf.kept_count, buf.extra_idx,
                   buf.extra_count, buf.ws)
    assert bsa.bsa_device_status(buf.ws) == 0
    return p, buf


def _row_all_dense(w, r):
    i = r % w.nQB
    lo, hi = i * w.q_block, min(w.N, (i + 1) * w.q_block)
    return lo >= w.dense_rows[0] and hi <= w.dense_rows[1]


def _check_rows(w, res, kc, gpu_idx, gpu_cnt, rows):
    """Compare GPU extras with the oracle's on `rows`; returns the exempted count."""
    ex, ec, _ = oracle.extra_tokens(res.qbar, oracle.as_raw(kc), res.keep, w.q_block, w.k_block,
                                    w.extra_tokens, rows)
    K = kc.double().numpy()
    g_d = gamma(w.d)
    exempt = 0
    for n, r in enumerate(rows):
        if _row_all_dense(w, r):
            assert gpu_cnt[r] == 0
            continue
        a = set(ex[n, :ec[n]].tolist())
        g_list = gpu_idx[r, :gpu_cnt[r]].tolist()
        assert g_list == sorted(g_list), f"row {r}: not ascending"
        g = set(g_list)
        assert len(g) == gpu_cnt[r] == ec[n], (r, len(g), gpu_cnt[r], ec[n])
        diff = a ^ g
        if not diff:
            continue
        b, h, i = r // (w.H * w.nQB), (r // w.nQB) % w.H, r % w.nQB
        qt = torch.from_numpy(res.qbar[b, h, i]).to(torch.bfloat16).double().numpy()
        rs = math.sqrt(w.d)

        def score(t):   # the oracle's score: fp64 sum, scaled, rounded to fp32
            return float(np.float32(float(K[b, t, h] @ qt) / rs))

        def delta(t):
            return g_d * float(np.abs(K[b, t, h] * qt).sum()) / rs + 2.0 ** -24 * abs(score(t))

        e_tok = min(a, key=lambda t: (score(t), -t))          # the oracle's E-th token
        t_e = score(e_tok)
        d_max = max(delta(t) for t in list(diff) + [e_tok])
        for t in diff:
            assert abs(score(t) - t_e) <= delta(t) + d_max, (r, t, score(t), t_e, delta(t), d_max)
        exempt += len(diff)
    return exempt


@pytest.mark.parametrize("E", [64, 256])
def test_extra_tokens_small(E):
    w = Workload("extra_small", B=1, H=2, N=2120, d=128, dtype="bf16", method="sol", q_block=64,
                 k_block=64, tau=1.3, prefix_len=200, dense_rows=(72, 200), extra_tokens=E,
                 grid=(3, 16, 40), seed=51)
    qc, kc, vc = make_qkv(w, "cpu")
    p, buf = _gpu_select(w, qc.cuda(), kc.cuda(), vc.cuda())
    res = oracle.routing(w, oracle.as_raw(qc), oracle.as_raw(kc), oracle.as_raw(vc), with_extra=False)
    exempt = _check_rows(w, res, kc, buf.extra_idx.cpu().numpy(), buf.extra_count.cpu().numpy(),
                         list(range(w.rows)))
    assert exempt <= w.rows * E // 1000 + 2, exempt


def test_extra_tokens_full_size_sampled():
    w = CONFIGS["sol_sinks"]
    q, k, v = make_qkv(w, "cuda")
    p, buf = _gpu_select(w, q, k, v)
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    res = oracle.routing(w, oracle.as_raw(qc), oracle.as_raw(kc), oracle.as_raw(vc), with_extra=False)
    rows = [(0 * w.H + h) * w.nQB + i for h in sample_heads(w) for i in sample_query_blocks(w, 64)]
    exempt = _check_rows(w, res, kc, buf.extra_idx.cpu().numpy(), buf.extra_count.cpu().numpy(), rows)
    print(f"sol_sinks: {len(rows)} sampled rows, exempted tokens {exempt}")
    assert exempt <= len(rows) * 2


def test_extra_tokens_all_scores_tied():
    """Every key token identical: every candidate ties, the survivors of the
    bucketed filter overflow the per-row buffer, and the per-row fallback must
    return the E lowest candidate indices (ties to the lower index)."""
    w = Workload("extra_tied", B=1, H=2, N=4200, d=128, dtype="bf16", method="sol", q_block=64,
                 k_block=64, tau=1.3, extra_tokens=64, grid=(3, 20, 70), seed=53)
    qc, kc, vc = make_qkv(w, "cpu")
    kc = kc[:, :1].expand_as(kc).contiguous()
    p, buf = _gpu_select(w, qc.cuda(), kc.cuda(), vc.cuda())
    res = oracle.routing(w, oracle.as_raw(qc), oracle.as_raw(kc), oracle.as_raw(vc), with_extra=False)
    ex, ec, _ = oracle.extra_tokens(res.qbar, oracle.as_raw(kc), res.keep, w.q_block, w.k_block,
                                    w.extra_tokens, list(range(w.rows)))
    gi, gc = buf.extra_idx.cpu().numpy(), buf.extra_count.cpu().numpy()
    keep = res.keep.reshape(w.rows, w.nKB)
    for r in range(w.rows):
        cand = [t for t in range(w.N) if not keep[r, t // w.k_block]]
        assert gc[r] == ec[r] == min(w.extra_tokens, len(cand)), r
        assert gi[r, :gc[r]].tolist() == cand[:gc[r]] == ex[r, :ec[r]].tolist(), r


def test_extra_tokens_fewer_candidates_than_E():
    """A low tau keeps most blocks, leaving some rows fewer unselected tokens
    than E: those rows take every candidate, in ascending order."""
    w = Workload("extra_short", B=1, H=2, N=1000, d=128, dtype="bf16", method="sol", q_block=64,
                 k_block=64, tau=-0.8, extra_tokens=256, grid=(2, 10, 50), seed=54)
    qc, kc, vc = make_qkv(w, "cpu")
    p, buf = _gpu_select(w, qc.cuda(), kc.cuda(), vc.cuda())
    res = oracle.routing(w, oracle.as_raw(qc), oracle.as_raw(kc), oracle.as_raw(vc), with_extra=False)
    keep = res.keep.reshape(w.rows, w.nKB)
    gi, gc = buf.extra_idx.cpu().numpy(), buf.extra_count.cpu().numpy()
    short = 0
    for r in range(w.rows):
        cand = [t for t in range(w.N) if not keep[r, t // w.k_block]]
        if len(cand) <= w.extra_tokens:
            short += 1
            assert gc[r] == len(cand) and gi[r, :gc[r]].tolist() == cand, r
    assert short > 0, "no row with fewer candidates than E: the case is not exercised"
    exempt = _check_rows(w, res, kc, gi, gc, list(range(w.rows)))
    assert exempt <= w.rows * w.extra_tokens // 1000 + 2, exempt
