"""The QKV projection with pooling in its epilogue (bsa_qkv_pool;
"minimax-h3-chunk-star7" README, "Sol": a producer with fused preprocessing).

The projection is checked against an fp64 product of the same bf16 operands.
With A = sum_k |x_k w_k| (which bounds |y|), the kernel's output differs from
it by at most the final rounding to bf16 (2^-9 relative, so 2^-9 A) plus the
error of the tensor cores' fp32 accumulation, for which the same generous
allowance as the routing certificate's is used (2^-12 A; round-to-nearest fp32
would stay below d_model * 2^-24 A).  A wrong row, column or head gives errors
of the order of |y| itself.  The block means must equal, bit for bit, the
oracle's pooling of the very tensors the kernel wrote.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_26_b200 as bsa
import oracle
from workloads import Workload

pytestmark = pytest.mark.gpu

CASES = [
    # (workload, d_model, layout)
    (Workload("prod_sol", B=1, H=2, N=1000, d=128, dtype="bf16", method="sol", q_block=64, k_block=64, tau=1.3,
              seed=91), 256, "bnhd"),
    (Workload("prod_sla_b2", B=2, H=4, N=700, d=64, dtype="bf16", method="sla", q_block=128, k_block=64,
              keep_percent=20.0, centroid=0, seed=92), 192, "bnhd"),
    (Workload("prod_strided", B=1, H=2, N=1500, d=128, dtype="bf16", method="sol", q_block=64, k_block=64, tau=1.0,
              seed=93), 320, "bhnd"),
]


def _bound(x, w):
    A = np.abs(x) @ np.abs(w).T
    return (2.0 ** -9 + 2.0 ** -12) * A + 1e-30


def _out(shape, layout, device="cuda"):
    B, N, H, d = shape
    if layout == "bnhd":
        return torch.empty((B, N, H, d), dtype=torch.bfloat16, device=device)
    return torch.empty((B, H, N, d), dtype=torch.bfloat16, device=device).permute(0, 2, 1, 3)


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_qkv_pool_matches_projection_and_pooling(case):
    w, dm, layout = case
    g = torch.Generator().manual_seed(w.seed)
    x = (torch.randn((w.B, w.N, dm), generator=g) * 0.5).to(torch.bfloat16)
    W = (torch.randn((3 * w.H * w.d, dm), generator=g) / dm ** 0.5).to(torch.bfloat16)
    xg, Wg = x.cuda(), W.cuda()
    q, k, v = (_out((w.B, w.N, w.H, w.d), layout) for _ in range(3))
    p = bsa.params_for(w, q)
    nQB, nKB, rows = bsa.dims(p)
    qbar = torch.empty((w.B, w.H, nQB, w.d), dtype=torch.float32, device="cuda")
    kbar = torch.empty((w.B, w.H, nKB, w.d), dtype=torch.float32, device="cuda")
    vbar = torch.empty_like(kbar)
    cnt = torch.empty((nKB,), dtype=torch.int32, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    bsa.bsa_qkv_pool(p, xg, Wg, q, k, v, qbar, kbar, vbar, cnt, ws)
    assert bsa.bsa_device_status(ws) == 0
    # projection against fp64
    X = x.double().numpy().reshape(w.B * w.N, dm)
    Wn = W.double().numpy()
    Y = X @ Wn.T
    bound = _bound(X, Wn)
    got = torch.cat([t.float().cpu().reshape(w.B * w.N, w.H * w.d) for t in (q, k, v)], dim=1).double().numpy()
    err = np.abs(got - Y)
    assert (err <= bound).all(), float((err / bound).max())
    # pooling: bit for bit against the oracle's means of the written tensors
    for t, mean in ((q, qbar), (k, kbar), (v, vbar)):
        blk = w.q_block if t is q else w.k_block
        ref, rcnt = oracle.block_means(oracle.as_raw(t.cpu()), blk)
        assert np.array_equal(mean.cpu().numpy(), ref)
    assert np.array_equal(cnt.cpu().numpy(), rcnt)
    # the rest of the layer from the producer's outputs equals the plain path
    buf = bsa.Buffers(p, q.device)
    out_a = torch.empty_like(q)
    bsa.run_layer(p, q, k, v, out_a, buf)
    assert torch.equal(buf.qbar, qbar) and torch.equal(buf.kbar, kbar) and torch.equal(buf.vbar, vbar)


def test_qkv_pool_rejects_unsupported_shapes():
    q = torch.empty((1, 1000, 3, 128), dtype=torch.bfloat16, device="cuda")     # H * d = 384
    p = bsa.make_params(q)
    fake = torch.empty(64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_qkv_pool(p, torch.empty((1, 1000, 256), dtype=torch.bfloat16, device="cuda"), fake, q, q, q,
                         torch.empty(1, device="cuda"), torch.empty(1, device="cuda"), torch.empty(1, device="cuda"),
                         None)
    assert e.value.status == 2
