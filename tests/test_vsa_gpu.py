"""GPU parity of cube tiling (method vsa: "BlockSparseAttention - ComfyUI
Built-in Node Documentation", vsa: 3-D video cube tiling; the fine stage
without the learned coarse branch) against the CPU oracle.

Pooled means are compared bit for bit in block order (prefix blocks, then the
grid's cubes), masks row by row (top-k exemption for near-ties at the k-th
score), outputs element by element in token order.
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_26_b200 as bsa
import oracle
from tests.gpu_helpers import compare_masks, compare_outputs, csr_to_mask, gpu_layer
from workloads import Workload, make_qkv

pytestmark = pytest.mark.gpu

CASES = {
    "vsa_plain": Workload("vsa_plain", B=1, H=2, N=2048, d=128, dtype="bf16", method="vsa", q_block=64, k_block=64,
                          keep_percent=20.0, centroid=0, grid=(4, 16, 32), seed=81),
    "vsa_prefix_dense": Workload("vsa_prefix_dense", B=1, H=2, N=128 + 960, d=64, dtype="bf16", method="vsa",
                                 q_block=64, k_block=64, keep_percent=15.0, centroid=0, prefix_len=128,
                                 dense_rows=(64, 128), grid=(4, 12, 20), seed=82),
    "vsa_flat_cubes": Workload("vsa_flat_cubes", B=1, H=3, N=2 * 32 * 48, d=128, dtype="bf16", method="vsa",
                               q_block=64, k_block=64, keep_percent=10.0, centroid=0, grid=(2, 32, 48),
                               cube=(1, 8, 8), seed=83),
    "vsa_keep_all": Workload("vsa_keep_all", B=1, H=2, N=64 + 1024, d=128, dtype="bf16", method="vsa",
                             q_block=64, k_block=64, keep_percent=100.0, centroid=0, prefix_len=64,
                             grid=(4, 16, 16), seed=84),
    "vsa_f32": Workload("vsa_f32", B=1, H=2, N=1024, d=64, dtype="f32", method="vsa", q_block=64, k_block=64,
                        keep_percent=25.0, centroid=0, grid=(4, 16, 16), seed=85),
}


@pytest.mark.parametrize("name", list(CASES))
def test_vsa_matches_oracle(name):
    w = CASES[name]
    qc, kc, vc = make_qkv(w, "cpu")
    p, buf, out, status = gpu_layer(w, qc.cuda(), kc.cuda(), vc.cuda())
    assert status == 0
    raw = [oracle.as_raw(t) for t in (qc, kc, vc)]
    res = oracle.routing(w, *raw)
    assert np.array_equal(buf.qbar.cpu().numpy(), res.qbar)
    assert np.array_equal(buf.kbar.cpu().numpy(), res.kbar)
    assert np.array_equal(buf.vbar.cpu().numpy(), res.vbar)
    mask = csr_to_mask(buf.row_ptr, buf.col_idx, w.rows, w.nKB)
    exempt = compare_masks(mask, res, w)
    assert exempt <= max(1, w.rows // 1000), exempt
    ref, ref_lse = oracle.layer_rows(w, *raw, res, oracle.all_tokens(w))
    got = out.float().cpu().permute(0, 2, 1, 3).reshape(-1, w.d).numpy()
    compare_outputs(got, ref, name)
    lse = buf.lse.cpu().numpy().reshape(-1)
    assert np.abs(lse - ref_lse).max() < 2e-2


def test_vsa_rejects_grids_that_cubes_do_not_tile():
    q = torch.empty((1, 1000, 2, 128), dtype=torch.bfloat16, device="cuda")
    for grid, prefix in (((5, 10, 20), 0), ((4, 10, 25), 0), ((4, 12, 20), 40)):
        p = bsa.make_params(q, "vsa", grid=grid, prefix_len=prefix, centroid=0)
        with pytest.raises(bsa.BsaError):
            bsa.bsa_workspace_size(p)
