"""bsa_select_static: kept-block selection for callers that cannot allocate.

Some callers of this library cannot call cudaMalloc at all -- a host framework
that owns every device allocation, a plugin that is not allowed to allocate on
its host's streams, a server that must not allocate while it serves requests.
bsa_select_static() keeps its scratch in a fixed device array inside the
library instead of a caller-provided workspace.  These tests call it through
the C ABI and check that it returns exactly what bsa_select (with a
workspace) returns, on two calls in a row (the array keeps the previous call's
contents), and that problems larger than the array are refused up front.

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import pytest
import torch

import block_sparse_attention_26_b200 as bsa
from block_sparse_attention_26_b200 import binding
from workloads import Workload, make_qkv


def _problem(w):
    q, k, v = make_qkv(w, "cpu")
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    p = bsa.params_for(w, q)
    buf = bsa.Buffers(p, q.device)
    bsa.bsa_pool(p, q, k, v, buf.qbar, buf.kbar, buf.vbar, buf.blk_count)
    bsa.bsa_select(p, buf.qbar, buf.kbar, k, buf.row_ptr, buf.col_idx, buf.kept_count, None, None, buf.ws)
    assert bsa.bsa_device_status(buf.ws) == 0
    return p, buf


def _static_call(p, buf, rows, cap):
    row_ptr = torch.full((rows + 1,), -7, dtype=torch.int64, device="cuda")
    col = torch.full((cap,), -7, dtype=torch.int32, device="cuda")
    kept = torch.full((rows,), -7, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    st = bsa.lib.bsa_select_static(ctypes.byref(p), ctypes.c_void_p(buf.qbar.data_ptr()),
                                   ctypes.c_void_p(buf.kbar.data_ptr()), ctypes.c_void_p(row_ptr.data_ptr()),
                                   ctypes.c_void_p(col.data_ptr()), cap, ctypes.c_void_p(kept.data_ptr()),
                                   ctypes.c_void_p(stream.cuda_stream))
    assert st == binding.BSA_OK, bsa.lib.bsa_last_error()
    torch.cuda.synchronize()
    return row_ptr, col, kept


CASES = [
    Workload("static_sol", B=1, H=3, N=3000, d=128, dtype="bf16", method="sol", q_block=64, k_block=64,
             tau=1.3, grid=(3, 20, 50), seed=41),
    Workload("static_sla", B=1, H=2, N=2880, d=128, dtype="bf16", method="sla", q_block=128, k_block=64,
             keep_percent=15.0, centroid=0, grid=(4, 24, 30), seed=42),
]


@pytest.mark.gpu
@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_static_select_matches_workspace_select(w):
    p, buf = _problem(w)
    nQB, nKB, rows = bsa.dims(p)
    ref_ptr = buf.row_ptr.cpu()
    nnz = int(ref_ptr[-1])
    ref_col = buf.col_idx[:nnz].cpu()
    ref_kept = buf.kept_count.cpu()
    for _ in range(2):                       # the second call sees the first call's leftovers
        row_ptr, col, kept = _static_call(p, buf, rows, rows * nKB)
        assert torch.equal(row_ptr.cpu(), ref_ptr)
        assert torch.equal(col[:nnz].cpu(), ref_col)
        assert torch.equal(kept.cpu(), ref_kept)


@pytest.mark.gpu
def test_static_select_refuses_oversized_problems():
    q = torch.empty((1, 207872, 40, 128), dtype=torch.bfloat16, device="meta")
    p = bsa.make_params(q, "sol")
    fake = ctypes.c_void_p(1 << 20)
    st = bsa.lib.bsa_select_static(ctypes.byref(p), fake, fake, fake, fake, 1, fake, None)
    assert st == binding.BSA_ERR_CAPACITY
    assert b"static array" in bsa.lib.bsa_last_error()
