"""Host-only checks of the C ABI: the library loads, exports every entry point
that include/bsa.h declares, and rejects bad arguments before any launch.

Nothing here touches a GPU: every call below fails host-side validation, which
runs before the library makes any CUDA call.
"""
import ctypes
import math
import os
import re

import pytest
import torch

import block_sparse_attention_26_b200 as bsa
from block_sparse_attention_26_b200 import binding

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "bsa.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"BSA_API\s+[\w\s\*]*?\b(bsa_\w+)\s*\(", text)))


def test_header_declarations_are_exported():
    names = _declared()
    assert len(names) >= 9
    for n in names:
        assert hasattr(bsa.lib, n), n          # ctypes resolves the symbol or raises
    assert sorted(bsa.EXPORTED) == names


def test_params_struct_layout():
    # int32 x4, int64 x3, int32 x4, double x2, int32 x15 (+4 padding)
    assert ctypes.sizeof(bsa.bsa_params) == 136
    assert bsa.bsa_params.tau.offset == 56
    assert bsa.bsa_params.centroid.offset == 96
    assert bsa.bsa_params.grid_t.offset == 100
    assert bsa.bsa_params.cube_w.offset == 120
    assert bsa.bsa_params.qk_fp8.offset == 124
    assert bsa.bsa_params.modcent_per_row.offset == 128
    assert bsa.bsa_params.pv_fp8.offset == 132


def _p(**kw):
    q = torch.empty((1, 1000, 2, 128), dtype=torch.bfloat16)
    p = bsa.make_params(q)
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def _status(fn, *args):
    return fn(*args)


FAKE = ctypes.c_void_p(1 << 20)          # aligned, never dereferenced (validation fails first)


@pytest.mark.parametrize("field,value,code", [
    ("d", 96, binding.BSA_ERR_UNSUPPORTED),
    ("d", 256, binding.BSA_ERR_UNSUPPORTED),
    ("N", 0, binding.BSA_ERR_INVALID_ARG),
    ("H", 0, binding.BSA_ERR_INVALID_ARG),
    ("dtype", 7, binding.BSA_ERR_INVALID_ARG),
    ("method", 2, binding.BSA_ERR_UNSUPPORTED),
    ("k_block", 128, binding.BSA_ERR_UNSUPPORTED),
    ("q_block", 32, binding.BSA_ERR_UNSUPPORTED),
    ("stride_n", 100, binding.BSA_ERR_INVALID_ARG),
    ("stride_h", 0, binding.BSA_ERR_INVALID_ARG),
    ("stride_h", 64, binding.BSA_ERR_INVALID_ARG),
    ("tau", math.nan, binding.BSA_ERR_INVALID_ARG),
    ("prefix_len", 1001, binding.BSA_ERR_INVALID_ARG),
    ("dense_row_end", 2000, binding.BSA_ERR_INVALID_ARG),
    ("extra_tokens", 300, binding.BSA_ERR_INVALID_ARG),
    ("sink_blocks", -1, binding.BSA_ERR_INVALID_ARG),
    ("centroid", 2, binding.BSA_ERR_INVALID_ARG),
    ("modcent_per_row", -1, binding.BSA_ERR_INVALID_ARG),
    ("pv_fp8", 2, binding.BSA_ERR_INVALID_ARG),
    ("pv_fp8", 1, binding.BSA_ERR_UNSUPPORTED),             # needs qk_fp8
])
def test_bad_params_rejected(field, value, code):
    p = _p(**{field: value})
    nbytes, nnz = ctypes.c_size_t(), ctypes.c_int64()
    st = bsa.lib.bsa_workspace_size(ctypes.byref(p), ctypes.byref(nbytes), ctypes.byref(nnz))
    assert st == code, bsa.lib.bsa_last_error()
    assert bsa.lib.bsa_last_error().decode() != ""


def test_sla_keep_percent_range():
    p = _p(method=binding.BSA_SLA, q_block=128, keep_percent=0.0)
    assert bsa.lib.bsa_workspace_size(ctypes.byref(p), ctypes.byref(ctypes.c_size_t()), None) == \
        binding.BSA_ERR_INVALID_ARG
    p.keep_percent = 100.0
    assert bsa.lib.bsa_workspace_size(ctypes.byref(p), ctypes.byref(ctypes.c_size_t()), None) == binding.BSA_OK


def test_workspace_size_and_capacity():
    p = _p()
    nbytes, nnz = bsa.bsa_workspace_size(p)
    nQB, nKB, rows = bsa.dims(p)
    assert (nQB, nKB, rows) == (16, 16, 32)
    assert nnz == rows * nKB
    assert nbytes >= rows * nKB * 4            # block-score scratch


def test_null_pointers_rejected():
    p = _p()
    st = bsa.lib.bsa_pool(ctypes.byref(p), None, FAKE, FAKE, FAKE, FAKE, FAKE, None, None)
    assert st == binding.BSA_ERR_INVALID_ARG
    assert b"q is NULL" in bsa.lib.bsa_last_error()
    st = bsa.lib.bsa_attention(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, None,
                               None, FAKE, None, FAKE, 1 << 30, None)
    assert st == binding.BSA_ERR_INVALID_ARG


def test_misaligned_pointer_rejected():
    p = _p()
    bad = ctypes.c_void_p((1 << 20) + 8)
    st = bsa.lib.bsa_pool(ctypes.byref(p), FAKE, bad, FAKE, FAKE, FAKE, FAKE, None, None)
    assert st == binding.BSA_ERR_INVALID_ARG
    assert b"aligned" in bsa.lib.bsa_last_error()


def test_workspace_checks():
    p = _p()
    nbytes, _ = bsa.bsa_workspace_size(p)
    st = bsa.lib.bsa_select(ctypes.byref(p), FAKE, FAKE, None, FAKE, FAKE, 10, FAKE, None, None, None, 0,
                            None)
    assert st == binding.BSA_ERR_WORKSPACE
    st = bsa.lib.bsa_select(ctypes.byref(p), FAKE, FAKE, None, FAKE, FAKE, 10, FAKE, None, None, FAKE,
                            nbytes - 1, None)
    assert st == binding.BSA_ERR_WORKSPACE
    st = bsa.lib.bsa_select(ctypes.byref(p), FAKE, FAKE, None, FAKE, FAKE, -1, FAKE, None, None, FAKE,
                            nbytes, None)
    assert st == binding.BSA_ERR_INVALID_ARG


def test_dense_rows_range_checked():
    p = _p()
    nbytes, _ = bsa.bsa_workspace_size(p)
    st = bsa.lib.bsa_dense_ref_rows(ctypes.byref(p), FAKE, FAKE, FAKE, 10, 5, FAKE, None, FAKE, nbytes, None)
    assert st == binding.BSA_ERR_INVALID_ARG
    st = bsa.lib.bsa_dense_ref_rows(ctypes.byref(p), FAKE, FAKE, FAKE, 0, 1001, FAKE, None, FAKE, nbytes,
                                    None)
    assert st == binding.BSA_ERR_INVALID_ARG


def test_status_strings():
    for s in range(7):
        assert bsa.lib.bsa_status_string(s)
    assert bsa.lib.bsa_device_status(None, None, None) == binding.BSA_ERR_INVALID_ARG


def test_binding_raises_on_error():
    p = _p(d=96)
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_workspace_size(p)
    assert e.value.status == binding.BSA_ERR_UNSUPPORTED


def test_defaults_follow_node_documentation():
    p = bsa.bsa_params()
    bsa.lib.bsa_default_params(ctypes.byref(p), binding.BSA_SOL)
    assert (p.tau, p.q_block, p.k_block, p.centroid, p.sink_blocks, p.keep_diag) == (1.3, 64, 64, 1, 1, 1)
    bsa.lib.bsa_default_params(ctypes.byref(p), binding.BSA_SLA)
    assert (p.keep_percent, p.q_block, p.centroid) == (10.0, 128, 0)


def test_modified_centroid_capacity_sizes_the_workspace():
    """The modified centroids take rows x modcent_per_row entries (0: min(E, nKB)
    per row), and the selection's scratch shares its bytes with the attention
    calls': on the 76k-token, 40-head workload with 256 extra tokens and 88
    entries per query block the workspace stays under 2.5 GB."""
    from workloads import CONFIGS
    w = CONFIGS["sol_sinks"]
    q = torch.empty((w.B, w.N, w.H, w.d), dtype=torch.bfloat16, device="meta")
    p = bsa.params_for(w, q)
    assert p.modcent_per_row == 88
    tight, _ = bsa.bsa_workspace_size(p)
    assert tight <= 2.5e9
    p.modcent_per_row = 0
    worst, _ = bsa.bsa_workspace_size(p)
    p.modcent_per_row = 10_000                 # more than min(E, nKB) = 256: the worst case
    assert bsa.bsa_workspace_size(p)[0] == worst
    # 2 (K and V) x 128 channels x 2 bytes, plus the bias, the slot and the mask, per entry
    entries = w.rows * (256 - 88)
    assert worst - tight >= entries * (2 * 128 * 2 + 4 + 4 + 8) - 4096


def test_layer_host_arguments_checked():
    """bsa_layer_host rejects missing arrays, a layout whose heads are not side by
    side, and a negative chunk size before doing anything."""
    p = _p()
    dev = binding.bsa_layer_device()
    st = bsa.lib.bsa_layer_host(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None, 0, None, None, None)
    assert st == binding.BSA_ERR_INVALID_ARG
    st = bsa.lib.bsa_layer_host(ctypes.byref(p), None, FAKE, FAKE, FAKE, ctypes.byref(dev), 0, None, None, None)
    assert st == binding.BSA_ERR_INVALID_ARG
    st = bsa.lib.bsa_layer_host(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, ctypes.byref(dev), -1, None, None, None)
    assert st == binding.BSA_ERR_INVALID_ARG
    p.stride_h, p.stride_n = p.N * p.d, p.d           # [B, H, N, d] storage
    st = bsa.lib.bsa_layer_host(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, ctypes.byref(dev), 0, None, None, None)
    assert st == binding.BSA_ERR_INVALID_ARG
    assert bsa.lib.bsa_last_error().decode() != ""
