"""ctypes binding of libbsa.so: argument marshalling only.

Every function here has the name of the C entry point it calls and takes
torch tensors (device memory) in place of raw pointers.  No step of the
method runs in Python; if the shared library cannot be loaded, importing this
module raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# BSA_LIBRARY may name another build of the same library (e.g. a debug build).
LIB_PATH = os.environ.get("BSA_LIBRARY") or os.path.join(_PKG, "libbsa.so")

BSA_OK = 0
BSA_ERR_INVALID_ARG = 1
BSA_ERR_UNSUPPORTED = 2
BSA_ERR_CAPACITY = 3
BSA_ERR_WORKSPACE = 4
BSA_ERR_CUDA = 5
BSA_ERR_DEVICE = 6

BSA_DT_BF16, BSA_DT_F32 = 0, 1
BSA_SOL, BSA_SLA, BSA_VSA = 0, 1, 2


class bsa_params(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32), ("d", ctypes.c_int32),
        ("stride_b", ctypes.c_int64), ("stride_n", ctypes.c_int64), ("stride_h", ctypes.c_int64),
        ("dtype", ctypes.c_int32), ("method", ctypes.c_int32),
        ("q_block", ctypes.c_int32), ("k_block", ctypes.c_int32),
        ("tau", ctypes.c_double), ("keep_percent", ctypes.c_double),
        ("sink_blocks", ctypes.c_int32), ("keep_diag", ctypes.c_int32),
        ("prefix_len", ctypes.c_int32),
        ("dense_row_begin", ctypes.c_int32), ("dense_row_end", ctypes.c_int32),
        ("extra_tokens", ctypes.c_int32), ("centroid", ctypes.c_int32),
        ("grid_t", ctypes.c_int32), ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32),
        ("cube_t", ctypes.c_int32), ("cube_h", ctypes.c_int32), ("cube_w", ctypes.c_int32),
        ("qk_fp8", ctypes.c_int32), ("modcent_per_row", ctypes.c_int32), ("pv_fp8", ctypes.c_int32),
    ]


class bsa_layer_device(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("out", ctypes.c_void_p),
        ("qbar", ctypes.c_void_p), ("kbar", ctypes.c_void_p), ("vbar", ctypes.c_void_p),
        ("blk_count", ctypes.c_void_p), ("row_ptr", ctypes.c_void_p), ("col_idx", ctypes.c_void_p),
        ("col_capacity", ctypes.c_int64), ("kept_count", ctypes.c_void_p),
        ("extra_idx", ctypes.c_void_p), ("extra_count", ctypes.c_void_p),
        ("ws", ctypes.c_void_p), ("ws_bytes", ctypes.c_size_t),
    ]


class bsa_policy(ctypes.Structure):
    _fields_ = [
        ("start_percent", ctypes.c_double), ("end_percent", ctypes.c_double),
        ("min_tokens", ctypes.c_int32), ("hybrid", ctypes.c_int32),
        ("hybrid_guard_steps", ctypes.c_int32), ("pad_", ctypes.c_int32),
        ("dense_blocks", ctypes.c_char_p),
    ]


BSA_RUN_SPARSE, BSA_DENSE_SHORT, BSA_DENSE_BLOCK, BSA_DENSE_HYBRID, BSA_DENSE_WINDOW = 0, 1, 2, 3, 4


class BsaError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: status {status} ({msg})")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libbsa.so not built at {LIB_PATH}; run python block_sparse_attention_26_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    PP = ctypes.POINTER(bsa_params)
    lib.bsa_default_params.argtypes = [PP, I32]
    lib.bsa_default_params.restype = None
    lib.bsa_workspace_size.argtypes = [PP, ctypes.POINTER(SZ), ctypes.POINTER(I64)]
    lib.bsa_pool.argtypes = [PP, P, P, P, P, P, P, P, P]
    lib.bsa_select.argtypes = [PP, P, P, P, P, P, I64, P, P, P, P, SZ, P]
    lib.bsa_qkv_pool.argtypes = [PP, P, I32, P, P, P, P, P, P, P, P, P, P]
    lib.bsa_select_static.argtypes = [PP, P, P, P, P, I64, P, P]
    lib.bsa_attention.argtypes = [PP, P, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
    lib.bsa_attention_prepare.argtypes = lib.bsa_attention.argtypes
    lib.bsa_attention_run.argtypes = lib.bsa_attention.argtypes
    lib.bsa_selftest_bounded_wait.argtypes = [P, I64, P]
    lib.bsa_launch_count.argtypes = []
    lib.bsa_launch_count.restype = I64
    lib.bsa_dense_ref_rows.argtypes = [PP, P, P, P, I32, I32, P, P, P, SZ, P]
    lib.bsa_layer_host.argtypes = [PP, P, P, P, P, ctypes.POINTER(bsa_layer_device), I32, P, P, P]
    lib.bsa_device_status.argtypes = [P, P, ctypes.POINTER(I32)]
    PolP = ctypes.POINTER(bsa_policy)
    lib.bsa_default_policy.argtypes = [PolP]
    lib.bsa_default_policy.restype = None
    lib.bsa_policy_decide.argtypes = [PolP, I32, I32, ctypes.c_double, I32, I32, ctypes.POINTER(I32)]
    lib.bsa_policy_decide.restype = I32
    lib.bsa_status_string.argtypes = [I32]
    lib.bsa_status_string.restype = ctypes.c_char_p
    lib.bsa_last_error.argtypes = []
    lib.bsa_last_error.restype = ctypes.c_char_p
    for f in ("bsa_workspace_size", "bsa_pool", "bsa_qkv_pool", "bsa_select", "bsa_select_static", "bsa_attention",
              "bsa_attention_prepare", "bsa_attention_run", "bsa_dense_ref_rows", "bsa_device_status",
              "bsa_selftest_bounded_wait", "bsa_layer_host"):
        getattr(lib, f).restype = I32
    return lib


lib = _load()

EXPORTED = ("bsa_default_params", "bsa_workspace_size", "bsa_pool", "bsa_qkv_pool", "bsa_select", "bsa_select_static",
            "bsa_attention", "bsa_attention_prepare", "bsa_attention_run", "bsa_dense_ref_rows",
            "bsa_device_status", "bsa_selftest_bounded_wait", "bsa_launch_count", "bsa_layer_host",
            "bsa_default_policy",
            "bsa_policy_decide",
            "bsa_status_string", "bsa_last_error")


def _check(status: int, where: str):
    if status != BSA_OK:
        msg = lib.bsa_last_error().decode() or lib.bsa_status_string(status).decode()
        raise BsaError(status, where, msg)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# ------------------------------------------------------------------ params

def make_params(q: torch.Tensor, method: str = "sol", *, q_block: Optional[int] = None,
                tau: float = 1.3, keep_percent: float = 10.0, sink_blocks: int = 1,
                keep_diag: int = 1, prefix_len: int = 0, dense_rows=(0, 0), extra_tokens: int = 0,
                centroid: Optional[int] = None, grid=None, cube=(4, 4, 4), qk_fp8: bool = False,
                modcent_per_row: int = 0, pv_fp8: bool = False) -> bsa_params:
    """Parameters for a [B, N, H, d] query tensor `q` (strides taken from q).
    method "vsa" needs `grid` = (T, Hs, Ws) of the tokens after the prefix."""
    m = {"sol": BSA_SOL, "sla": BSA_SLA, "vsa": BSA_VSA}[method]
    p = bsa_params()
    lib.bsa_default_params(ctypes.byref(p), m)
    B, N, H, d = q.shape
    p.B, p.H, p.N, p.d = B, H, N, d
    p.stride_b, p.stride_n, p.stride_h = q.stride(0), q.stride(1), q.stride(2)
    p.dtype = {torch.bfloat16: BSA_DT_BF16, torch.float32: BSA_DT_F32}[q.dtype]
    if q_block is not None:
        p.q_block = q_block
    p.tau = float(tau)
    p.keep_percent = float(keep_percent)
    p.sink_blocks, p.keep_diag, p.prefix_len = sink_blocks, keep_diag, prefix_len
    p.dense_row_begin, p.dense_row_end = dense_rows
    p.extra_tokens = extra_tokens
    if centroid is not None:
        p.centroid = centroid
    p.qk_fp8 = int(bool(qk_fp8))
    p.modcent_per_row = int(modcent_per_row)
    p.pv_fp8 = int(bool(pv_fp8))
    if m == BSA_VSA:
        if grid is None:
            raise ValueError("method vsa needs the latent grid (T, Hs, Ws)")
        p.grid_t, p.grid_h, p.grid_w = grid
        p.cube_t, p.cube_h, p.cube_w = cube
    return p


def params_for(w, q: torch.Tensor) -> bsa_params:
    """Parameters from any object carrying the method's fields (method, q_block,
    tau, keep_percent, sink_blocks, keep_diag, prefix_len, dense_rows,
    extra_tokens, centroid) for query tensor `q`."""
    return make_params(q, w.method, q_block=w.q_block, tau=w.tau, keep_percent=w.keep_percent,
                       sink_blocks=w.sink_blocks, keep_diag=w.keep_diag, prefix_len=w.prefix_len,
                       dense_rows=tuple(w.dense_rows), extra_tokens=w.extra_tokens, centroid=w.centroid,
                       grid=getattr(w, "grid", None), cube=getattr(w, "cube", (4, 4, 4)),
                       qk_fp8=getattr(w, "qk_fp8", False), modcent_per_row=getattr(w, "modcent_per_row", 0),
                       pv_fp8=getattr(w, "pv_fp8", False))


def dims(p: bsa_params):
    nQB = -(-p.N // p.q_block)
    nKB = -(-p.N // p.k_block)
    return nQB, nKB, p.B * p.H * nQB


# ------------------------------------------------------------------ entry points

def bsa_workspace_size(p: bsa_params):
    nbytes, nnz = ctypes.c_size_t(), ctypes.c_int64()
    _check(lib.bsa_workspace_size(ctypes.byref(p), ctypes.byref(nbytes), ctypes.byref(nnz)),
           "bsa_workspace_size")
    return nbytes.value, nnz.value


def bsa_pool(p, q, k, v, qbar, kbar, vbar, blk_count, stream=None):
    _check(lib.bsa_pool(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(qbar), _ptr(kbar), _ptr(vbar),
                        _ptr(blk_count), _stream(stream)), "bsa_pool")


def bsa_qkv_pool(p, x, w_qkv, q, k, v, qbar, kbar, vbar, blk_count, ws=None, stream=None):
    _check(lib.bsa_qkv_pool(ctypes.byref(p), _ptr(x), int(x.shape[-1]), _ptr(w_qkv), _ptr(q), _ptr(k), _ptr(v),
                            _ptr(qbar), _ptr(kbar), _ptr(vbar), _ptr(blk_count), _ptr(ws), _stream(stream)),
           "bsa_qkv_pool")


def bsa_select(p, qbar, kbar, k, row_ptr, col_idx, kept_count, extra_idx, extra_count, ws,
               stream=None):
    cap = 0 if col_idx is None else col_idx.numel()
    _check(lib.bsa_select(ctypes.byref(p), _ptr(qbar), _ptr(kbar), _ptr(k), _ptr(row_ptr), _ptr(col_idx),
                          cap, _ptr(kept_count), _ptr(extra_idx), _ptr(extra_count), _ptr(ws),
                          ws.numel() * ws.element_size(), _stream(stream)), "bsa_select")


def bsa_select_static(p, qbar, kbar, row_ptr, col_idx, kept_count, stream=None):
    cap = 0 if col_idx is None else col_idx.numel()
    _check(lib.bsa_select_static(ctypes.byref(p), _ptr(qbar), _ptr(kbar), _ptr(row_ptr), _ptr(col_idx), cap,
                                 _ptr(kept_count), _stream(stream)), "bsa_select_static")


def bsa_attention(p, q, k, v, kbar, vbar, blk_count, row_ptr, col_idx, extra_idx, extra_count, out,
                  lse, ws, stream=None):
    _check(lib.bsa_attention(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(kbar), _ptr(vbar),
                             _ptr(blk_count), _ptr(row_ptr), _ptr(col_idx), _ptr(extra_idx),
                             _ptr(extra_count), _ptr(out), _ptr(lse), _ptr(ws),
                             ws.numel() * ws.element_size(), _stream(stream)), "bsa_attention")


def bsa_attention_prepare(p, q, k, v, kbar, vbar, blk_count, row_ptr, col_idx, extra_idx, extra_count, out,
                          lse, ws, stream=None):
    _check(lib.bsa_attention_prepare(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(kbar), _ptr(vbar),
                                     _ptr(blk_count), _ptr(row_ptr), _ptr(col_idx), _ptr(extra_idx),
                                     _ptr(extra_count), _ptr(out), _ptr(lse), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)), "bsa_attention_prepare")


def bsa_attention_run(p, q, k, v, kbar, vbar, blk_count, row_ptr, col_idx, extra_idx, extra_count, out,
                      lse, ws, stream=None):
    _check(lib.bsa_attention_run(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(kbar), _ptr(vbar),
                                 _ptr(blk_count), _ptr(row_ptr), _ptr(col_idx), _ptr(extra_idx),
                                 _ptr(extra_count), _ptr(out), _ptr(lse), _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream(stream)), "bsa_attention_run")


def bsa_launch_count() -> int:
    """Kernels the library has launched since it was loaded."""
    return int(lib.bsa_launch_count())


def bsa_selftest_bounded_wait(ws, cycles: int, stream=None):
    _check(lib.bsa_selftest_bounded_wait(_ptr(ws), int(cycles), _stream(stream)), "bsa_selftest_bounded_wait")


def bsa_dense_ref_rows(p, q, k, v, row_begin, row_end, out, lse, ws, stream=None):
    _check(lib.bsa_dense_ref_rows(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), int(row_begin),
                                  int(row_end), _ptr(out), _ptr(lse), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream)),
           "bsa_dense_ref_rows")


def bsa_device_status(ws, stream=None) -> int:
    code = ctypes.c_int32()
    _check(lib.bsa_device_status(_ptr(ws), _stream(stream), ctypes.byref(code)), "bsa_device_status")
    return code.value


def make_policy(start_percent: float = 0.2, end_percent: float = 1.0, min_tokens: int = 12288,
                hybrid: bool = False, hybrid_guard_steps: int = 1, dense_blocks: str = "") -> bsa_policy:
    pol = bsa_policy()
    lib.bsa_default_policy(ctypes.byref(pol))
    pol.start_percent, pol.end_percent = float(start_percent), float(end_percent)
    pol.min_tokens, pol.hybrid, pol.hybrid_guard_steps = int(min_tokens), int(bool(hybrid)), int(hybrid_guard_steps)
    pol._dense_blocks_bytes = dense_blocks.encode()      # kept alive with the struct
    pol.dense_blocks = pol._dense_blocks_bytes
    return pol


def bsa_policy_decide(pol: bsa_policy, n_tokens: int, block_index: int, progress: float, step: int = -1,
                      n_steps: int = 0) -> int:
    out = ctypes.c_int32()
    _check(lib.bsa_policy_decide(ctypes.byref(pol), int(n_tokens), int(block_index), float(progress), int(step),
                                 int(n_steps), ctypes.byref(out)), "bsa_policy_decide")
    return out.value


# ------------------------------------------------------------------ buffers

class Buffers:
    """Device buffers for one layer of a given parameter set (allocated by torch)."""

    def __init__(self, p: bsa_params, device, capacity: Optional[int] = None):
        nQB, nKB, rows = dims(p)
        BH, d = p.B * p.H, p.d
        f32, i32 = torch.float32, torch.int32
        self.qbar = torch.empty((p.B, p.H, nQB, d), dtype=f32, device=device)
        self.kbar = torch.empty((p.B, p.H, nKB, d), dtype=f32, device=device)
        self.vbar = torch.empty((p.B, p.H, nKB, d), dtype=f32, device=device)
        self.blk_count = torch.empty((nKB,), dtype=i32, device=device)
        self.row_ptr = torch.empty((rows + 1,), dtype=torch.int64, device=device)
        ws_bytes, max_nnz = bsa_workspace_size(p)
        if capacity is None:
            capacity = max_nnz
        self.col_idx = torch.empty((max(capacity, 1),), dtype=i32, device=device)
        self.kept_count = torch.empty((rows,), dtype=i32, device=device)
        E = p.extra_tokens
        self.extra_idx = torch.empty((rows, E), dtype=i32, device=device) if E > 0 else None
        self.extra_count = torch.empty((rows,), dtype=i32, device=device) if E > 0 else None
        self.ws = torch.zeros((ws_bytes + 255) // 256 * 256, dtype=torch.uint8, device=device)
        self.lse = torch.empty((p.B, p.H, p.N), dtype=f32, device=device)
        del BH


class HostLayer:
    """Device buffers for bsa_layer_host: the whole layer's Q, K, V and O
    ([B, N, H, d], contiguous, as p's strides must be) and one chunk's buffers
    (heads_per_chunk heads; 0: about a sixteenth of them, as the library chooses)."""

    def __init__(self, p: bsa_params, device, heads_per_chunk: int = 0):
        if (p.stride_h, p.stride_n, p.stride_b) != (p.d, p.H * p.d, p.N * p.H * p.d):
            raise ValueError("HostLayer needs contiguous [B, N, H, d] strides")
        hc = heads_per_chunk if heads_per_chunk > 0 else max(1, (p.H + 15) // 16)
        self.hc = min(hc, p.H)
        dt = torch.bfloat16 if p.dtype == BSA_DT_BF16 else torch.float32
        shape = (p.B, p.N, p.H, p.d)
        self.q, self.k, self.v, self.out = (torch.empty(shape, dtype=dt, device=device) for _ in range(4))
        pc = bsa_params.from_buffer_copy(p)
        pc.H = self.hc
        self.buf = Buffers(pc, device)
        b = self.buf
        self.dev = bsa_layer_device(
            _vp(self.q), _vp(self.k), _vp(self.v), _vp(self.out), _vp(b.qbar), _vp(b.kbar), _vp(b.vbar),
            _vp(b.blk_count), _vp(b.row_ptr), _vp(b.col_idx), b.col_idx.numel(), _vp(b.kept_count),
            _vp(b.extra_idx), _vp(b.extra_count), _vp(b.ws), b.ws.numel())


def _vp(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def bsa_layer_host(p: bsa_params, q_host, k_host, v_host, out_host, hl: HostLayer, stream=None,
                   copy_in=None, copy_out=None):
    """One layer from pinned host tensors (bsa_layer_host); copy_in / copy_out are
    torch streams for the copies (None: everything on `stream`)."""
    cin = None if copy_in is None else ctypes.c_void_p(copy_in.cuda_stream)
    cout = None if copy_out is None else ctypes.c_void_p(copy_out.cuda_stream)
    _check(lib.bsa_layer_host(ctypes.byref(p), _ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(out_host),
                              ctypes.byref(hl.dev), hl.hc, _stream(stream), cin, cout), "bsa_layer_host")


def run_step(p: bsa_params, pol: bsa_policy, q, k, v, out, buf: Buffers, block_index: int, progress: float,
             step: int = -1, n_steps: int = 0, stream=None, lse: bool = True) -> int:
    """One attention call under the per-step policy: the sparse hot path, or
    dense attention over every row; returns the bsa_decision taken."""
    decision = bsa_policy_decide(pol, p.N, block_index, progress, step, n_steps)
    if decision == BSA_RUN_SPARSE:
        run_layer(p, q, k, v, out, buf, stream, lse)
    else:
        bsa_dense_ref_rows(p, q, k, v, 0, p.N, out, buf.lse if lse else None, buf.ws, stream)
    return decision


def run_layer(p: bsa_params, q, k, v, out, buf: Buffers, stream=None, lse: bool = True):
    """The whole hot path for one layer: pool -> select -> attention (+ dense rows)."""
    bsa_pool(p, q, k, v, buf.qbar, buf.kbar, buf.vbar, buf.blk_count, stream)
    bsa_select(p, buf.qbar, buf.kbar, k, buf.row_ptr, buf.col_idx, buf.kept_count, buf.extra_idx,
               buf.extra_count, buf.ws, stream)
    bsa_attention(p, q, k, v, buf.kbar, buf.vbar, buf.blk_count, buf.row_ptr, buf.col_idx,
                  buf.extra_idx, buf.extra_count, out, buf.lse if lse else None, buf.ws, stream)
