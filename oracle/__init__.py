"""CPU oracle for block-sparse "sol-attn" attention -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The library's own path never touches it.

The arithmetic lives in ``oracle.c`` (plain C, fp64 accumulation, OpenMP over
independent rows); this module compiles it with gcc, marshals numpy/torch CPU
arrays into it and composes the steps in the order the pages give them:
pool -> block scores -> select (+ forced blocks) -> extra tokens -> attention.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "_build", "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into a shared library (gcc, OpenMP)."""
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-mfma", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    P, I, L, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.orc_block_means.argtypes = [P, I, L, L, L, I, I, I, I, I, P, P]
    lib.orc_block_scores.argtypes = [P, P, I, I, I, I, P]
    lib.orc_forced_blocks.argtypes = [I, I, I, I, I, I, I, I, P]
    lib.orc_select.argtypes = [P, L, I, I, I, I, I, I, D, D, I, I, I, P, P]
    lib.orc_extra_tokens.argtypes = [P, P, I, L, L, L, I, I, I, I, I, I, P, I, P, L, P, P]
    lib.orc_attention_rows.argtypes = [P, P, P, I, L, L, L, I, I, I, I, I, I, P, P, P, P, P, P,
                                       I, I, I, I, P, L, P, P]
    for f in (lib.orc_block_means, lib.orc_block_scores, lib.orc_forced_blocks, lib.orc_select,
              lib.orc_extra_tokens, lib.orc_attention_rows):
        f.restype = ctypes.c_int
    _lib = lib
    return lib


def threads() -> int:
    """Threads OpenMP will use (OMP_NUM_THREADS, else the affinity mask)."""
    env = os.environ.get("OMP_NUM_THREADS")
    if env:
        return int(env)
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


# ------------------------------------------------------------------ inputs

@dataclass
class Raw:
    """A [B, N, H, d] tensor as raw CPU storage plus element strides."""
    arr: np.ndarray          # owning buffer (uint16 for bf16, float32 for f32)
    dtype: int               # 0 = bf16, 1 = f32
    sb: int
    sn: int
    sh: int
    B: int
    N: int
    H: int
    d: int

    @property
    def ptr(self):
        return self.arr.ctypes.data


def as_raw(t) -> Raw:
    """Wrap a torch CPU tensor of shape [B, N, H, d] (any strides, d contiguous)."""
    import torch
    assert t.device.type == "cpu" and t.dim() == 4 and t.stride(3) == 1
    B, N, H, d = t.shape
    # base storage as numpy without copying; strides in elements
    if t.dtype == torch.bfloat16:
        dtype = 0
    elif t.dtype == torch.float32:
        dtype = 1
    else:
        raise TypeError(f"unsupported dtype {t.dtype}")
    sb, sn, sh = t.stride(0), t.stride(1), t.stride(2)
    # span of storage touched by the view
    span = (B - 1) * sb + (N - 1) * sn + (H - 1) * sh + d
    base = t.as_strided((span,), (1,), t.storage_offset())
    if dtype == 0:
        arr = base.view(torch.int16).numpy().view(np.uint16)
    else:
        arr = base.numpy()
    return Raw(arr, dtype, sb, sn, sh, B, N, H, d)


def _c(a: np.ndarray, dt):
    a = np.ascontiguousarray(a, dtype=dt)
    return a, a.ctypes.data


# ------------------------------------------------------------------ steps

def block_means(x: Raw, blk: int):
    """Block means [B, H, nb, d] fp32 and block sizes [nb] (pooling step)."""
    lib = _load()
    nb = -(-x.N // blk)
    mean = np.empty((x.B, x.H, nb, x.d), np.float32)
    cnt = np.empty((nb,), np.int32)
    rc = lib.orc_block_means(x.ptr, x.dtype, x.sb, x.sn, x.sh, x.B, x.N, x.H, x.d, blk,
                             mean.ctypes.data, cnt.ctypes.data)
    assert rc == 0
    return mean, cnt


def block_scores(qbar: np.ndarray, kbar: np.ndarray):
    """Pooled block scores S [B, H, nQB, nKB] fp32."""
    lib = _load()
    B, H, nQB, d = qbar.shape
    nKB = kbar.shape[2]
    q, qp = _c(qbar, np.float32)
    k, kp = _c(kbar, np.float32)
    S = np.empty((B, H, nQB, nKB), np.float32)
    lib.orc_block_scores(qp, kp, B * H, nQB, nKB, d, S.ctypes.data)
    return S


def forced_blocks(i: int, nKB: int, N: int, Bq: int, Bk: int, sink_blocks: int,
                  prefix_len: int, keep_diag: int) -> np.ndarray:
    lib = _load()
    out = np.empty((nKB,), np.uint8)
    lib.orc_forced_blocks(i, nKB, N, Bq, Bk, sink_blocks, prefix_len, keep_diag, out.ctypes.data)
    return out


def select(S: np.ndarray, N: int, Bq: int, Bk: int, method: str, tau: float = 1.3,
           keep_percent: float = 10.0, sink_blocks: int = 1, prefix_len: int = 0,
           keep_diag: int = 1):
    """Kept-block mask [.., nQB, nKB] uint8 and per-row threshold (or k-th score)."""
    lib = _load()
    nQB, nKB = S.shape[-2], S.shape[-1]
    rows = int(np.prod(S.shape[:-1]))
    s, sp = _c(S, np.float32)
    keep = np.empty(S.shape, np.uint8)
    thr = np.empty(S.shape[:-1], np.float32)
    m = {"sol": 0, "sla": 1}[method]
    rc = lib.orc_select(sp, rows, nQB, nKB, N, Bq, Bk, m, float(tau), float(keep_percent),
                        sink_blocks, prefix_len, keep_diag, keep.ctypes.data, thr.ctypes.data)
    assert rc == 0
    return keep, thr


def extra_tokens(qbar: np.ndarray, k: Raw, keep: np.ndarray, Bq: int, Bk: int, E: int,
                 rows: Optional[Sequence[int]] = None):
    """Top-E extra tokens for the given rows (all rows if None).

    Returns (extra [R, E] int32 ascending, -1 padded; count [R] int32; rows [R]).
    """
    lib = _load()
    B, H, nQB, d = qbar.shape
    total = B * H * nQB
    rows = np.arange(total, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    q, qp = _c(qbar, np.float32)
    kp_, kp = _c(keep.reshape(total, -1), np.uint8)
    rr, rp = _c(rows, np.int64)
    extra = np.empty((len(rows), max(E, 1)), np.int32)
    cnt = np.empty((len(rows),), np.int32)
    lib.orc_extra_tokens(qp, k.ptr, k.dtype, k.sb, k.sn, k.sh, k.B, k.H, k.N, k.d, Bq, Bk, kp,
                         E, rp, len(rows), extra.ctypes.data, cnt.ctypes.data)
    return extra[:, :E], cnt, rows


def attention_rows(q: Raw, k: Raw, v: Raw, Bq: int, Bk: int, kbar, vbar, count, keep,
                   tokens: np.ndarray, extra=None, ecnt=None, centroid: int = 1,
                   dense_rows=(0, 0)):
    """Fine-pass outputs for query tokens `tokens` [m, 3] = (b, h, n).

    keep: [B*H*nQB, nKB] mask; extra/ecnt: full [B*H*nQB, E] / [B*H*nQB] tables
    (or None).  Returns (out [m, d] fp64, lse [m] fp64).
    """
    lib = _load()
    assert q.dtype == k.dtype == v.dtype and (q.sb, q.sn, q.sh) == (k.sb, k.sn, k.sh) == (v.sb, v.sn, v.sh)
    B, N, H, d = q.B, q.N, q.H, q.d
    nQB, nKB = -(-N // Bq), -(-N // Bk)
    kb, kbp = _c(kbar, np.float32)
    vb, vbp = _c(vbar, np.float32)
    ct, ctp = _c(count, np.int32)
    kp_, kpp = _c(np.asarray(keep).reshape(B * H * nQB, nKB), np.uint8)
    tk, tkp = _c(tokens, np.int64)
    if extra is not None and extra.shape[-1] > 0:
        E = extra.shape[-1]
        ex, exp_ = _c(extra.reshape(B * H * nQB, E), np.int32)
        ec, ecp = _c(ecnt.reshape(B * H * nQB), np.int32)
    else:
        E, exp_, ecp = 0, None, None
    m = tk.shape[0]
    out = np.empty((m, d), np.float64)
    lse = np.empty((m,), np.float64)
    rc = lib.orc_attention_rows(q.ptr, k.ptr, v.ptr, q.dtype, q.sb, q.sn, q.sh, B, H, N, d, Bq, Bk,
                                kbp, vbp, ctp, kpp, exp_, ecp, E, int(centroid),
                                int(dense_rows[0]), int(dense_rows[1]), tkp, m,
                                out.ctypes.data, lse.ctypes.data)
    assert rc == 0
    return out, lse


def cube_order(w) -> np.ndarray:
    """Block order of the tokens under 3-D cube tiling ("BlockSparseAttention -
    ComfyUI Built-in Node Documentation", vsa: 3-D video cube tiling): position p
    of the block-ordered sequence holds token cube_order(w)[p].  The packed
    prefix keeps its own order (its 64-token runs are blocks); then come the
    cubes of the T x Hs x Ws grid in t-major order, each cube's tokens t-major
    inside it."""
    P = w.prefix_len
    T, Hs, Ws = w.grid
    ct, cy, cx = w.cube
    order = list(range(P))
    for t0 in range(0, T, ct):
        for y0 in range(0, Hs, cy):
            for x0 in range(0, Ws, cx):
                for dt in range(ct):
                    for dy in range(cy):
                        for dx in range(cx):
                            order.append(P + ((t0 + dt) * Hs + (y0 + dy)) * Ws + (x0 + dx))
    return np.asarray(order, np.int64)


def reorder(x: Raw, order: np.ndarray) -> Raw:
    """The tokens of x taken in the given order, as a contiguous [B, N, H, d] Raw."""
    item = x.arr.itemsize
    full = np.lib.stride_tricks.as_strided(x.arr, shape=(x.B, x.N, x.H, x.d),
                                           strides=(x.sb * item, x.sn * item, x.sh * item, item))
    arr = np.ascontiguousarray(full[:, order])
    return Raw(arr.reshape(-1), x.dtype, x.N * x.H * x.d, x.H * x.d, x.d, x.B, x.N, x.H, x.d)


def mask_to_csr(keep: np.ndarray):
    """CSR (row_ptr [rows+1], col [nnz] ascending, count [rows]) of a 0/1 mask."""
    flat = keep.reshape(-1, keep.shape[-1]).astype(bool)
    count = flat.sum(axis=1).astype(np.int32)
    row_ptr = np.zeros(flat.shape[0] + 1, np.int64)
    np.cumsum(count, out=row_ptr[1:])
    col = np.nonzero(flat)[1].astype(np.int32)
    return row_ptr, col, count


# ------------------------------------------------------------------ composite

@dataclass
class LayerResult:
    qbar: np.ndarray
    kbar: np.ndarray
    vbar: np.ndarray
    count: np.ndarray
    S: np.ndarray
    keep: np.ndarray
    thr: np.ndarray
    extra: Optional[np.ndarray]
    ecnt: Optional[np.ndarray]
    order: Optional[np.ndarray] = None     # vsa: block-order position -> token


def routing(w, q: Raw, k: Raw, v: Raw, extra_rows: Optional[Sequence[int]] = None,
            with_extra: bool = True) -> LayerResult:
    """Pool, score, select and (if E > 0) pick extra tokens for workload `w`.

    extra_rows restricts the (expensive) extra-token search to those rows; the
    other rows get an empty list.

    Method "vsa" (the fine stage of the vsa method without its learned coarse
    branch): blocks are the cubes of cube_order; the top keep_percent % of key
    cubes per query cube are kept, with the sink and diagonal blocks, as SLA
    keeps blocks; pooled means and masks are in block order.
    """
    order = None
    method = w.method
    if w.method == "vsa":
        order = cube_order(w)
        q, k, v = reorder(q, order), reorder(k, order), reorder(v, order)
        method = "sla"
    qbar, _ = block_means(q, w.q_block)
    kbar, count = block_means(k, w.k_block)
    vbar, _ = block_means(v, w.k_block)
    S = block_scores(qbar, kbar)
    keep, thr = select(S, w.N, w.q_block, w.k_block, method, w.tau, w.keep_percent,
                       w.sink_blocks, w.prefix_len, w.keep_diag)
    extra = ecnt = None
    E = w.extra_tokens
    if E > 0 and with_extra:
        total = w.rows
        extra = np.full((total, E), -1, np.int32)
        ecnt = np.zeros((total,), np.int32)
        ex, ec, rows = extra_tokens(qbar, k, keep, w.q_block, w.k_block, E, extra_rows)
        extra[rows] = ex
        ecnt[rows] = ec
    return LayerResult(qbar, kbar, vbar, count, S, keep, thr, extra, ecnt, order)


def layer_rows(w, q: Raw, k: Raw, v: Raw, r: LayerResult, tokens: np.ndarray):
    """Final outputs (sparse + centroid, dense rows applied) for `tokens`
    ([m, 3] = (b, h, token))."""
    if r.order is not None:
        q, k, v = reorder(q, r.order), reorder(k, r.order), reorder(v, r.order)
        pos = np.empty_like(r.order)
        pos[r.order] = np.arange(len(r.order))
        tokens = tokens.copy()
        tokens[:, 2] = pos[tokens[:, 2]]
    return attention_rows(q, k, v, w.q_block, w.k_block, r.kbar, r.vbar, r.count,
                          r.keep.reshape(w.rows, w.nKB), tokens, r.extra, r.ecnt,
                          centroid=w.centroid, dense_rows=w.dense_rows)


def all_tokens(w) -> np.ndarray:
    b, h, n = np.meshgrid(np.arange(w.B), np.arange(w.H), np.arange(w.N), indexing="ij")
    return np.stack([b.ravel(), h.ravel(), n.ravel()], axis=1).astype(np.int64)


__all__ = ["build", "threads", "Raw", "as_raw", "block_means", "block_scores", "forced_blocks",
           "select", "extra_tokens", "attention_rows", "mask_to_csr", "routing", "layer_rows", "cube_order",
           "reorder",
           "all_tokens", "LayerResult"]
