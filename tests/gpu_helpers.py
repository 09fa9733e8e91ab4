"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
(via the ctypes binding) and compare with the CPU oracle on the same inputs."""
import numpy as np
import torch

import block_sparse_attention_26_b200 as bsa
import oracle

# Acceptance bars for outputs from bf16 inputs (and, with the same numbers,
# for the f32 case whose fine pass rounds operands to bf16).
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
# Near-threshold exemption: a block whose score lies within this relative
# distance of its row's threshold (Sol) or k-th score (SLA) may differ.
EXEMPT_REL = 1e-5


params_for = bsa.params_for


def gpu_layer(w, q, k, v, capacity=None):
    """One pass of the whole hot path on the GPU; returns (params, buffers, out, device status)."""
    p = params_for(w, q)
    buf = bsa.Buffers(p, q.device, capacity)
    out = torch.empty_like(q)
    bsa.run_layer(p, q, k, v, out, buf)
    status = bsa.bsa_device_status(buf.ws)
    return p, buf, out, status


def csr_to_mask(row_ptr: torch.Tensor, col: torch.Tensor, rows: int, nKB: int) -> np.ndarray:
    rp = row_ptr.cpu().numpy()
    cl = col.cpu().numpy()
    mask = np.zeros((rows, nKB), np.uint8)
    for r in range(rows):
        c = cl[rp[r]:rp[r + 1]]
        assert np.all(np.diff(c) > 0), f"row {r}: columns not strictly ascending"
        mask[r, c] = 1
    return mask


def compare_masks(gpu_mask: np.ndarray, res, w) -> int:
    """Masks must agree bit for bit except for near-threshold blocks; returns the
    number of exempted differences."""
    ora = res.keep.reshape(w.rows, w.nKB)
    diff = np.argwhere(gpu_mask != ora)
    if len(diff) == 0:
        return 0
    S = res.S.reshape(w.rows, w.nKB).astype(np.float64)
    thr = res.thr.reshape(w.rows).astype(np.float64)
    bad = []
    for r, j in diff:
        if abs(S[r, j] - thr[r]) > EXEMPT_REL * abs(thr[r]):
            bad.append((int(r), int(j), float(S[r, j]), float(thr[r])))
    assert not bad, f"{len(bad)} mask differences outside the exemption band, e.g. {bad[:5]}"
    return len(diff)


def to_cpu_raw(t: torch.Tensor):
    return oracle.as_raw(t.cpu())


def compare_outputs(out_gpu: np.ndarray, out_ref: np.ndarray, what: str = "out"):
    err = np.abs(out_gpu.astype(np.float64) - out_ref)
    assert np.isfinite(out_gpu).all(), f"{what}: non-finite values"
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= MAX_ABS, f"{what}: max abs err {mx:.3e} > {MAX_ABS}"
    assert mean <= MEAN_ABS, f"{what}: mean abs err {mean:.3e} > {MEAN_ABS}"
    return mx, mean
