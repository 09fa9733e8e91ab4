"""Seeded synthetic workloads for block-sparse "sol-attn" attention.

This module only draws inputs. It holds none of the method's arithmetic
(no pooling, scoring, selection or attention), so that both the CPU oracle
and the CUDA path can consume the very same tensors.

Token order follows the MiniMax-H3 packing described on the ComfyUI
BlockSparseAttention node page (``sink_conditioning`` row): the packed
conditioning rows come first, then the video latent grid flattened t-major
(t, y, x) in row-major order.

Field recipe (the pages give no activations, so these stand in for them):
  * for every (head, channel) white noise on the latent grid T x Hs x Ws is
    smoothed by a periodic Gaussian filter of sigma = 4 tokens per axis
    (applied in the Fourier domain) and normalised to unit standard deviation;
  * Q = F + 0.5 * eps_Q and K = F + 0.5 * eps_K share that field F, which gives
    video attention its local structure; V = eps_V ~ N(0, 1);
  * packed conditioning rows (the prefix) are i.i.d. N(0, 1) for Q, K and V;
  * bf16 inputs are produced by a round-to-nearest-even cast of the fp32 draw.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One problem instance: shapes, dtype and the method's parameters."""

    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str                      # "bf16" | "f32"
    method: str                     # "sol" | "sla" | "vsa"
    q_block: int
    k_block: int
    tau: float = 1.3
    keep_percent: float = 10.0
    sink_blocks: int = 1
    keep_diag: int = 1
    prefix_len: int = 0
    dense_rows: Tuple[int, int] = (0, 0)
    extra_tokens: int = 0
    centroid: int = 1
    grid: Optional[Tuple[int, int, int]] = None   # latent grid (T, Hs, Ws); None = iid tokens
    cube: Tuple[int, int, int] = (4, 4, 4)         # vsa: cube extents (t, y, x)
    qk_fp8: bool = False                           # fine pass with S = Q K^T in fp8 (e4m3)
    modcent_per_row: int = 0                       # modified-centroid capacity per query block (0: worst case)
    pv_fp8: bool = False                           # with qk_fp8: P V in fp8 (e4m3) as well
    seed: int = 0
    field_sigma: float = 4.0
    noise: float = 0.5

    @property
    def nQB(self) -> int:
        return -(-self.N // self.q_block)

    @property
    def nKB(self) -> int:
        return -(-self.N // self.k_block)

    @property
    def rows(self) -> int:
        return self.B * self.H * self.nQB

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five problem sizes of the headline measurement, plus their parameters.
TINY_SOL = Workload("tiny_sol", B=1, H=2, N=1024, d=64, dtype="f32", method="sol",
                    q_block=64, k_block=64, tau=1.0, sink_blocks=1, keep_diag=1,
                    centroid=1, grid=None, seed=1000)
SOL_MID = Workload("sol_mid", B=1, H=24, N=16384, d=128, dtype="bf16", method="sol",
                   q_block=64, k_block=64, tau=1.3, centroid=1, grid=(8, 32, 64), seed=2000)
SLA_TOPK = Workload("sla_topk", B=1, H=24, N=46080, d=128, dtype="bf16", method="sla",
                    q_block=128, k_block=64, keep_percent=15.0, centroid=0,
                    grid=(12, 48, 80), seed=3000)
SOL_SINKS = Workload("sol_sinks", B=1, H=40, N=76112, d=128, dtype="bf16", method="sol",
                     q_block=64, k_block=64, tau=1.3, prefix_len=512, dense_rows=(256, 512),
                     extra_tokens=256, centroid=1, grid=(21, 45, 80), seed=4000,
                     modcent_per_row=88)   # these inputs need 83.9 per query block on average
LONG = Workload("long", B=1, H=40, N=207872, d=128, dtype="bf16", method="sol",
                q_block=64, k_block=64, tau=1.5, prefix_len=512, dense_rows=(256, 512),
                extra_tokens=0, centroid=1, grid=(24, 90, 96), seed=5000)

# Cube tiling (the vsa method's fine stage without its learned coarse branch)
# on the SLA workload's grid, whose extents are multiples of 4; keep_percent 10,
# the value the FastH3-VSA checkpoint is trained at.
VSA_CUBES = Workload("vsa_cubes", B=1, H=24, N=46080, d=128, dtype="bf16", method="vsa",
                     q_block=64, k_block=64, keep_percent=10.0, centroid=0,
                     grid=(12, 48, 80), seed=6000)

CONFIGS = {w.name: w for w in (TINY_SOL, SOL_MID, SLA_TOPK, SOL_SINKS, LONG, VSA_CUBES)}


def _gaussian_transfer(n: int, sigma: float, device) -> torch.Tensor:
    """Fourier transfer function of a periodic Gaussian blur of std `sigma` samples."""
    f = torch.fft.fftfreq(n, device=device, dtype=torch.float64)
    return torch.exp(-2.0 * (math.pi ** 2) * (sigma ** 2) * f * f).to(torch.float32)


def _smooth_fields(gen: torch.Generator, count: int, grid, sigma: float, device) -> torch.Tensor:
    """`count` unit-variance smooth random fields on `grid`, shape [count, T*Hs*Ws]."""
    T, Hs, Ws = grid
    noise = torch.randn((count, T, Hs, Ws), generator=gen, device=device, dtype=torch.float32)
    spec = torch.fft.rfftn(noise, dim=(1, 2, 3))
    gt = _gaussian_transfer(T, sigma, device).view(T, 1, 1)
    gy = _gaussian_transfer(Hs, sigma, device).view(1, Hs, 1)
    gx = _gaussian_transfer(Ws, sigma, device)[: Ws // 2 + 1].view(1, 1, Ws // 2 + 1)
    field = torch.fft.irfftn(spec * (gt * gy * gx), s=(T, Hs, Ws), dim=(1, 2, 3))
    field = field.reshape(count, -1)
    field = field - field.mean(dim=1, keepdim=True)
    field = field / field.std(dim=1, keepdim=True)
    return field


def make_qkv(w: Workload, device="cpu", layout: str = "bnhd"):
    """Draw (Q, K, V) for workload `w` on `device`.

    layout "bnhd" gives contiguous [B, N, H, d] tensors (the usual model layout);
    "bhnd" gives [B, H, N, d] storage returned as a [B, N, H, d] strided view.
    Seeds: base seed w.seed; +0 field, +1 Q noise, +2 K noise, +3 V, +4 prefix.
    Returns tensors in the workload dtype (bf16 or fp32).
    """
    dev = torch.device(device)
    B, H, N, d = w.B, w.H, w.N, w.d
    out_dtype = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def gen(off):
        g = torch.Generator(device=dev)
        g.manual_seed(w.seed + off)
        return g

    store_shape = (B, N, H, d) if layout == "bnhd" else (B, H, N, d)
    q = torch.empty(store_shape, dtype=out_dtype, device=dev)
    k = torch.empty(store_shape, dtype=out_dtype, device=dev)
    v = torch.empty(store_shape, dtype=out_dtype, device=dev)
    qv, kv, vv = (t if layout == "bnhd" else t.permute(0, 2, 1, 3) for t in (q, k, v))

    P = w.prefix_len if w.grid is not None else 0
    if w.grid is None:
        gq, gk, gv = gen(1), gen(2), gen(3)
        for b in range(B):
            qv[b].copy_(torch.randn((N, H, d), generator=gq, device=dev))
            kv[b].copy_(torch.randn((N, H, d), generator=gk, device=dev))
            vv[b].copy_(torch.randn((N, H, d), generator=gv, device=dev))
        return qv, kv, vv

    T, Hs, Ws = w.grid
    G = T * Hs * Ws
    assert P + G == N, f"{w.name}: prefix {P} + grid {G} != N {N}"
    gf, gq, gk, gv, gp = gen(0), gen(1), gen(2), gen(3), gen(4)
    for b in range(B):
        if P:
            qv[b, :P].copy_(torch.randn((P, H, d), generator=gp, device=dev))
            kv[b, :P].copy_(torch.randn((P, H, d), generator=gp, device=dev))
            vv[b, :P].copy_(torch.randn((P, H, d), generator=gp, device=dev))
        for h in range(H):
            field = _smooth_fields(gf, d, w.grid, w.field_sigma, dev).t()   # [G, d]
            eq = torch.randn((G, d), generator=gq, device=dev)
            ek = torch.randn((G, d), generator=gk, device=dev)
            ev = torch.randn((G, d), generator=gv, device=dev)
            qv[b, P:, h].copy_(field + w.noise * eq)
            kv[b, P:, h].copy_(field + w.noise * ek)
            vv[b, P:, h].copy_(ev)
    return qv, kv, vv


def sample_query_blocks(w: Workload, count: int = 64, seed: int = 7):
    """Seeded sample of query-block indices for sampled parity on large sizes.

    Always includes block 0, the block holding the first dense row (if any),
    and the last (possibly partial) block.
    """
    g = torch.Generator()
    g.manual_seed(w.seed + 100 + seed)
    must = {0, w.nQB - 1}
    if w.dense_rows[1] > w.dense_rows[0]:
        must.add(w.dense_rows[0] // w.q_block)
    rest = torch.randperm(w.nQB, generator=g).tolist()
    picked = list(sorted(must))
    for i in rest:
        if len(picked) >= count:
            break
        if i not in must:
            picked.append(i)
    return sorted(picked)


def sample_heads(w: Workload):
    """Head subset {0, H/3, 2H/3, H-1} used for sampled parity."""
    return sorted({0, w.H // 3, (2 * w.H) // 3, w.H - 1})
