"""Seeded synthetic inputs for the block-sparse video-attention path.

This module only draws numbers: it holds none of the method's arithmetic
(no attention, no scoring, no selection, no token partition).  Both the CUDA
path and the CPU oracle consume the tensors it returns, so parity depends only
on the two sides reading the same bytes.

Workloads (shapes follow the video DiT layers the pages discuss: a Wan2.1-like
21x30x52 latent grid and a HunyuanVideo-like 33x45x80 grid; the pages measure
on trained models and VBench, which these seeded tensors stand in for):

  tiny       B=1 H=2  d=64  fp32  grid 4x8x8     block 64
  wan        B=1 H=12 d=128 bf16  grid 21x30x52  block 64
  hunyuan    B=1 H=24 d=128 bf16  grid 33x45x80  block 128 (re-drawn per step)
  wan_proxy  as wan
  wan_skew   as wan, half the heads low-entropy (alpha in [2,4]) and half
             high-entropy (alpha in [0.25,0.5])

Recipe (per head h):
  F      3D sinusoidal position features of the raster-ordered grid, dim d:
         m = d//6 frequencies per axis (t, y, x), omega_k = s_h * 100**(-k/m),
         features sin(omega_k*pos), cos(omega_k*pos); the last d-6m dims are 0.
  s_h    log-uniform in [0.05, 0.5]
  W_h    d x d, entries N(0, 1/d)
  alpha  U[0.5, 2]  (skewed workload: see above)
  Q = alpha*(F W_h) + N(0, 0.5^2),  K = alpha*(F W_h) + N(0, 0.5^2)
  (the same F W_h for Q and K, independent noise), V ~ N(0, 1).
  bf16 workloads are rounded to bf16 (round-to-nearest-even) at the end.
Re-drawn steps (index-reuse workload): X_{t+1} = 0.9 X_t + 0.1 eps with
eps ~ N(0, 0.5^2) for Q, K and N(0, 1) for V, kept in fp32 and cast per step.

Every draw comes from a torch.Generator seeded with
  seed = 1_000_003*workload_id + 10_007*tensor_id + step
on the device the tensors are made on (CPU and CUDA generators give different
streams; a parity check always hands the oracle the bytes the GPU used).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

__all__ = ["Workload", "WORKLOADS", "get_workload", "make_qkv", "redraw_qkv", "small_workload"]


@dataclass(frozen=True)
class Workload:
    name: str
    wid: int
    B: int
    H: int
    d: int
    grid: tuple          # (T, H, W) token grid
    block: int
    dtype: str           # "f32" | "bf16"
    p: float = 0.99
    skew: bool = False
    extra: dict = field(default_factory=dict)

    @property
    def n_valid(self) -> int:
        t, h, w = self.grid
        return t * h * w

    @property
    def n_blocks(self) -> int:
        return -(-self.n_valid // self.block)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = {
    "tiny": Workload("tiny", 0, 1, 2, 64, (4, 8, 8), 64, "f32"),
    "wan": Workload("wan", 1, 1, 12, 128, (21, 30, 52), 64, "bf16",
                    extra={"partition": "3d", "tile": (4, 4, 4)}),
    "hunyuan": Workload("hunyuan", 2, 1, 24, 128, (33, 45, 80), 128, "bf16",
                        extra={"partition": "raster", "steps": 49}),
    "wan_proxy": Workload("wan_proxy", 3, 1, 12, 128, (21, 30, 52), 64, "bf16", p=0.25,
                          extra={"partition": "cycle", "tile": (4, 4, 4), "frame_tile": (8, 8)}),
    "wan_skew": Workload("wan_skew", 4, 1, 12, 128, (21, 30, 52), 64, "bf16", skew=True,
                         extra={"partition": "3d", "tile": (4, 4, 4),
                                "p_sweep": (0.90, 0.95, 0.99, 0.999)}),
}


def get_workload(name: str) -> Workload:
    return WORKLOADS[name]


def small_workload(name: str, B: int, H: int, d: int, grid: tuple, block: int,
                   dtype: str = "bf16", wid: int = 100, skew: bool = False) -> Workload:
    """A custom-shaped workload drawn with the same recipe (for parity tests)."""
    return Workload(name, wid, B, H, d, tuple(grid), block, dtype, skew=skew)


def _gen(device, wid: int, tensor_id: int, step: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(1_000_003 * wid + 10_007 * tensor_id + step)
    return g


def _features(grid, d, scale, device):
    """3D sinusoidal features [N, d] (fp32) of the raster-ordered grid for one head."""
    T, Hh, Ww = grid
    m = d // 6
    t = torch.arange(T, device=device, dtype=torch.float64)
    y = torch.arange(Hh, device=device, dtype=torch.float64)
    x = torch.arange(Ww, device=device, dtype=torch.float64)
    k = torch.arange(m, device=device, dtype=torch.float64)
    omega = scale * torch.pow(torch.tensor(100.0, dtype=torch.float64, device=device), -k / m)
    tt, yy, xx = torch.meshgrid(t, y, x, indexing="ij")
    cols = []
    for pos in (tt.reshape(-1), yy.reshape(-1), xx.reshape(-1)):
        ang = pos[:, None] * omega[None, :]
        cols.append(torch.sin(ang))
        cols.append(torch.cos(ang))
    F = torch.cat(cols, dim=1)
    if F.shape[1] < d:
        F = torch.cat([F, torch.zeros(F.shape[0], d - F.shape[1], dtype=F.dtype, device=device)], 1)
    return F.to(torch.float32)


def make_qkv_f32(wl: Workload, device="cpu"):
    """fp32 master tensors Q, K, V of shape [B, H, N_valid, d] in raster token order."""
    B, H, d, N = wl.B, wl.H, wl.d, wl.n_valid
    g = _gen(device, wl.wid, 0, 0)
    u = torch.rand(H, generator=g, device=device, dtype=torch.float64)
    scale = torch.exp(math.log(0.05) + u * (math.log(0.5) - math.log(0.05)))
    ua = torch.rand(H, generator=g, device=device, dtype=torch.float64)
    if wl.skew:
        half = H // 2
        alpha = torch.empty(H, dtype=torch.float64, device=device)
        alpha[:half] = 2.0 + 2.0 * ua[:half]
        alpha[half:] = 0.25 + 0.25 * ua[half:]
    else:
        alpha = 0.5 + 1.5 * ua
    Wm = torch.randn(H, d, d, generator=g, device=device, dtype=torch.float32) / math.sqrt(d)
    q = torch.empty(B, H, N, d, dtype=torch.float32, device=device)
    k = torch.empty_like(q)
    for h in range(H):
        F = _features(wl.grid, d, float(scale[h]), device)
        base = (F @ Wm[h]) * float(alpha[h])
        q[:, h] = base
        k[:, h] = base
    gq = _gen(device, wl.wid, 1, 0)
    gk = _gen(device, wl.wid, 2, 0)
    gv = _gen(device, wl.wid, 3, 0)
    q += 0.5 * torch.randn(q.shape, generator=gq, device=device, dtype=torch.float32)
    k += 0.5 * torch.randn(k.shape, generator=gk, device=device, dtype=torch.float32)
    v = torch.randn(q.shape, generator=gv, device=device, dtype=torch.float32)
    return q, k, v


def make_qkv(wl: Workload, device="cpu"):
    """Q, K, V [B, H, N_valid, d] in the workload's dtype, raster token order."""
    q, k, v = make_qkv_f32(wl, device)
    dt = wl.torch_dtype
    return q.to(dt), k.to(dt), v.to(dt)


def redraw_qkv(wl: Workload, q32, k32, v32, step: int):
    """One re-draw step of the index-reuse workload (in place on the fp32 masters)."""
    dev = q32.device
    for tid, (x, sigma) in enumerate(((q32, 0.5), (k32, 0.5), (v32, 1.0))):
        g = _gen(dev, wl.wid, 4 + tid, step)
        eps = torch.randn(x.shape, generator=g, device=dev, dtype=torch.float32)
        x.mul_(0.9).add_(eps, alpha=0.1 * sigma)
    dt = wl.torch_dtype
    return q32.to(dt), k32.to(dt), v32.to(dt)
