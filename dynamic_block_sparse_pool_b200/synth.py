"""Seeded synthetic Q/K/V for video-DiT self-attention workloads.

This module only draws inputs.  It holds none of the attention method's
arithmetic (no pooling, no scores, no selection, no attention), so both the
CUDA path and the CPU oracle can consume exactly the same tensors.

Recipe (one head, tokens of a T x H x W latent grid in row-major (t, y, x)
order, optionally preceded by ``n_prefix`` text-like tokens):

* phi(u) = sqrt(2) * cos(Omega u + beta), a random-Fourier feature of the
  token's grid coordinate u = (t, y, x) / ell.  Omega ~ N(0, I_3) per feature,
  beta ~ U[0, 2 pi).  E[phi(u) . phi(u')] / D = exp(-|u - u'|^2 / 2), so
  nearby tokens get correlated queries and keys (locality).
* ell is per axis: ``bandwidth`` (counted in blocks) times the extent of one
  block of consecutive row-major tokens along that axis, i.e.
  e_x = min(W, block), e_y = clamp(block / W, 1, H),
  e_t = clamp(block / (W H), 1, T).  A block's tokens then lie well inside
  one correlation length, so block means keep the locality signal, and a
  smaller bandwidth concentrates attention on fewer blocks.
* q = 0.7 phi + 0.5 N(0,1), k = 0.7 phi + 0.5 N(0,1) (independent noise).
* 4 "sink" key tokens per head at seeded uniform positions get
  k += 3 * mean_t(q_t), which gives every query a high score on them
  (vertical stripes in the attention map).
* V ~ N(0, 1).  Prefix tokens: q, k, v ~ N(0, 1), no phi.
* The result is cast to the workload dtype (bf16, or fp32 for the tiny case).

The structure follows the workloads the GSRS and Sparse-vDiT abstracts
measure (CogVideoX, Wan2.1 and HunyuanVideo text-to-video DiTs): their real
activations are not available, so these tensors stand in for them.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention workload: a latent token grid, heads and head_dim."""

    name: str
    T: int
    Hg: int
    W: int
    heads: int
    head_dim: int
    block: int
    dtype: torch.dtype
    p: Tuple[float, ...]
    n_prefix: int = 0
    batch: int = 1
    bandwidth: float = 4.0
    n_sinks: int = 4

    @property
    def n_grid(self) -> int:
        return self.T * self.Hg * self.W

    @property
    def N(self) -> int:
        return self.n_prefix + self.n_grid

    @property
    def n_blocks(self) -> int:
        return (self.N + self.block - 1) // self.block

    @property
    def BH(self) -> int:
        return self.batch * self.heads

    def dtype_name(self) -> str:
        return {torch.float32: "f32", torch.bfloat16: "bf16"}[self.dtype]

    def describe(self) -> str:
        pre = f"+{self.n_prefix} prefix" if self.n_prefix else ""
        return (f"{self.name}: B={self.batch} H={self.heads} D={self.head_dim} "
                f"grid {self.T}x{self.Hg}x{self.W}{pre} (N={self.N}) "
                f"block {self.block} {self.dtype_name()}")


TINY = Workload("tiny-f32", 4, 8, 8, heads=2, head_dim=64, block=64,
                dtype=torch.float32, p=(0.9,))
SMALL = Workload("small-bf16", 8, 16, 16, heads=4, head_dim=64, block=128,
                 dtype=torch.bfloat16, p=(0.95,))
COGVIDEOX = Workload("cogvideox-like", 13, 30, 45, heads=48, head_dim=64,
                     block=128, dtype=torch.bfloat16, p=(0.9,), n_prefix=226)
WAN21 = Workload("wan2.1-14b-like", 21, 45, 80, heads=40, head_dim=128,
                 block=128, dtype=torch.bfloat16,
                 p=(0.5, 0.7, 0.9, 0.95, 1.0))
HUNYUAN = Workload("hunyuanvideo-like", 33, 45, 80, heads=24, head_dim=128,
                   block=128, dtype=torch.bfloat16, p=(0.95,))

WORKLOADS = {w.name: w for w in (TINY, SMALL, COGVIDEOX, WAN21, HUNYUAN)}


def hunyuan_schedule(n_steps: int = 10):
    """Growing-sparsity driver for the HunyuanVideo-like grid.

    Step s of ``n_steps``: Top-p falls linearly 0.95 -> 0.6 and the locality
    bandwidth shrinks linearly 4 -> 1 blocks (attention concentrates as
    denoising proceeds); inputs of step s use seed s.
    Returns a list of (step, p, bandwidth, seed).
    """
    out = []
    for s in range(n_steps):
        f = s / (n_steps - 1) if n_steps > 1 else 0.0
        out.append((s, 0.95 - 0.35 * f, 4.0 - 3.0 * f, s))
    return out


def grid_coords(T: int, Hg: int, W: int) -> torch.Tensor:
    """(t, y, x) coordinates of the grid tokens in row-major order, [N, 3]."""
    t = torch.arange(T, dtype=torch.float64)
    y = torch.arange(Hg, dtype=torch.float64)
    x = torch.arange(W, dtype=torch.float64)
    tt, yy, xx = torch.meshgrid(t, y, x, indexing="ij")
    return torch.stack([tt.reshape(-1), yy.reshape(-1), xx.reshape(-1)], 1)


def lengthscales(w: Workload, bandwidth: float) -> torch.Tensor:
    """Per-axis (t, y, x) correlation lengths in grid units."""
    e_x = min(w.W, w.block)
    e_y = min(max(w.block / w.W, 1.0), w.Hg)
    e_t = min(max(w.block / (w.W * w.Hg), 1.0), w.T)
    return bandwidth * torch.tensor([e_t, e_y, e_x], dtype=torch.float64)


def make_qkv(w: Workload, seed: int, bandwidth: Optional[float] = None,
             heads: Optional[Sequence[int]] = None, device: str = "cpu"):
    """Draw (q, k, v), each [B, H, N, D] in ``w.dtype``, on the CPU.

    ``heads`` restricts the draw to a subset of heads (same values as the
    full draw for those heads: every head has its own generator stream).
    ``device="cuda"`` draws with the same recipe on the GPU (a different
    random stream, so different values with the same distribution): for
    timing runs that need many large inputs, not for comparisons with a
    CPU draw.
    """
    bw = w.bandwidth if bandwidth is None else bandwidth
    coords = (grid_coords(w.T, w.Hg, w.W) / lengthscales(w, bw)).to(torch.float32).to(device)
    D, N, P = w.head_dim, w.N, w.n_prefix
    head_ids = list(range(w.heads)) if heads is None else list(heads)
    shape = (w.batch, len(head_ids), N, D)
    q = torch.empty(shape, dtype=w.dtype, device=device)
    k = torch.empty(shape, dtype=w.dtype, device=device)
    v = torch.empty(shape, dtype=w.dtype, device=device)
    for b in range(w.batch):
        for hi, h in enumerate(head_ids):
            g = torch.Generator(device=device).manual_seed(
                (seed * 1000003 + b * 1009 + h) & 0x7FFFFFFF)
            omega = torch.randn(D, 3, generator=g, device=device)
            beta = torch.rand(D, generator=g, device=device) * (2.0 * math.pi)
            phi = math.sqrt(2.0) * torch.cos(coords @ omega.T + beta)
            qh = torch.empty(N, D, device=device)
            kh = torch.empty(N, D, device=device)
            qh[P:] = 0.7 * phi + 0.5 * torch.randn(N - P, D, generator=g, device=device)
            kh[P:] = 0.7 * phi + 0.5 * torch.randn(N - P, D, generator=g, device=device)
            if P:
                qh[:P] = torch.randn(P, D, generator=g, device=device)
                kh[:P] = torch.randn(P, D, generator=g, device=device)
            sinks = torch.randint(0, N, (w.n_sinks,), generator=g, device=device)
            kh[sinks] += 3.0 * qh.mean(0)
            vh = torch.randn(N, D, generator=g, device=device)
            q[b, hi] = qh.to(w.dtype)
            k[b, hi] = kh.to(w.dtype)
            v[b, hi] = vh.to(w.dtype)
    return q, k, v


def random_qkv(B: int, H: int, N: int, D: int, dtype: torch.dtype, seed: int,
               scale: float = 1.0):
    """Unstructured N(0, scale^2) q, k, v of shape [B, H, N, D]."""
    g = torch.Generator().manual_seed(seed)
    out = []
    for _ in range(3):
        out.append((scale * torch.randn(B, H, N, D, generator=g)).to(dtype))
    return tuple(out)


def random_csr(rows: int, n_cols: int, density: float, seed: int,
               min_per_row: int = 0):
    """A seeded random CSR block mask: (row_ptr int32 [rows+1], col int32).

    Columns are ascending within a row.  Used as reduced-search candidate
    sets and as fixed masks for attention parity.
    """
    g = torch.Generator().manual_seed(seed)
    keep = torch.rand(rows, n_cols, generator=g) < density
    if min_per_row > 0:
        for r in range(rows):
            if int(keep[r].sum()) < min_per_row:
                perm = torch.randperm(n_cols, generator=g)[:min_per_row]
                keep[r, perm] = True
    counts = keep.sum(1).to(torch.int64)
    row_ptr = torch.zeros(rows + 1, dtype=torch.int64)
    row_ptr[1:] = torch.cumsum(counts, 0)
    col = keep.nonzero()[:, 1]
    return row_ptr.to(torch.int32), col.to(torch.int32)
