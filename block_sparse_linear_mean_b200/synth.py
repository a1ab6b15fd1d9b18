"""Seeded synthetic inputs for hybrid block-sparse + linear attention.

This module is the single source of test and benchmark inputs.  Both the CUDA
path and the CPU oracle consume what it produces; it contains none of the
attention method's arithmetic (no pooling, scoring, classification, softmax or
linear attention) -- only the construction of the inputs.

Recipe (video-DiT-shaped, spatio-temporally local activations):

* tokens live on a (F, R, C) latent grid (frames, rows, columns) and are laid
  out in raster order ``t = (f * R + r) * C + c``;
* per (batch, head) a white-noise field ``[F, R, C, d]`` is smoothed by a
  separable Gaussian (sigma = 3 grid steps on every axis, truncated at 4 sigma,
  half-sample-symmetric reflection at the borders) and each channel is then
  standardised (zero mean, unit variance over the grid);
* ``Q = S + a * eps_q`` and ``K = S + a * eps_k`` share one smooth field ``S``
  so attention is local in space and time; ``V = S_v + a * eps_v`` uses an
  independent smooth field; ``eps`` are N(0, 1);
* the projection ``W`` is ``[d, d]`` with N(0, (1/8)^2) entries, the upstream
  gradient ``dO`` is N(0, 1);
* bf16 workloads round Q, K, V and dO to bf16 once (round to nearest even);
  every consumer sees those exact values.

All randomness comes from ``torch.Generator`` objects seeded from the caller's
seed (data: seed, projection: seed + 1, upstream gradient: seed + 2), drawn in
a fixed order per (batch, head): S, S_v, eps_q, eps_k, eps_v.  A generator on
the CPU and one on a CUDA device give different (but each reproducible)
streams, so a test draws its inputs once and hands the same tensors to both
implementations.
"""

from __future__ import annotations

import functools
import math
from dataclasses import dataclass, field, replace
from typing import Optional, Tuple

import torch


@dataclass(frozen=True)
class Workload:
    """Shape, precision and selection rule of one hybrid-attention workload."""

    name: str
    B: int
    H: int
    grid: Tuple[int, int, int]
    d: int
    dtype: str                 # "f32" or "bf16"
    block_q: int
    block_k: int
    mode: str                  # "topk" or "cdf"
    frac_crit: float = 0.0
    frac_marg: float = 0.0
    thr: float = 0.0
    noise: float = 0.5
    sigma: float = 3.0
    backward: bool = False
    description: str = ""

    @property
    def N(self) -> int:
        f, r, c = self.grid
        return f * r * c

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads the library is built and measured for.
WORKLOADS = {
    "tiny": Workload(
        name="tiny", B=1, H=2, grid=(4, 16, 16), d=64, dtype="f32",
        block_q=64, block_k=64, mode="topk", frac_crit=0.25, frac_marg=0.25,
        noise=1.0,
        description="Tiny: B=1 H=2 N=1024 (4x16x16) d=64 fp32, block 64x64, "
                    "top-k 25% critical / 25% marginal"),
    "sla_1p3b": Workload(
        name="sla_1p3b", B=1, H=12, grid=(21, 30, 52), d=128, dtype="bf16",
        block_q=64, block_k=64, mode="topk", frac_crit=0.05, frac_marg=0.10,
        description="1.3B-DiT-shaped SLA forward: B=1 H=12 N=32760 (21x30x52) "
                    "d=128 bf16, block 64, 5% critical / 10% marginal"),
    "nabla_14b": Workload(
        name="nabla_14b", B=1, H=40, grid=(21, 45, 80), d=128, dtype="bf16",
        block_q=64, block_k=64, mode="cdf", thr=0.2,
        description="14B-DiT-shaped NABLA-style forward: B=1 H=40 N=75600 "
                    "(21x45x80) d=128 bf16, block 64, CDF threshold thr=0.2, "
                    "sparse only"),
    "long_clip": Workload(
        name="long_clip", B=1, H=40, grid=(60, 64, 64), d=128, dtype="bf16",
        block_q=128, block_k=128, mode="topk", frac_crit=0.03, frac_marg=0.02,
        description="Long-clip forward: B=1 H=40 N=245760 (60x64x64) d=128 "
                    "bf16, block 128x128, 3% critical / 2% marginal"),
    "finetune": Workload(
        name="finetune", B=1, H=12, grid=(21, 30, 52), d=128, dtype="bf16",
        block_q=64, block_k=64, mode="topk", frac_crit=0.05, frac_marg=0.10,
        backward=True,
        description="SLA fine-tune step: forward + backward at the 1.3B-DiT "
                    "shape (H=12 N=32760 d=128 bf16, 5%/10%)"),
}


def reflect_index(i: int, n: int) -> int:
    """Half-sample-symmetric reflection of index ``i`` into ``[0, n)``."""
    period = 2 * n
    i %= period
    return i if i < n else period - 1 - i


@functools.lru_cache(maxsize=None)
def gaussian_operator(n: int, sigma: float, truncate: float = 4.0) -> torch.Tensor:
    """Dense ``(n, n)`` matrix applying a truncated Gaussian blur along one axis
    (cached; callers copy it with ``.to``)."""
    radius = int(truncate * sigma + 0.5)
    offs = torch.arange(-radius, radius + 1, dtype=torch.float64)
    w = torch.exp(-0.5 * (offs / sigma) ** 2)
    w /= w.sum()
    m = torch.zeros(n, n, dtype=torch.float64)
    for i in range(n):
        for o, wo in zip(range(-radius, radius + 1), w.tolist()):
            m[i, reflect_index(i + o, n)] += wo
    return m


def smooth_field(grid, d: int, sigma: float, gen: torch.Generator,
                 device) -> torch.Tensor:
    """One standardised smooth field, returned as ``[F*R*C, d]`` float32."""
    f, r, c = grid
    x = torch.randn(f, r, c, d, generator=gen, device=device, dtype=torch.float32)
    mf = gaussian_operator(f, sigma).to(device=device, dtype=torch.float32)
    mr = gaussian_operator(r, sigma).to(device=device, dtype=torch.float32)
    mc = gaussian_operator(c, sigma).to(device=device, dtype=torch.float32)
    x = torch.einsum("fg,grcd->frcd", mf, x)
    x = torch.einsum("rs,fscd->frcd", mr, x)
    x = torch.einsum("ct,frtd->frcd", mc, x)
    x = x.reshape(f * r * c, d)
    x = x - x.mean(dim=0, keepdim=True)
    x = x / x.std(dim=0, keepdim=True, correction=0).clamp_min(1e-12)
    return x


@dataclass
class Inputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    proj: torch.Tensor
    dout: Optional[torch.Tensor] = None
    seed: int = 0
    extra: dict = field(default_factory=dict)


def make_inputs(wl: Workload, seed: int = 0, device="cpu",
                heads: Optional[int] = None, with_dout: bool = False) -> Inputs:
    """Draw Q, K, V ``[B, H, N, d]`` (workload dtype), W ``[d, d]`` fp32 and
    optionally dO ``[B, H, N, d]`` (workload dtype) for ``wl``.

    ``heads`` overrides H (used to draw a head-subset of a large workload;
    head h of a subset equals head h of the full draw because every head is
    drawn in order from the same generator)."""
    H = wl.H if heads is None else heads
    N, d = wl.N, wl.d
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    out_dtype = wl.torch_dtype
    q = torch.empty(wl.B, H, N, d, dtype=out_dtype, device=dev)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    a = wl.noise
    for b in range(wl.B):
        for h in range(H):
            s = smooth_field(wl.grid, d, wl.sigma, gen, dev)
            sv = smooth_field(wl.grid, d, wl.sigma, gen, dev)
            eq = torch.randn(N, d, generator=gen, device=dev)
            ek = torch.randn(N, d, generator=gen, device=dev)
            ev = torch.randn(N, d, generator=gen, device=dev)
            q[b, h] = (s + a * eq).to(out_dtype)
            k[b, h] = (s + a * ek).to(out_dtype)
            v[b, h] = (sv + a * ev).to(out_dtype)
    gw = torch.Generator(device=dev)
    gw.manual_seed(seed + 1)
    proj = torch.randn(d, d, generator=gw, device=dev) * (1.0 / 8.0)
    dout = None
    if with_dout:
        gd = torch.Generator(device=dev)
        gd.manual_seed(seed + 2)
        dout = torch.randn(wl.B, H, N, d, generator=gd, device=dev).to(out_dtype)
    return Inputs(q=q, k=k, v=v, proj=proj, dout=dout, seed=seed)


def small_case(d=64, grid=(2, 5, 100), H=2, B=1, dtype="f32", block_q=64,
               block_k=64, mode="topk", frac_crit=0.25, frac_marg=0.25,
               thr=0.2, noise=0.5, name="small") -> Workload:
    """A workload small enough for the oracle that still spans several tiles
    and a ragged tail block (default N = 1000 = 15 full blocks of 64 + 40)."""
    return Workload(name=name, B=B, H=H, grid=grid, d=d, dtype=dtype,
                    block_q=block_q, block_k=block_k, mode=mode,
                    frac_crit=frac_crit, frac_marg=frac_marg, thr=thr,
                    noise=noise)
