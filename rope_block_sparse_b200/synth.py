"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws numbers: Q, K, V as bf16 ``[B, N, heads, head_dim]``
(token-major, ``N = T*H*W`` in row-major grid order) and the two RMSNorm gain
vectors as fp32 ``[head_dim]``.  It holds none of the attention core's own
arithmetic, so both the CUDA path and the CPU oracle can be fed from it.

Distributions (one recipe per workload family):

* ``normal``      : Q, K, V ~ N(0, 1).
* ``head_scaled`` : N(0, 1) times a per-head factor drawn from U[0.5, 2],
                    drawn separately for Q, K and V.
* ``structured``  : N(0, 1) + 0.5 * s(t, h, w), where for every (head, channel)
                    s is the sum of three separable products of cosines, one
                    cosine per grid axis with an integer frequency in 1..3 and a
                    uniform random phase, scaled to unit RMS over the grid.  The
                    smooth part makes pooled block scores structured, as video
                    latents are.

The gains are ``1 + 0.1 * N(0, 1)``.  Every tensor has its own torch CPU
generator seeded from ``(seed, tensor name)``; values are generated one time
slice at a time, so the stream does not depend on available memory.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

HEAD_DIM = 96


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    heads: int
    grid: tuple  # (T, H, W)
    dist: str
    sparsity: float | None  # None = dense attention
    also_dense: bool = False
    head_dim: int = HEAD_DIM

    @property
    def N(self) -> int:
        T, H, W = self.grid
        return T * H * W


WORKLOADS = {
    # 2 heads, 2x4x8 grid: the tiny correctness case.
    "tiny": Workload("tiny", 1, 2, (2, 4, 8), "normal", None),
    # one DiT attention layer at the H3 head geometry (56 heads x 96), 8,064 tokens.
    "layer8k": Workload("layer8k", 1, 56, (8, 24, 42), "head_scaled", None),
    # 5 s 1344x768 clip latent: 31x48x84 = 124,992 tokens, dense.
    "video5s": Workload("video5s", 1, 56, (31, 48, 84), "structured", None),
    # the same sequence, block-sparse at sparsity 0.75.
    "video5s_sparse": Workload("video5s_sparse", 1, 56, (31, 48, 84), "structured", 0.75),
    # 10 s clip latent: 61x48x84 = 245,952 tokens, block-sparse at 0.80 plus a dense run.
    "video10s": Workload("video10s", 1, 56, (61, 48, 84), "structured", 0.80, also_dense=True),
    # a 16x32x64 = 32,768-token clip for profiler captures: Q, K, V still exceed L2 (352 MB each).
    "clip32k": Workload("clip32k", 1, 56, (16, 32, 64), "structured", 0.75),
    # the 5 s clip at SubBlock's stated head size: the same 5376-wide hidden state as
    # 42 heads x 128, block-sparse at 0.75 (router and attention only: the 3D RoPE
    # layout is defined for 96 channels).
    "video5s_d128": Workload("video5s_d128", 1, 42, (31, 48, 84), "structured", 0.75, head_dim=128),
}

_STREAM = {"q": 1, "k": 2, "v": 3, "gamma_q": 4, "gamma_k": 5,
           "x": 11, "f": 12, "gate": 13, "shift": 14, "scale": 15, "ffn": 16, "prev": 17, "delta": 18}


def _gen(seed: int, name: str) -> torch.Generator:
    return torch.Generator().manual_seed(int(seed) * 1_000_003 + _STREAM[name])


def _smooth_factors(g: torch.Generator, grid, heads: int, d: int):
    """Per-axis cosine tables [3 terms, L, heads, d] and the unit-RMS scale [heads, d]."""
    freq = torch.randint(1, 4, (3, 3, heads, d), generator=g).to(torch.float64)
    phase = torch.rand((3, 3, heads, d), generator=g, dtype=torch.float64) * (2 * math.pi)
    tables = []
    for a, L in enumerate(grid):
        pos = torch.arange(L, dtype=torch.float64).view(1, L, 1, 1)
        tables.append(torch.cos(2 * math.pi * freq[:, a].unsqueeze(1) * pos / L + phase[:, a].unsqueeze(1)))
    # mean square over the grid of sum_m A_m(t) B_m(h) C_m(w), exact by separability
    ms = torch.ones(3, 3, heads, d, dtype=torch.float64)
    for tab in tables:
        ms = ms * (tab.unsqueeze(1) * tab.unsqueeze(0)).mean(dim=2)
    scale = 1.0 / ms.sum(dim=(0, 1)).sqrt()
    return [t.to(torch.float32) for t in tables], scale.to(torch.float32)


def draw_tensor(name: str, B: int, heads: int, grid, dist: str, seed: int = 0,
                head_dim: int = HEAD_DIM) -> torch.Tensor:
    """One bf16 [B, N, heads, head_dim] CPU tensor of the given distribution."""
    T, H, W = grid
    N = T * H * W
    g = _gen(seed, name)
    out = torch.empty((B, N, heads, head_dim), dtype=torch.bfloat16)
    if dist == "head_scaled":
        fac = (0.5 + 1.5 * torch.rand((B, heads), generator=g)).view(B, 1, heads, 1)
    elif dist == "structured":
        tabs, scale = _smooth_factors(g, grid, heads, head_dim)
    elif dist != "normal":
        raise ValueError(f"unknown distribution {dist!r}")
    slab = H * W
    for b in range(B):
        for t in range(T):
            x = torch.randn((slab, heads, head_dim), generator=g)
            if dist == "head_scaled":
                x = x * fac[b, 0]
            elif dist == "structured":
                A, Bt, C = tabs
                s = torch.zeros((H, W, heads, head_dim))
                for m in range(3):
                    s += A[m, t].view(1, 1, heads, head_dim) * (Bt[m].unsqueeze(1) * C[m].unsqueeze(0))
                x = x + 0.5 * scale * s.view(slab, heads, head_dim)
            out[b, t * slab:(t + 1) * slab] = x.to(torch.bfloat16)
    return out


def draw_gamma(name: str, seed: int = 0, head_dim: int = HEAD_DIM) -> torch.Tensor:
    g = _gen(seed, name)
    return (1.0 + 0.1 * torch.randn(head_dim, generator=g)).to(torch.float32)


def draw(B: int, heads: int, grid, dist: str = "normal", seed: int = 0, head_dim: int = HEAD_DIM,
         names=("q", "k", "v")) -> dict:
    """Q, K, V (bf16) and gamma_q, gamma_k (fp32) on the CPU."""
    out = {n: draw_tensor(n, B, heads, grid, dist, seed, head_dim) for n in names}
    out["gamma_q"] = draw_gamma("gamma_q", seed, head_dim)
    out["gamma_k"] = draw_gamma("gamma_k", seed, head_dim)
    return out


def draw_workload(name: str, seed: int = 0, names=("q", "k", "v")) -> dict:
    w = WORKLOADS[name]
    return draw(w.B, w.heads, w.grid, w.dist, seed, head_dim=w.head_dim, names=names)


def sample_rows(B: int, heads: int, N: int, count: int, seed: int = 1234) -> torch.Tensor:
    """``count`` distinct query rows r = (b*heads + h)*N + n, uniform over (b, h, n), sorted."""
    total = B * heads * N
    count = min(count, total)
    g = torch.Generator().manual_seed(seed)
    return torch.randperm(total, generator=g)[:count].sort().values


def draw_dit(B: int, rows: int, width: int, ffn_width: int = 0, seed: int = 0) -> dict:
    """Inputs of the gated residual + AdaLN update and of SwiGLU, on the CPU.

    x (residual stream) and f (branch output): bf16 [B, rows, width] ~ N(0, 1);
    gate, shift, scale (per-batch conditioning, as a timestep embedding gives):
    fp32 [B, width] ~ 0.5 * N(0, 1); with ffn_width > 0 also ffn: bf16
    [B * rows, 2 * ffn_width] ~ N(0, 1), the [a | b] input of SwiGLU.  Generated
    a batch at a time from one generator per tensor."""
    out = {}
    for name in ("x", "f"):
        g = _gen(seed, name)
        t = torch.empty((B, rows, width), dtype=torch.bfloat16)
        for b in range(B):
            t[b] = torch.randn((rows, width), generator=g).to(torch.bfloat16)
        out[name] = t
    for name in ("gate", "shift", "scale"):
        out[name] = (0.5 * torch.randn((B, width), generator=_gen(seed, name))).to(torch.float32)
    if ffn_width > 0:
        g = _gen(seed, "ffn")
        t = torch.empty((B * rows, 2 * ffn_width), dtype=torch.bfloat16)
        step = max(1, (1 << 24) // (2 * ffn_width))
        for r0 in range(0, B * rows, step):
            r1 = min(B * rows, r0 + step)
            t[r0:r1] = torch.randn((r1 - r0, 2 * ffn_width), generator=g).to(torch.bfloat16)
        out["ffn"] = t
    return out


def draw_step_pair(n: int, sigma: float, seed: int = 0):
    """Residuals of two adjacent denoising steps, bf16 [n]: prev ~ N(0, 1) and
    cur = prev + sigma * N(0, 1), so sum|cur - prev| / sum|prev| is close to sigma."""
    prev = torch.randn(n, generator=_gen(seed, "prev"))
    cur = prev + sigma * torch.randn(n, generator=_gen(seed, "delta"))
    return cur.to(torch.bfloat16), prev.to(torch.bfloat16)
