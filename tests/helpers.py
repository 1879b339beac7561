"""Shared helpers of the parity tests: bit views and the comparison rules.

Comparison rules (the problem statement's, plus one reading for the prologue):
  * prologue  -- at least 99.9% of outputs equal the oracle's fp64 result
                 rounded to bf16 (nearest-even), and every output is within one
                 bf16 ulp of it or, for results near zero, within 2^-18 of it in
                 absolute terms: the kernel computes in fp32, and a rotation
                 whose two products nearly cancel keeps only fp32-level absolute
                 accuracy (the outputs have unit RMS per head after the norm);
  * router    -- the kept block sets equal the oracle's exactly, except for
                 blocks whose oracle score lies within 1e-5 of the row's top-k
                 cut; each row ascending, distinct, of length k;
  * attention -- max abs error <= 2e-2 and relative RMS error <= 1e-2 against
                 the fp64 oracle.
"""
from __future__ import annotations

import numpy as np
import torch

PROLOGUE_MIN_EXACT = 0.999
PROLOGUE_ABS_FLOOR = 2.0 ** -18
ROUTER_TIE_WINDOW = 1e-5
ATTN_MAX_ABS = 2e-2
ATTN_REL_RMS = 1e-2


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> uint16 numpy array of its bit patterns."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(b: np.ndarray) -> torch.Tensor:
    """uint16 bit patterns -> bf16 CPU tensor."""
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16)


def bf16_order(b: np.ndarray) -> np.ndarray:
    """Monotone integer image of bf16 bit patterns (adjacent values differ by 1)."""
    b = b.astype(np.int32)
    return np.where(b & 0x8000, 0x8000 - (b & 0x7FFF), 0x8000 + b)


def check_prologue(gpu_bits: np.ndarray, want_bits: np.ndarray, label: str = ""):
    """gpu_bits vs the oracle's correctly rounded result (both uint16)."""
    assert gpu_bits.shape == want_bits.shape
    exact = np.mean(gpu_bits == want_bits)
    ulps = np.abs(bf16_order(gpu_bits) - bf16_order(want_bits))
    assert exact >= PROLOGUE_MIN_EXACT, f"{label}: only {exact:.6f} of outputs correctly rounded"
    far = ulps > 1
    if far.any():
        g = bits_to_f64(gpu_bits[far])
        w = bits_to_f64(want_bits[far])
        worst = float(np.max(np.abs(g - w)))
        assert worst <= PROLOGUE_ABS_FLOOR, (
            f"{label}: {int(far.sum())} outputs beyond 1 ulp, worst absolute error {worst:.3g}")
    return exact


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def check_router(gpu_idx: np.ndarray, ora_idx: np.ndarray, ora_scores: np.ndarray, label: str = ""):
    """Per row: ascending distinct indices; set differences only inside the tie window at the cut."""
    assert gpu_idx.shape == ora_idx.shape, (gpu_idx.shape, ora_idx.shape)
    k = gpu_idx.shape[-1]
    g = gpu_idx.reshape(-1, k)
    o = ora_idx.reshape(-1, k)
    s = ora_scores.reshape(g.shape[0], -1)
    assert (g >= 0).all() and (g < s.shape[1]).all(), f"{label}: index out of range"
    if k > 1:
        assert (np.diff(g, axis=1) > 0).all(), f"{label}: rows not strictly ascending"
    differing = np.nonzero((g != o).any(axis=1))[0]
    inside = 0
    for r in differing:
        cut = np.sort(s[r])[::-1][k - 1]
        sym = set(g[r].tolist()) ^ set(o[r].tolist())
        for j in sym:
            assert abs(float(s[r, j]) - float(cut)) <= ROUTER_TIE_WINDOW, (
                f"{label}: row {r} block {j} score {s[r, j]} outside the tie window of cut {cut}")
        inside += 1
    return inside


def check_attention(gpu_rows: np.ndarray, ora_rows: np.ndarray, label: str = ""):
    g = np.asarray(gpu_rows, dtype=np.float64)
    o = np.asarray(ora_rows, dtype=np.float64)
    err = g - o
    max_abs = float(np.max(np.abs(err)))
    rel_rms = float(np.sqrt(np.mean(err ** 2)) / max(np.sqrt(np.mean(o ** 2)), 1e-30))
    assert max_abs <= ATTN_MAX_ABS, f"{label}: max abs error {max_abs}"
    assert rel_rms <= ATTN_REL_RMS, f"{label}: relative RMS error {rel_rms}"
    return max_abs, rel_rms


def gather_rows(o: torch.Tensor, rows: np.ndarray) -> np.ndarray:
    """Rows r = (b*heads + h)*N + n of a [B, N, heads, d] tensor -> fp64 [len(rows), d]."""
    B, N, H, D = o.shape
    r = torch.as_tensor(rows, dtype=torch.int64)
    bh, n = r // N, r % N
    b, h = bh // H, bh % H
    return o[b.to(o.device), n.to(o.device), h.to(o.device)].double().cpu().numpy()


def check_fp32_rounding(gpu_bits: np.ndarray, want_bits: np.ndarray, label: str = "", floor: int = 3):
    """The prologue rule for outputs computed in fp32 and rounded once to bf16,
    sized for small cases: every output within one bf16 ulp (or 2^-18 near
    zero) of the oracle's correctly rounded value, and at most
    max(0.1% of the outputs, `floor`) of them not equal to it.  fp32 arithmetic
    (an approximate rsqrt, another summation order) moves a result across a
    bf16 rounding boundary with a probability of about 1e-4 per output, so on a
    few hundred outputs "99.9% exact" would forbid even one such crossing."""
    assert gpu_bits.shape == want_bits.shape
    inexact = int(np.sum(gpu_bits != want_bits))
    allowed = max(int(0.001 * gpu_bits.size), floor)
    assert inexact <= allowed, f"{label}: {inexact} of {gpu_bits.size} outputs not correctly rounded (> {allowed})"
    ulps = np.abs(bf16_order(gpu_bits) - bf16_order(want_bits))
    far = ulps > 1
    if far.any():
        worst = float(np.max(np.abs(bits_to_f64(gpu_bits[far]) - bits_to_f64(want_bits[far]))))
        assert worst <= PROLOGUE_ABS_FLOOR, (
            f"{label}: {int(far.sum())} outputs beyond 1 ulp, worst absolute error {worst:.3g}")
    return inexact
