"""The other fused DiT operators (news.cocoloop.cn MiniMax-H3 SGLang report,
fused-operator paragraph): the gated residual + AdaLN update and SwiGLU,
against the fp64 oracle.  Rule (helpers.check_fp32_rounding): every output
within one bf16 ulp of the oracle's result rounded to bf16 (or, near zero,
within 2^-18), and at most max(0.1%, 3) outputs not equal to it.  Cases: the 5376-wide H3 hidden state,
B = 2, the narrowest (8) and widest (14,336) rows, a width whose vectors do not
fill the CTA, the AdaLN update alone, in place.
"""
import numpy as np
import pytest
import torch

import rope_block_sparse_b200 as h3a
from rope_block_sparse_b200 import synth
from helpers import bits, check_fp32_rounding

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

EPS = 1e-6

ADALN_CASES = [
    ("h3a_width", 1, 37, 5376, True),
    ("b2_narrow", 2, 5, 96, True),
    ("min_width", 1, 3, 8, True),
    ("ragged_vectors", 1, 6, 2000, True),   # 250 vectors: 2 per thread, the last partly idle
    ("max_width", 1, 4, 14336, True),
    ("adaln_only", 2, 9, 5376, False),
]


@pytest.mark.parametrize("name,B,R,C,residual", ADALN_CASES, ids=[c[0] for c in ADALN_CASES])
def test_residual_adaln_parity(orc, name, B, R, C, residual):
    d = synth.draw_dit(B, R, C, seed=1)
    f = d["f"] if residual else None
    h, y = h3a.residual_adaln(d["x"].cuda(), None if f is None else f.cuda(), d["gate"].cuda(),
                              d["shift"].cuda(), d["scale"].cuda(), EPS)
    torch.cuda.synchronize()
    want_h, want_y = orc.residual_adaln(d["x"], f, d["gate"].numpy(), d["shift"].numpy(), d["scale"].numpy(), EPS)
    if residual:
        check_fp32_rounding(bits(h), want_h, f"{name} h")
    else:
        assert h is None
    check_fp32_rounding(bits(y), orc.round_bf16(want_y), f"{name} y")


def test_residual_adaln_in_place_matches():
    d = synth.draw_dit(2, 11, 5376, seed=2)
    x = d["x"].cuda()
    args = (d["f"].cuda(), d["gate"].cuda(), d["shift"].cuda(), d["scale"].cuda(), EPS)
    h, y = h3a.residual_adaln(x, *args)
    y2 = torch.empty_like(y)
    xi = x.clone()
    h3a.residual_adaln(xi, *args, out=(xi, y2))
    torch.cuda.synchronize()
    assert torch.equal(xi.view(torch.int16), h.view(torch.int16))
    assert torch.equal(y2.view(torch.int16), y.view(torch.int16))


# the model's FFN width is 14,336 (52hbtv.com H3-Image page, section 二, model table)
SWIGLU_CASES = [("small", 33, 1344), ("min_width", 5, 8), ("h3_ffn", 7, 14336), ("wide", 3, 21504)]


@pytest.mark.parametrize("name,R,F", SWIGLU_CASES, ids=[c[0] for c in SWIGLU_CASES])
def test_swiglu_parity(orc, name, R, F):
    d = synth.draw_dit(1, R, 8, ffn_width=F, seed=3)
    out = h3a.swiglu(d["ffn"].cuda())
    torch.cuda.synchronize()
    check_fp32_rounding(bits(out), orc.round_bf16(orc.swiglu(d["ffn"])), name)


def test_dit_ops_reject_bad_widths():
    x = torch.zeros(1, 2, 12, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros(1, 12, dtype=torch.float32, device="cuda")
    with pytest.raises(h3a.H3AError, match="INVALID_ARG"):
        h3a.residual_adaln(x, None, None, v, v)
    with pytest.raises(h3a.H3AError, match="INVALID_ARG"):
        h3a.swiglu(torch.zeros(2, 24, dtype=torch.bfloat16, device="cuda"))


# ---------------------------------------------------------------- Cache-DiT residual difference

@pytest.mark.parametrize("n", [8, 8 * 1_000_003, 8064 * 5376])
def test_residual_diff_matches_oracle(orc, n):
    cur, prev = synth.draw_step_pair(n, 0.05, seed=n % 97)
    rel, reuse = h3a.residual_diff(cur.cuda(), prev.cuda(), 0.04)
    torch.cuda.synchronize()
    want = orc.residual_diff(cur, prev)
    got = float(rel.item())
    assert abs(got - want) <= 1e-6 * want, (got, want)
    assert int(reuse.item()) == int(want < 0.04) or abs(want - 0.04) <= 1e-6 * 0.04


@pytest.mark.parametrize("sigma", [0.02, 0.06, 0.1])
def test_residual_diff_decisions(orc, sigma):
    """rel near 0.02 reuses at both page thresholds, near 0.06 only in stride mode
    (0.08), near 0.1 at neither; the decision is the oracle's rel < threshold."""
    cur, prev = synth.draw_step_pair(1 << 20, sigma, seed=5)
    want = orc.residual_diff(cur, prev)
    for thr in (0.04, 0.08):
        assert abs(want - thr) > 1e-3
        rel, reuse = h3a.residual_diff(cur.cuda(), prev.cuda(), thr)
        torch.cuda.synchronize()
        assert int(reuse.item()) == int(want < thr)


def test_residual_diff_deterministic_and_special_values():
    cur, prev = synth.draw_step_pair(1 << 22, 0.05, seed=6)
    c, p = cur.cuda(), prev.cuda()
    r1, _ = h3a.residual_diff(c, p)
    r2, _ = h3a.residual_diff(c, p)
    z = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    rz, uz = h3a.residual_diff(z, z)
    ri, ui = h3a.residual_diff(torch.ones_like(z), z)
    torch.cuda.synchronize()
    assert r1.item() == r2.item()
    assert rz.item() == 0.0 and uz.item() == 1
    assert ri.item() == float("inf") and ui.item() == 0


def test_residual_diff_refuses_small_workspace():
    z = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(h3a.H3AError, match="WORKSPACE"):
        h3a.residual_diff(z, z, workspace=small)
