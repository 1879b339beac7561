"""The prologue with the RMSNorm over each token's whole hidden state
(h3a_qk_fullnorm_rope) against the fp64 oracle, by the prologue rule:
at least 99.9% of outputs correctly rounded to bf16, every output within one
ulp (or 2^-18 near zero).  Cases: 2 heads, the 56-head layer with per-head
scales, 57 heads (a partial head group), B = 2 with a ragged grid, and heads
0..4 of a 7-head buffer written in place."""
import numpy as np
import pytest
import torch

import rope_block_sparse_b200 as h3a
from rope_block_sparse_b200 import synth
from helpers import bits, check_prologue

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

THETA, EPS = 10000.0, 1e-6

CASES = [
    ("tiny", 1, 2, (2, 4, 8), "normal"),
    ("layer8k", 1, 56, (8, 24, 42), "head_scaled"),
    ("heads57", 1, 57, (2, 3, 4), "normal"),
    ("ragged_b2", 2, 5, (3, 5, 7), "normal"),
]


def _gains(heads, seed=0):
    return (synth.draw_gamma("gamma_q", seed, heads * 96), synth.draw_gamma("gamma_k", seed, heads * 96))


@pytest.mark.parametrize("name,B,heads,grid,dist", CASES, ids=[c[0] for c in CASES])
def test_fullnorm_prologue_parity(orc, name, B, heads, grid, dist):
    d = synth.draw(B, heads, grid, dist, 0)
    gq, gk = _gains(heads)
    qo, ko = h3a.qk_fullnorm_rope(d["q"].cuda(), d["k"].cuda(), gq.cuda(), gk.cuda(), grid, THETA, EPS)
    torch.cuda.synchronize()
    for x, g, out in ((d["q"], gq, qo), (d["k"], gk, ko)):
        check_prologue(bits(out), orc.qk_fullnorm_rope_bf16(x, g.numpy(), grid, THETA, EPS), name)


def test_fullnorm_prologue_strided_inplace(orc):
    grid, heads = (2, 6, 5), 5
    d = synth.draw(1, 7, grid, "normal", 2)
    qbuf, kbuf = d["q"].cuda(), d["k"].cuda()
    q, k = qbuf[:, :, :heads], kbuf[:, :, :heads]
    untouched = qbuf[:, :, heads:].clone()
    gq, gk = _gains(heads, 2)
    qo, ko = h3a.qk_fullnorm_rope(q, k, gq.cuda(), gk.cuda(), grid, THETA, EPS, inplace=True)
    torch.cuda.synchronize()
    assert qo.data_ptr() == q.data_ptr()
    for x, g, out in ((d["q"], gq, qo), (d["k"], gk, ko)):
        want = orc.qk_fullnorm_rope_bf16(x[:, :, :heads].contiguous(), g.numpy(), grid, THETA, EPS)
        check_prologue(bits(out), want, "strided")
    assert torch.equal(qbuf[:, :, heads:], untouched)
