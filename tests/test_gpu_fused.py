"""The prologue with the router's block pooling folded in (h3a_qk_norm_rope_pool)
and the scoring half of the router that reads its means (h3a_route_pooled).

Pinned three ways:
  * against the oracle: the prologue outputs by the prologue rule, the block
    means by the oracle's fp64 pooling of the same rounded outputs (within the
    error bound of an fp32 sum of the block's terms), the block lists by the
    router rule;
  * against the unfused calls: outputs, block means and block lists are
    bit-identical to h3a_qk_norm_rope followed by h3a_route (both sum the same
    fp32 values in token order);
  * edge cases: one partial block, tail blocks, B = 2, 57 and 5 heads, strided
    heads written in place.
"""
import numpy as np
import pytest
import torch

import rope_block_sparse_b200 as h3a
from rope_block_sparse_b200 import synth
from helpers import bits, check_prologue, check_router

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

THETA, EPS = 10000.0, 1e-6

CASES = [
    ("tiny", 1, 2, (2, 4, 8), 0.75, "normal"),           # 64 tokens: one partial block
    ("layer8k", 1, 56, (8, 24, 42), 0.75, "head_scaled"),  # 63 blocks, tail of 0
    ("ragged", 2, 5, (3, 7, 55), 0.6, "structured"),     # 1155 tokens: tail of 3, B = 2
    ("heads57", 1, 57, (2, 9, 20), 0.8, "normal"),        # 360 tokens, 57 heads (3 head chunks)
]


def _pooled_halves(ws: torch.Tensor, B: int, heads: int, nblk: int):
    """The block means in a router workspace, both as fp32 [B, heads, nblk, 96]:
    Q's are stored that way, K's channel-major ([B, heads, 96, nblk rounded up
    to 4]) after Q's, on the next 256-byte boundary."""
    n = B * heads * nblk * 96
    nblk4 = (nblk + 3) // 4 * 4
    half = (n * 4 + 255) // 256 * 256
    f = ws.view(torch.uint8)
    q = f[:n * 4].view(torch.float32).view(B, heads, nblk, 96)
    kt = f[half:half + B * heads * 96 * nblk4 * 4].view(torch.float32).view(B, heads, 96, nblk4)
    return q, kt[..., :nblk].transpose(2, 3)


def _pool_bound(orc, out_bits: np.ndarray) -> np.ndarray:
    """Error bound of an fp32 block mean: (len + 2) * 2^-24 * mean |x| per entry."""
    B, N, heads, d = out_bits.shape
    mean_abs = orc.pool(out_bits & np.uint16(0x7FFF))
    nblk = mean_abs.shape[2]
    lens = np.minimum(N - 128 * np.arange(nblk), 128).astype(np.float64)
    return (lens[None, None, :, None] + 2.0) * 2.0 ** -24 * mean_abs.astype(np.float64) + 1e-30


@pytest.mark.parametrize("name,B,heads,grid,s,dist", CASES, ids=[c[0] for c in CASES])
def test_fused_prologue_pool_and_route(orc, name, B, heads, grid, s, dist):
    d = synth.draw(B, heads, grid, dist, 0)
    q, k = d["q"].cuda(), d["k"].cuda()
    gq, gk = d["gamma_q"].cuda(), d["gamma_k"].cuda()
    N = grid[0] * grid[1] * grid[2]
    nblk = (N + 127) // 128

    qo, ko, ws = h3a.qk_norm_rope_pool(q, k, gq, gk, grid, THETA, EPS)
    idx = h3a.route_pooled(qo, s, ws)
    # the unfused calls on the same inputs
    qu, ku = h3a.qk_norm_rope(q, k, gq, gk, grid, THETA, EPS)
    ws_u = torch.empty_like(ws)
    idx_u = h3a.route(qu, ku, s, workspace=ws_u)
    torch.cuda.synchronize()

    # oracle: prologue rule
    for x, g, out in ((d["q"], d["gamma_q"], qo), (d["k"], d["gamma_k"], ko)):
        check_prologue(bits(out), orc.qk_norm_rope_bf16(x, g.numpy(), grid, THETA, EPS), name)
    # oracle: block means of the kernel's own rounded outputs
    pq, pk = _pooled_halves(ws, B, heads, nblk)
    for out, got in ((qo, pq), (ko, pk)):
        ob = bits(out)
        want = orc.pool(ob).astype(np.float64)
        err = np.abs(got.cpu().numpy().astype(np.float64) - want)
        bound = _pool_bound(orc, ob)
        assert np.all(err <= bound), f"{name}: block mean off by {float(np.max(err / bound)):.2f} x its bound"
    # oracle: router rule on the kernel's outputs
    ora_idx, ora_sc = orc.route(bits(qo), bits(ko), s)
    check_router(idx.cpu().numpy(), ora_idx, ora_sc, name)

    # bit-identical to the unfused path
    assert torch.equal(qo.view(torch.int16), qu.view(torch.int16))
    assert torch.equal(ko.view(torch.int16), ku.view(torch.int16))
    pq_u, pk_u = _pooled_halves(ws_u, B, heads, nblk)
    assert torch.equal(pq.view(torch.int32), pq_u.view(torch.int32))
    assert torch.equal(pk.view(torch.int32), pk_u.view(torch.int32))
    assert torch.equal(idx, idx_u)


def test_fused_prologue_strided_inplace(orc):
    """Heads 0..4 of a 7-head buffer (token stride 7*96), written in place."""
    grid, heads, s = (2, 6, 25), 5, 0.5
    d = synth.draw(1, 7, grid, "structured", 3)
    qbuf, kbuf = d["q"].cuda(), d["k"].cuda()
    q, k = qbuf[:, :, :heads], kbuf[:, :, :heads]
    untouched = kbuf[:, :, heads:].clone()
    gq, gk = d["gamma_q"].cuda(), d["gamma_k"].cuda()
    qo, ko, ws = h3a.qk_norm_rope_pool(q, k, gq, gk, grid, THETA, EPS, inplace=True)
    idx = h3a.route_pooled(qo, s, ws)
    torch.cuda.synchronize()
    assert qo.data_ptr() == q.data_ptr() and ko.data_ptr() == k.data_ptr()
    for x, g, out in ((d["q"], d["gamma_q"], qo), (d["k"], d["gamma_k"], ko)):
        want = orc.qk_norm_rope_bf16(x[:, :, :heads].contiguous(), g.numpy(), grid, THETA, EPS)
        check_prologue(bits(out), want, "strided")
    assert torch.equal(kbuf[:, :, heads:], untouched)
    ora_idx, ora_sc = orc.route(bits(qo), bits(ko), s)
    check_router(idx.cpu().numpy(), ora_idx, ora_sc, "strided")


def test_fused_workspace_too_small_is_refused():
    grid = (2, 4, 16)
    d = synth.draw(1, 4, grid, "normal", 0)
    q, k = d["q"].cuda(), d["k"].cuda()
    need = h3a.route_workspace_size(q)
    small = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(h3a.H3AError, match="WORKSPACE"):
        h3a.qk_norm_rope_pool(q, k, d["gamma_q"].cuda(), d["gamma_k"].cuda(), grid, workspace=small)
    with pytest.raises(h3a.H3AError, match="WORKSPACE"):
        h3a.route_pooled(q, 0.5, small)


def test_attention_core_follows_the_step_schedule():
    """attention_core with a denoising step: dense (no block lists) before step 10,
    the routed sparse path from step 10 on -- each equal, bit for bit, to the
    calls it stands for."""
    grid, heads = (4, 16, 40), 3                   # 2560 tokens, 20 blocks
    d = synth.draw(1, heads, grid, "structured", 4)
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    gq, gk = d["gamma_q"].cuda(), d["gamma_k"].cuda()
    o9, b9 = h3a.attention_core(q, k, v, gq, gk, grid, sparsity=0.75, step=9)
    o10, b10 = h3a.attention_core(q, k, v, gq, gk, grid, sparsity=0.75, step=10)
    qn, kn = h3a.qk_norm_rope(q, k, gq, gk, grid)
    dense = h3a.attention(qn, kn, v)
    blocks = h3a.route(qn, kn, 0.75)
    sparse = h3a.attention(qn, kn, v, blocks)
    torch.cuda.synchronize()
    assert b9 is None and torch.equal(o9, dense)
    assert torch.equal(b10, blocks) and torch.equal(o10, sparse)
