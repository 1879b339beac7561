"""The router and attention at head_dim 128 -- SubBlock's stated head size
(news.cocoloop.cn MiniMax-H3 SGLang report, section "Ein paar Grenzen") --
against the fp64 oracle, whose functions take the head size from their inputs.

The prologue is not part of this path: its 3D RoPE layout (32 channels per
axis) is defined for 96 channels only, so these inputs go to the router and
attention as drawn.  Cases cover one partial block, tail blocks, an odd
number of query tiles (a CTA with one tile), B = 2, sparse lists, and a
42-head sampled case (the 5376-wide hidden state as 42 heads x 128).
"""
import numpy as np
import pytest
import torch

import rope_block_sparse_b200 as h3a
from rope_block_sparse_b200 import synth
from helpers import check_attention, check_router, gather_rows

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

D = 128


def _inputs(B, heads, grid, dist="normal", seed=0):
    return synth.draw(B, heads, grid, dist, seed, head_dim=D)


def _dev(t):
    return t.cuda()


ATTN_CASES = [
    ("tiny", 1, 2, (2, 4, 8)),            # 64 tokens: one partial block
    ("ragged", 2, 3, (3, 5, 7)),          # 105 tokens, B = 2
    ("odd_tiles", 1, 4, (3, 10, 10)),     # 300 tokens: 3 query tiles (the last CTA has one)
    ("tail1", 1, 2, (1, 1, 257)),         # 257 tokens: a tail block of one token
]


@pytest.mark.parametrize("name,B,heads,grid", ATTN_CASES, ids=[c[0] for c in ATTN_CASES])
def test_dense_attention_parity_d128(orc, name, B, heads, grid):
    d = _inputs(B, heads, grid)
    o = h3a.attention(_dev(d["q"]), _dev(d["k"]), _dev(d["v"]))
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0
    N = grid[0] * grid[1] * grid[2]
    rows = np.arange(B * heads * N)
    want = orc.attention_rows(d["q"], d["k"], d["v"], rows)
    check_attention(gather_rows(o, rows), want, name)


@pytest.mark.parametrize("s", [0.5, 0.8])
def test_sparse_attention_parity_d128(orc, s):
    grid, heads = (4, 16, 40), 5                  # 2560 tokens, 20 blocks
    d = _inputs(1, heads, grid, "structured")
    ora_idx, _ = orc.route(d["q"], d["k"], s)
    o = h3a.attention(_dev(d["q"]), _dev(d["k"]), _dev(d["v"]), _dev(torch.from_numpy(ora_idx)))
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0
    rows = np.arange(heads * 2560)
    want = orc.attention_rows(d["q"], d["k"], d["v"], rows, ora_idx)
    check_attention(gather_rows(o, rows), want, f"d128-s{s}")


ROUTER_CASES = [
    ("tiny", 1, 2, (2, 4, 8), 0.75),
    ("ragged", 2, 3, (3, 7, 55), 0.6),            # 1155 tokens: 10 blocks, tail of 3
    ("k_all", 1, 4, (4, 16, 40), 0.0),
    ("heads43", 1, 43, (2, 8, 40), 0.75),         # more heads than one pooling CTA covers (42)
]


@pytest.mark.parametrize("name,B,heads,grid,s", ROUTER_CASES, ids=[c[0] for c in ROUTER_CASES])
def test_router_parity_d128(orc, name, B, heads, grid, s):
    d = _inputs(B, heads, grid, "structured" if name != "tiny" else "normal")
    idx = h3a.route(_dev(d["q"]), _dev(d["k"]), s)
    torch.cuda.synchronize()
    ora_idx, ora_sc = orc.route(d["q"], d["k"], s)
    check_router(idx.cpu().numpy(), ora_idx, ora_sc, name)


def test_sparse_with_every_block_equals_dense_bitwise_d128():
    grid, heads = (4, 16, 40), 3
    d = _inputs(1, heads, grid, "structured")
    q, k, v = (_dev(d[n]) for n in "qkv")
    nblk = 20
    all_blocks = torch.arange(nblk, dtype=torch.int32).expand(1, heads, nblk, nblk).contiguous()
    dense = h3a.attention(q, k, v)
    sparse = h3a.attention(q, k, v, all_blocks.cuda())
    torch.cuda.synchronize()
    assert torch.equal(dense, sparse)


def test_identical_keys_give_mean_value_d128():
    grid, heads = (4, 32, 32), 3                  # 4096 tokens
    d = _inputs(1, heads, grid)
    k = d["k"][:, :1].expand(-1, 4096, -1, -1).contiguous()
    o = h3a.attention(_dev(d["q"]), _dev(k), _dev(d["v"]))
    torch.cuda.synchronize()
    mean_v = d["v"].double().mean(dim=1)
    err = (o.cpu().double() - mean_v[:, None]).abs().max().item()
    assert err <= 2e-3, err


def test_layer8k_42_heads_sampled_d128(orc):
    """8,064 tokens x 42 heads x 128: router over all rows, dense and sparse (0.75)
    attention on 2048 sampled rows (seed 1234)."""
    grid, heads = (8, 24, 42), 42
    d = _inputs(1, heads, grid, "structured")
    q, k, v = (_dev(d[n]) for n in "qkv")
    idx = h3a.route(q, k, 0.75)
    o_dense = h3a.attention(q, k, v)
    torch.cuda.synchronize()
    ora_idx, ora_sc = orc.route(d["q"], d["k"], 0.75)
    check_router(idx.cpu().numpy(), ora_idx, ora_sc, "layer8k-d128 router")
    o_sparse = h3a.attention(q, k, v, _dev(torch.from_numpy(ora_idx)))
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0
    rows = synth.sample_rows(1, heads, 8064, 2048).numpy()
    check_attention(gather_rows(o_dense, rows), orc.attention_rows(d["q"], d["k"], d["v"], rows), "d128 dense")
    check_attention(gather_rows(o_sparse, rows), orc.attention_rows(d["q"], d["k"], d["v"], rows, ora_idx),
                    "d128 sparse")


def test_reference_moves_up_d128(orc):
    """Key blocks scaled 0.05, 1, 4, 0.05, 16, 32 (the last one a tail of 16
    keys): most rows move their reference max up at blocks 2 and 4 and two in
    three at the tail, so O (128 columns here) is rescaled in TMEM mid-row."""
    grid, heads = (2, 8, 41), 2                   # 656 tokens, 6 blocks
    d = _inputs(1, heads, grid, seed=5)
    f = torch.tensor([0.05, 1.0, 4.0, 0.05, 16.0, 32.0]).repeat_interleave(128)[:656]
    d["k"] = (d["k"].float() * f[None, :, None, None]).to(torch.bfloat16)
    d["v"] = (d["v"].float() * 0.25).to(torch.bfloat16)   # |O| < 2: one bf16 ulp well inside 2e-2
    o = h3a.attention(_dev(d["q"]), _dev(d["k"]), _dev(d["v"]))
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0
    rows = np.arange(heads * 656)
    check_attention(gather_rows(o, rows), orc.attention_rows(d["q"], d["k"], d["v"], rows), "d128 growing keys")
