"""GPU parity on sizes the oracle finishes in seconds: every output compared.

Inputs of each stage come from the seeded generator or from the oracle (its
prologue output, its block lists), never from a CUDA kernel, so each kernel is
checked on its own; test_gpu_chain.py checks the stages run back to back.
"""
import numpy as np
import pytest
import torch

import rope_block_sparse_b200 as h3a
from rope_block_sparse_b200 import synth
from helpers import (bits, check_attention, check_prologue, check_router, from_bits, gather_rows)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

THETA, EPS = 10000.0, 1e-6


def _inputs(B, heads, grid, dist="normal", seed=0):
    return synth.draw(B, heads, grid, dist, seed)


def _dev(t):
    return t.cuda()


# ---------------------------------------------------------------- self-checks

def test_selftest_mma_matches_torch():
    g = torch.Generator().manual_seed(3)
    a = torch.randn(128, 96, generator=g).to(torch.bfloat16)
    b = torch.randn(128, 96, generator=g).to(torch.bfloat16)
    s, r = h3a.selftest_mma(a.cuda(), b.cuda())
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0
    s_ref = a.double() @ b.double().T
    assert torch.allclose(s.cpu().double(), s_ref, rtol=0, atol=2e-3)
    r_ref = s.cpu().to(torch.bfloat16).double() @ b.double()
    assert torch.allclose(r.cpu().double(), r_ref, rtol=0, atol=2e-2)


def test_bounded_wait_reports_timeout_and_context_survives():
    assert h3a.selftest_wait_timeout(2000) == 4  # H3A_ERR_TIMEOUT
    assert h3a.last_device_error() == 0          # cleared
    d = _inputs(1, 2, (2, 4, 8))
    q, k, v = (_dev(d[n]) for n in "qkv")
    o = h3a.attention(q, k, v)
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0 and torch.isfinite(o.float()).all()


def test_timeout_on_one_stream_is_reported_once_while_attention_runs_on_another():
    """The status word is shared by every stream of the device.  A self-check
    that times out on one stream while dense attention runs on another is
    reported exactly once -- to the reader on its own stream -- and neither the
    attention's stream nor a later read sees it again; the attention result is
    unaffected."""
    assert h3a.last_device_error() == 0
    g = torch.Generator(device="cuda").manual_seed(5)
    N, heads = 16384, 56
    q, k, v = (torch.randn(1, N, heads, 96, device="cuda", generator=g).to(torch.bfloat16) for _ in range(3))
    torch.cuda.synchronize()
    s_attn, s_wait = torch.cuda.Stream(), torch.cuda.Stream()
    with torch.cuda.stream(s_attn):
        o = h3a.attention(q, k, v)  # about 5 ms of work, queued first
    with torch.cuda.stream(s_wait):
        assert h3a.selftest_wait_timeout(2000) == 4  # H3A_ERR_TIMEOUT, taken by this reader
    with torch.cuda.stream(s_attn):
        assert h3a.last_device_error() == 0
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0
    rows = torch.arange(0, N, 977)
    qf, kf, vf = (t[0, :, 3].float() for t in (q, k, v))
    ref = torch.softmax(qf[rows] @ kf.T / 96 ** 0.5, -1) @ vf
    assert (o[0, rows, 3].float() - ref).abs().max().item() <= 2e-2


# ---------------------------------------------------------------- prologue

PROLOGUE_CASES = [
    ("tiny", 1, 2, (2, 4, 8), "normal"),
    ("layer8k", 1, 56, (8, 24, 42), "head_scaled"),
    ("ragged", 2, 5, (3, 5, 7), "normal"),
    ("heads57", 1, 57, (2, 3, 4), "normal"),
]


@pytest.mark.parametrize("name,B,heads,grid,dist", PROLOGUE_CASES, ids=[c[0] for c in PROLOGUE_CASES])
def test_prologue_parity(orc, name, B, heads, grid, dist):
    d = _inputs(B, heads, grid, dist)
    qo, ko = h3a.qk_norm_rope(_dev(d["q"]), _dev(d["k"]), _dev(d["gamma_q"]), _dev(d["gamma_k"]), grid, THETA, EPS)
    torch.cuda.synchronize()
    for x, g, out in ((d["q"], d["gamma_q"], qo), (d["k"], d["gamma_k"], ko)):
        want = orc.qk_norm_rope_bf16(x, g.numpy(), grid, THETA, EPS)
        check_prologue(bits(out), want, name)


def test_prologue_strided_and_inplace(orc):
    """Heads 0..4 of a 7-head buffer (token stride 7*96), in place."""
    grid, heads = (2, 6, 5), 5
    d = _inputs(1, 7, grid)
    qbuf, kbuf = _dev(d["q"]), _dev(d["k"])
    q, k = qbuf[:, :, :heads], kbuf[:, :, :heads]
    untouched = kbuf[:, :, heads:].clone()
    qo, ko = h3a.qk_norm_rope(q, k, _dev(d["gamma_q"]), _dev(d["gamma_k"]), grid, THETA, EPS, inplace=True)
    torch.cuda.synchronize()
    assert qo.data_ptr() == q.data_ptr()
    for x, g, out in ((d["q"], d["gamma_q"], qo), (d["k"], d["gamma_k"], ko)):
        want = orc.qk_norm_rope_bf16(x[:, :, :heads].contiguous(), g.numpy(), grid, THETA, EPS)
        check_prologue(bits(out), want, "strided")
    assert torch.equal(kbuf[:, :, heads:], untouched)


# ---------------------------------------------------------------- router

ROUTER_CASES = [
    ("tiny", 1, 2, (2, 4, 8), 0.75),             # one block: k = 1
    ("layer8k", 1, 56, (8, 24, 42), 0.75),       # 63 blocks, k = 16
    ("ragged", 2, 3, (3, 7, 55), 0.6),           # 1155 tokens: 10 blocks, tail of 3
    ("k_all", 1, 4, (4, 16, 40), 0.0),           # k = nblk
]


@pytest.mark.parametrize("name,B,heads,grid,s", ROUTER_CASES, ids=[c[0] for c in ROUTER_CASES])
def test_router_parity(orc, name, B, heads, grid, s):
    d = _inputs(B, heads, grid, "structured" if name != "tiny" else "normal")
    qb = orc.qk_norm_rope_bf16(d["q"], d["gamma_q"].numpy(), grid)
    kb = orc.qk_norm_rope_bf16(d["k"], d["gamma_k"].numpy(), grid)
    idx = h3a.route(_dev(from_bits(qb)), _dev(from_bits(kb)), s)
    torch.cuda.synchronize()
    ora_idx, ora_sc = orc.route(qb, kb, s)
    check_router(idx.cpu().numpy(), ora_idx, ora_sc, name)


def test_router_exact_ties_pick_lower_index(orc):
    """Key blocks that are exact copies score identically; the lower index wins."""
    grid = (4, 8, 16)                      # 512 tokens, 4 blocks
    d = _inputs(1, 2, grid)
    k = d["k"].clone()
    k[:, 256:384] = k[:, 0:128]            # block 2 == block 0
    k[:, 384:512] = k[:, 128:256]          # block 3 == block 1
    q = d["q"]
    for s in (0.75, 0.5):
        idx = h3a.route(_dev(q), _dev(k), s).cpu().numpy()
        ora_idx, ora_sc = orc.route(q, k, s)
        np.testing.assert_array_equal(idx, ora_idx)
        for row in idx.reshape(-1, idx.shape[-1]):
            sel = set(row.tolist())
            if len(sel) == 1:
                assert sel <= {0, 1}           # one pick among tied copies: the lower index
            for j in (2, 3):                   # a later copy only together with its twin
                assert j not in sel or (j - 2) in sel


# ---------------------------------------------------------------- attention

ATTN_CASES = [
    ("tiny", 1, 2, (2, 4, 8)),               # N = 64 < one tile
    ("one_block", 1, 3, (2, 8, 8)),          # N = 128
    ("tail1", 1, 2, (1, 1, 257)),            # N = 257: a tail of one token
    ("ragged", 2, 3, (3, 11, 13)),           # N = 429, B = 2
    ("odd_tiles", 1, 2, (5, 8, 16)),         # N = 640: 5 tiles, the last pair has one tile
]


@pytest.mark.parametrize("name,B,heads,grid", ATTN_CASES, ids=[c[0] for c in ATTN_CASES])
def test_dense_attention_parity(orc, name, B, heads, grid):
    d = _inputs(B, heads, grid, "normal")
    o = h3a.attention(_dev(d["q"]), _dev(d["k"]), _dev(d["v"]))
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0
    N = grid[0] * grid[1] * grid[2]
    rows = np.arange(B * heads * N)
    want = orc.attention_rows(d["q"], d["k"], d["v"], rows)
    check_attention(gather_rows(o, rows), want, name)


@pytest.mark.parametrize("name,B,heads,grid", ATTN_CASES[2:], ids=[c[0] for c in ATTN_CASES[2:]])
@pytest.mark.parametrize("s", [0.5, 0.8])
def test_sparse_attention_parity(orc, name, B, heads, grid, s):
    d = _inputs(B, heads, grid, "structured")
    ora_idx, _ = orc.route(d["q"], d["k"], s)
    o = h3a.attention(_dev(d["q"]), _dev(d["k"]), _dev(d["v"]), _dev(torch.from_numpy(ora_idx)))
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0
    N = grid[0] * grid[1] * grid[2]
    rows = np.arange(B * heads * N)
    want = orc.attention_rows(d["q"], d["k"], d["v"], rows, ora_idx)
    check_attention(gather_rows(o, rows), want, f"{name}-s{s}")


def test_sparse_with_every_block_equals_dense_bitwise():
    grid, heads = (4, 16, 40), 3                 # 2560 tokens, 20 blocks
    d = _inputs(1, heads, grid, "structured")
    q, k, v = (_dev(d[n]) for n in "qkv")
    nblk = 20
    all_blocks = torch.arange(nblk, dtype=torch.int32).expand(1, heads, nblk, nblk).contiguous()
    dense = h3a.attention(q, k, v)
    sparse = h3a.attention(q, k, v, all_blocks.cuda())
    torch.cuda.synchronize()
    assert torch.equal(dense, sparse)


def test_identical_keys_give_mean_value():
    """All keys equal: every query sees uniform weights, so O = mean(V) per head."""
    grid, heads = (4, 32, 32), 4                 # 4096 tokens
    d = _inputs(1, heads, grid)
    k = d["k"][:, :1].expand(-1, 4096, -1, -1).contiguous()
    o = h3a.attention(_dev(d["q"]), _dev(k), _dev(d["v"]))
    torch.cuda.synchronize()
    mean_v = d["v"].double().mean(dim=1)         # [1, heads, 96]
    err = (o.cpu().double() - mean_v[:, None]).abs().max().item()
    assert err <= 2e-3, err


def test_chain_head_major_storage(orc):
    """Q, K, V and every output stored head-major ([B, heads, N, 96] memory
    viewed as [B, N, heads, 96]: token stride 96, head stride N*96) through
    the prologue, the router and dense and sparse attention, each stage
    against the oracle on the previous stage's GPU output."""
    grid, heads = (3, 8, 25), 3                   # 600 tokens, 5 blocks
    d = _inputs(1, heads, grid, "structured", 8)
    hm = {n: _dev(d[n].transpose(1, 2).contiguous()).transpose(1, 2) for n in "qkv"}
    assert hm["q"].stride() == (heads * 600 * 96, 96, 600 * 96, 1)
    qn, kn = h3a.qk_norm_rope(hm["q"], hm["k"], _dev(d["gamma_q"]), _dev(d["gamma_k"]), grid, THETA, EPS)
    idx = h3a.route(qn, kn, 0.6)
    dense = h3a.attention(qn, kn, hm["v"])
    sparse = h3a.attention(qn, kn, hm["v"], idx)
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0
    assert qn.stride() == dense.stride() == sparse.stride() == hm["q"].stride()
    for x, g, out in ((d["q"], d["gamma_q"], qn), (d["k"], d["gamma_k"], kn)):
        check_prologue(bits(out), orc.qk_norm_rope_bf16(x, g.numpy(), grid, THETA, EPS), "head-major")
    qb, kb = bits(qn), bits(kn)
    ora_idx, ora_sc = orc.route(qb, kb, 0.6)
    gpu_idx = idx.cpu().numpy()
    check_router(gpu_idx, ora_idx, ora_sc, "head-major")
    rows = np.arange(heads * 600)
    check_attention(gather_rows(dense, rows), orc.attention_rows(qb, kb, d["v"], rows), "head-major dense")
    check_attention(gather_rows(sparse, rows), orc.attention_rows(qb, kb, d["v"], rows, gpu_idx),
                    "head-major sparse")


def test_attention_heads_of_a_wider_buffer(orc):
    """Heads 2..6 of a 9-head buffer (token stride 9*96, offset 2*96), output
    written into the same columns of another 9-head buffer; the rest untouched."""
    grid, heads = (2, 8, 20), 9                   # 320 tokens, 3 blocks
    d = _inputs(1, heads, grid, "normal", 9)
    q, k, v = (_dev(d[n])[:, :, 2:7] for n in "qkv")
    obuf = torch.full((1, 320, heads, 96), 7.0, dtype=torch.bfloat16, device="cuda")
    o = obuf[:, :, 2:7]
    h3a.attention(q, k, v, out=o)
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0
    assert bool((obuf[:, :, :2] == 7.0).all()) and bool((obuf[:, :, 7:] == 7.0).all())
    sub = {n: d[n][:, :, 2:7].contiguous() for n in "qkv"}
    rows = np.arange(5 * 320)
    check_attention(gather_rows(o, rows), orc.attention_rows(sub["q"], sub["k"], sub["v"], rows), "head slice")


@pytest.mark.parametrize("scale", [0.02, 0.4])
def test_attention_explicit_scale(orc, scale):
    """A caller-given logit scale instead of 1/sqrt(96): nearly uniform weights
    at 0.02, sharp rows (reference moved up often) at 0.4; dense and sparse."""
    grid, heads = (2, 8, 30), 2                   # 480 tokens, 4 blocks (tail of 96)
    d = _inputs(1, heads, grid, "structured", 10)
    d["v"] = (d["v"].float() * 0.25).to(torch.bfloat16)   # sharp rows: keep |O| < 2
    q, k, v = (_dev(d[n]) for n in "qkv")
    ora_idx, _ = orc.route(d["q"], d["k"], 0.5)
    dense = h3a.attention(q, k, v, scale=scale)
    sparse = h3a.attention(q, k, v, _dev(torch.from_numpy(ora_idx)), scale=scale)
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0
    rows = np.arange(heads * 480)
    check_attention(gather_rows(dense, rows), orc.attention_rows(d["q"], d["k"], d["v"], rows, scale=scale),
                    f"scale {scale} dense")
    check_attention(gather_rows(sparse, rows),
                    orc.attention_rows(d["q"], d["k"], d["v"], rows, ora_idx, scale=scale), f"scale {scale} sparse")


def _growing_keys(heads, grid, scales, seed=5):
    """Seeded inputs whose key block b is scaled by scales[b]: the logits of a
    later block outgrow the reference max fixed by the first block -- by far
    more than 2^8 in the log2 domain for most rows of blocks 2, 4 and the
    ragged tail, by less for others -- so the kernel must move its reference
    up and rescale O and the row sum, in some rows of a warp and not others."""
    d = _inputs(1, heads, grid, "normal", seed)
    N = grid[0] * grid[1] * grid[2]
    assert len(scales) == (N + 127) // 128
    f = torch.tensor(scales, dtype=torch.float32).repeat_interleave(128)[:N]
    d["k"] = (d["k"].float() * f[None, :, None, None]).to(torch.bfloat16)
    # a few keys dominate each row, so O is close to single rows of V: V is
    # scaled down to keep |O| < 2, where one bf16 ulp of the output stays well
    # inside the 2e-2 bound
    d["v"] = (d["v"].float() * 0.25).to(torch.bfloat16)
    return d


GROWING = [0.05, 1.0, 4.0, 0.05, 16.0, 32.0]     # 6 blocks: 5 full + a tail of 16 keys


def test_attention_reference_moves_up_dense(orc):
    grid, heads = (2, 8, 41), 3                  # 656 tokens
    d = _growing_keys(heads, grid, GROWING)
    o = h3a.attention(_dev(d["q"]), _dev(d["k"]), _dev(d["v"]))
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0
    rows = np.arange(heads * 656)
    want = orc.attention_rows(d["q"], d["k"], d["v"], rows)
    check_attention(gather_rows(o, rows), want, "growing keys, dense")


def test_attention_reference_moves_up_sparse(orc):
    """Hand-made ascending lists: a small block first and larger ones after,
    a large block first with a small one after it, the tail block last."""
    grid, heads = (2, 8, 41), 2
    d = _growing_keys(heads, grid, GROWING, seed=6)
    lists = [[0, 2, 3, 5], [2, 3, 4, 5], [0, 1, 2, 4], [1, 3, 4, 5], [0, 3, 4, 5], [1, 2, 4, 5]]
    idx = np.array(lists, dtype=np.int32)[None, None].repeat(heads, axis=1)   # [1, heads, 6, 4]
    o = h3a.attention(_dev(d["q"]), _dev(d["k"]), _dev(d["v"]), _dev(torch.from_numpy(np.ascontiguousarray(idx))))
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0
    rows = np.arange(heads * 656)
    want = orc.attention_rows(d["q"], d["k"], d["v"], rows, idx)
    check_attention(gather_rows(o, rows), want, "growing keys, sparse")


def test_dense_attention_layer8k_sampled(orc):
    d = synth.draw_workload("layer8k")
    o = h3a.attention(_dev(d["q"]), _dev(d["k"]), _dev(d["v"]))
    torch.cuda.synchronize()
    rows = synth.sample_rows(1, 56, 8064, 4096).numpy()
    want = orc.attention_rows(d["q"], d["k"], d["v"], rows)
    check_attention(gather_rows(o, rows), want, "layer8k")


def test_softmax_exp2_within_its_bound():
    """The softmax's exponential (ex2.approx, log2 domain) against 2^x (fp64):
    within the bound CUDA documents for it (2 ulp, here 2^-22 relative) wherever
    the result is a normal float (x >= -125); below that at most 2^-125 (the
    instruction flushes subnormal results; P is zero there for bf16 purposes),
    exactly 0 at -inf (a masked key)."""
    g = torch.Generator().manual_seed(5)
    x = torch.cat([torch.rand(1 << 20, generator=g) * 140.0 - 130.0,
                   torch.tensor([0.0, 0.5, -0.5, 1.0, -1.0, 8.0, -125.0, -126.0, -127.5, -1e4, float("-inf")])])
    want = torch.exp2(x.double())
    y = h3a.selftest_exp2(x.cuda()).cpu().double()
    normal = x >= -125.0
    rel = ((y[normal] - want[normal]).abs() / want[normal]).max().item()
    assert rel <= 2.0 ** -22, rel
    assert (y[~normal].abs() <= 2.0 ** -125).all()
    assert (y >= 0).all() and y[-1].item() == 0.0
