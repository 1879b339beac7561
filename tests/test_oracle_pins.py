"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each test fixes one part of the oracle with a closed form, an invariant, a
special case that reduces to something known, a brute force on tiny inputs
(written here independently, in numpy), or a number the pages print
(tests/golden/page_facts.txt).  They are chosen so that a dropped term, a wrong
sign, index or section, a transposed operand or a wrong tie rule fails at
least one of them.  CPU only.
"""
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
THETA = 10000.0
D = 96


def _facts():
    facts = {}
    with open(os.path.join(GOLDEN, "page_facts.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                key, *vals = line.split()
                facts.setdefault(key, []).append(vals)
    return facts


def _bf16(a) -> torch.Tensor:
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


# ---------------------------------------------------------------- page facts

def test_page_geometry_gives_head_dim_96():
    f = _facts()
    hidden, heads = int(f["hidden"][0][0]), int(f["heads"][0][0])
    assert hidden % heads == 0 and hidden // heads == D
    assert D % 3 == 0 and (D // 3) % 2 == 0  # three RoPE sections of whole pairs


def test_kept_blocks_match_page_sparsities(orc):
    f = _facts()
    sparsities = sorted(float(v[0]) for v in f["sparsity"])
    assert sparsities == [0.75, 0.80]
    for N, s, nblk, kept in f["kept"]:
        assert orc.num_blocks(int(N), 128) == int(nblk)
        assert orc.k_blocks(int(nblk), float(s)) == int(kept)


def test_k_rule_edges(orc):
    assert orc.k_blocks(977, 0.0) == 977       # sparsity 0 keeps everything
    assert orc.k_blocks(10, 0.9) == 1          # 0.1 * 10 = 1 exactly, not 2
    assert orc.k_blocks(4, 0.75) == 1
    assert orc.k_blocks(3, 0.999) == 1         # never below one block
    assert orc.k_blocks(8, 0.5) == 4
    assert orc.k_blocks(7, 0.5) == 4           # 3.5 rounds up


def test_bf16_decoding(orc):
    assert orc.bf16_to_double(0x3F80) == 1.0
    assert orc.bf16_to_double(0xC000) == -2.0
    assert orc.bf16_to_double(0x3E80) == 0.25
    assert orc.bf16_to_double(0x4049) == 3.140625
    assert orc.bf16_to_double(0x0000) == 0.0


# ---------------------------------------------------------------- RMSNorm

def test_rmsnorm_constant_vector(orc):
    for c in (0.5, -3.0, 1e-3):
        y = orc.rmsnorm(np.full(D, c), np.ones(D), 1e-6)
        np.testing.assert_allclose(y, c / math.sqrt(c * c + 1e-6), rtol=1e-14)


def test_rmsnorm_one_hot_uses_own_gain(orc):
    gamma = 1.0 + np.arange(D) / 10.0          # distinct gain per channel
    for i in (0, 37, 95):
        x = np.zeros(D)
        x[i] = 2.0
        y = orc.rmsnorm(x, gamma, 1e-6)
        expect = 2.0 * gamma[i] / math.sqrt(4.0 / D + 1e-6)
        assert abs(y[i] - expect) <= 1e-13 * expect
        assert np.count_nonzero(y) == 1


def test_rmsnorm_mean_square_closed_form(orc):
    rng = np.random.default_rng(0)
    for eps in (1e-6, 0.3):
        x = rng.normal(size=D) * 0.1
        ms = np.mean(x * x)
        y = orc.rmsnorm(x, np.ones(D), eps)
        assert abs(np.mean(y * y) - ms / (ms + eps)) < 1e-14


def test_rmsnorm_scale_invariance(orc):
    rng = np.random.default_rng(1)
    x = rng.normal(size=D)
    g = 1 + 0.1 * rng.normal(size=D)
    y1 = orc.rmsnorm(x, g, 0.0)
    y2 = orc.rmsnorm(7.5 * x, g, 0.0)
    np.testing.assert_allclose(y1, y2, rtol=1e-13)


# ---------------------------------------------------------------- 3D RoPE

def test_rope_identity_at_origin(orc):
    y = np.random.default_rng(2).normal(size=D)
    assert np.array_equal(orc.rope3d(y, (0, 0, 0), THETA), y)


def test_rope_preserves_norm(orc):
    rng = np.random.default_rng(3)
    for _ in range(20):
        y = rng.normal(size=D)
        pos = rng.integers(0, 200, size=3)
        r = orc.rope3d(y, pos, THETA)
        assert abs(np.linalg.norm(r) - np.linalg.norm(y)) <= 1e-12 * np.linalg.norm(y)


def test_rope_relative_offset(orc):
    rng = np.random.default_rng(4)
    for _ in range(20):
        a, b = rng.normal(size=D), rng.normal(size=D)
        p, q, dlt = (rng.integers(0, 90, size=3) for _ in range(3))
        lhs = orc.rope3d(a, p, THETA) @ orc.rope3d(b, q, THETA)
        rhs = orc.rope3d(a, p + dlt, THETA) @ orc.rope3d(b, q + dlt, THETA)
        assert abs(lhs - rhs) <= 1e-10 * (1 + abs(lhs))


@pytest.mark.parametrize("axis", [0, 1, 2])
@pytest.mark.parametrize("j", [0, 1, 8, 15])
@pytest.mark.parametrize("p", [1, 3])
def test_rope_single_axis_closed_form(orc, axis, j, p):
    """Unit vectors of pair j in section `axis`, moved along that axis only,
    turn by p * 10000^(-j/16) (section width 32, theta 10000); nothing else moves."""
    ang = p * THETA ** (-j / 16.0)
    pos = [0, 0, 0]
    pos[axis] = p
    i0 = 32 * axis + 2 * j
    e0 = np.zeros(D)
    e0[i0] = 1.0
    r0 = orc.rope3d(e0, pos, THETA)
    expect0 = np.zeros(D)
    expect0[i0], expect0[i0 + 1] = math.cos(ang), math.sin(ang)
    np.testing.assert_allclose(r0, expect0, atol=1e-15)
    e1 = np.zeros(D)
    e1[i0 + 1] = 1.0
    r1 = orc.rope3d(e1, pos, THETA)
    expect1 = np.zeros(D)
    expect1[i0], expect1[i0 + 1] = -math.sin(ang), math.cos(ang)
    np.testing.assert_allclose(r1, expect1, atol=1e-15)
    # the other two axes leave this section alone
    other = [0, 0, 0]
    other[(axis + 1) % 3] = 5
    other[(axis + 2) % 3] = 7
    np.testing.assert_array_equal(orc.rope3d(e0, other, THETA), e0)


def test_token_position_row_major(orc):
    grid = (3, 4, 5)
    assert orc.token_position(0, grid) == (0, 0, 0)
    assert orc.token_position(1, grid) == (0, 0, 1)
    assert orc.token_position(5, grid) == (0, 1, 0)
    assert orc.token_position(20, grid) == (1, 0, 0)
    assert orc.token_position(59, grid) == (2, 3, 4)


# ---------------------------------------------------------------- fused prologue

def test_prologue_is_norm_then_rope(orc):
    """Per token and head: RMSNorm with gains, then RoPE at the token's grid
    position; the order matters because the gains are per channel."""
    rng = np.random.default_rng(5)
    grid = (2, 3, 4)
    B, heads = 2, 3
    N = 24
    x = _bf16(rng.normal(size=(B, N, heads, D)))
    gamma = (1 + 0.1 * rng.normal(size=D)).astype(np.float32)
    out = orc.qk_norm_rope(x, gamma, grid, THETA, 1e-6)
    xf = x.float().numpy().astype(np.float64)
    for b, n, h in [(0, 0, 0), (1, 23, 2), (0, 17, 1), (1, 5, 0)]:
        pos = orc.token_position(n, grid)
        want = orc.rope3d(orc.rmsnorm(xf[b, n, h], gamma.astype(np.float64), 1e-6), pos, THETA)
        np.testing.assert_allclose(out[b, n, h], want, rtol=0, atol=1e-14)
        wrong = orc.rmsnorm(orc.rope3d(xf[b, n, h], pos, THETA), gamma.astype(np.float64), 1e-6)
        if pos != (0, 0, 0):
            assert np.max(np.abs(out[b, n, h] - wrong)) > 1e-6


def test_prologue_constant_input_closed_form(orc):
    """x = c on every channel, unit gains, token 0 (position (0,0,0)):
    y = c / sqrt(c^2 + eps) on every channel."""
    x = _bf16(np.full((1, 4, 1, D), 0.5))
    out = orc.qk_norm_rope(x, np.ones(D, np.float32), (1, 2, 2), THETA, 1e-6)
    np.testing.assert_allclose(out[0, 0, 0], 0.5 / math.sqrt(0.25 + 1e-6), rtol=1e-14)
    # mean square is position independent (RoPE is a rotation)
    for n in range(4):
        assert abs(np.mean(out[0, n, 0] ** 2) - 0.25 / (0.25 + 1e-6)) < 1e-14


def test_prologue_position_reaches_right_section(orc):
    """Token n = H*W sits at (1, 0, 0): only the t-section turns, by angle 1 for pair 0."""
    grid = (2, 3, 4)
    x = np.zeros((1, 24, 1, D), np.float32)
    x[0, 12, 0, :] = 1.0
    out = orc.qk_norm_rope(_bf16(x), np.ones(D, np.float32), grid, THETA, 0.0)
    y = out[0, 12, 0]
    # pair 0 of section t: (1, 1) turned by 1 rad
    assert abs(y[0] - (math.cos(1) - math.sin(1))) < 1e-14
    assert abs(y[1] - (math.sin(1) + math.cos(1))) < 1e-14
    np.testing.assert_allclose(y[32:], 1.0, rtol=1e-14)  # h and w sections at position 0


# ---------------------------------------------------------------- router

def _router_case(N, block, heads, coeff_fn, q_dir=None):
    """q tokens all equal u; K tokens of block j equal coeff(j) * u (u a fixed unit-ish vector)."""
    u = np.zeros(D, np.float32)
    u[:4] = 0.5  # |u| = 1, exactly representable
    q = np.zeros((1, N, heads, D), np.float32)
    k = np.zeros((1, N, heads, D), np.float32)
    q[:] = u if q_dir is None else q_dir
    for n in range(N):
        for h in range(heads):
            k[0, n, h] = coeff_fn(n // block, h) * u
    return _bf16(q), _bf16(k)


def test_router_selects_largest_constructed_scores(orc):
    block, nblk, heads = 8, 10, 2
    coeffs = np.array([[3, 9, 1, 7, 5, 0.5, 8, 2, 6, 4],
                       [9, 8, 7, 6, 5, 4, 3, 2, 1, 0.5]], np.float32)
    q, k = _router_case(block * nblk, block, heads, lambda j, h: coeffs[h, j])
    idx, sc = orc.route(q, k, 0.7, block)
    assert idx.shape == (1, heads, nblk, 3)
    for i in range(nblk):
        assert idx[0, 0, i].tolist() == [1, 3, 6]     # coefficients 9, 8, 7
        assert idx[0, 1, i].tolist() == [0, 1, 2]
    # scores are (u . c u) / sqrt(96) = c / sqrt(96), rounded to fp32
    np.testing.assert_array_equal(sc[0, 0, 0], (coeffs[0].astype(np.float64) / math.sqrt(D)).astype(np.float32))


def test_router_ties_go_to_lower_index(orc):
    block, nblk = 4, 8
    coeffs = [1, 5, 2, 5, 5, 0, 5, 1]
    q, k = _router_case(block * nblk, block, 1, lambda j, h: coeffs[j])
    idx, _ = orc.route(q, k, 0.75, block)     # k = 2 of four tied blocks
    assert idx[0, 0, 0].tolist() == [1, 3]
    idx, _ = orc.route(q, k, 0.5, block)      # k = 4: all ties kept
    assert idx[0, 0, 0].tolist() == [1, 3, 4, 6]
    idx, _ = orc.route(q, k, 0.4, block)      # k = 5: next best (2) after the ties
    assert idx[0, 0, 0].tolist() == [1, 2, 3, 4, 6]


def test_router_tail_block_mean_uses_real_length(orc):
    """Last block holds 3 of 8 tokens, all 1.5 u; a mean over 8 would give 0.5625 u."""
    block, N = 8, 3 * 8 + 3
    q, k = _router_case(N, block, 1, lambda j, h: 1.5 if j == 3 else 1.0)
    idx, sc = orc.route(q, k, 0.75, block)    # 4 blocks, keep 1
    assert idx[0, 0, 0].tolist() == [3]
    assert sc[0, 0, 0, 3] == np.float32(1.5 / math.sqrt(D))


def test_router_scores_respect_query_block(orc):
    """Query blocks pointing at different directions pick different key blocks."""
    block, nblk = 4, 4
    e = np.eye(D, dtype=np.float32)
    q = np.zeros((1, block * nblk, 1, D), np.float32)
    k = np.zeros_like(q)
    for j in range(nblk):
        q[0, j * block:(j + 1) * block, 0] = e[j]
        k[0, j * block:(j + 1) * block, 0] = e[(j + 1) % nblk]
    idx, _ = orc.route(_bf16(q), _bf16(k), 0.75, block)
    assert [idx[0, 0, i, 0] for i in range(nblk)] == [3, 0, 1, 2]


def test_router_permutation_equivariance(orc):
    rng = np.random.default_rng(6)
    block, nblk, heads = 4, 12, 2
    q = _bf16(rng.normal(size=(1, block * nblk, heads, D)))
    k = rng.normal(size=(1, block * nblk, heads, D)).astype(np.float32)
    perm = rng.permutation(nblk)
    kp = k.reshape(1, nblk, block, heads, D)[:, perm].reshape(k.shape)
    idx, _ = orc.route(q, _bf16(k), 0.7, block)
    idxp, _ = orc.route(q, _bf16(kp), 0.7, block)
    inv = np.argsort(perm)
    for h in range(heads):
        for i in range(nblk):
            assert sorted(perm[idxp[0, h, i]].tolist()) == idx[0, h, i].tolist()
            assert sorted(inv[idx[0, h, i]].tolist()) == idxp[0, h, i].tolist()


def test_router_brute_force_tiny(orc):
    """Independent numpy restatement on a tiny random grid: block means, scaled
    dot products, a full stable sort by (-score, index)."""
    rng = np.random.default_rng(7)
    block, B, heads, N = 8, 2, 3, 8 * 9 + 5
    q = _bf16(rng.normal(size=(B, N, heads, D)))
    k = _bf16(rng.normal(size=(B, N, heads, D)))
    s = 0.6
    idx, sc = orc.route(q, k, s, block)
    qf, kf = q.double().numpy(), k.double().numpy()
    nblk = -(-N // block)
    kk = math.ceil((1 - s) * nblk - 1e-9)
    for b in range(B):
        for h in range(heads):
            qm = np.stack([qf[b, i * block:(i + 1) * block, h].mean(0) for i in range(nblk)]).astype(np.float32)
            km = np.stack([kf[b, j * block:(j + 1) * block, h].mean(0) for j in range(nblk)]).astype(np.float32)
            S = (qm.astype(np.float64) @ km.astype(np.float64).T / math.sqrt(D)).astype(np.float32)
            np.testing.assert_array_equal(sc[b, h], S)
            for i in range(nblk):
                order = sorted(range(nblk), key=lambda j: (-float(S[i, j]), j))
                assert idx[b, h, i].tolist() == sorted(order[:kk])


def test_topk_output_is_ascending_and_unique(orc):
    rng = np.random.default_rng(8)
    s = rng.normal(size=(5, 50)).astype(np.float32)
    s[:, 10] = s[:, 20] = s[:, 30] = 4.0
    out = orc.topk(s, 7)
    for row in out:
        assert list(row) == sorted(set(row.tolist()))
        assert {10, 20, 30} <= set(row.tolist())


# ---------------------------------------------------------------- attention

def _rows_all(B, heads, N):
    return np.arange(B * heads * N, dtype=np.int64)


def test_attention_identical_keys_give_mean_v(orc):
    rng = np.random.default_rng(9)
    B, N, heads = 1, 40, 2
    q = _bf16(rng.normal(size=(B, N, heads, D)))
    krow = rng.normal(size=(1, 1, heads, D))
    k = _bf16(np.broadcast_to(krow, (B, N, heads, D)))
    v = _bf16(rng.normal(size=(B, N, heads, D)))
    out = orc.attention_rows(q, k, v, _rows_all(B, heads, N))
    vf = v.double().numpy()
    for h in range(heads):
        want = vf[0, :, h].mean(0)
        for n in range(N):
            np.testing.assert_allclose(out[h * N + n], want, rtol=0, atol=1e-13)


def test_attention_two_keys_closed_form(orc):
    q = np.zeros((1, 2, 1, D), np.float32)
    k = np.zeros_like(q)
    v = np.zeros_like(q)
    q[0, :, 0, 0] = 1.0
    k[0, 0, 0, 0], k[0, 1, 0, 0] = 2.0, -1.0        # logits 2/sqrt(96), -1/sqrt(96)
    v[0, 0, 0, 5], v[0, 1, 0, 7] = 1.0, 1.0
    out = orc.attention_rows(_bf16(q), _bf16(k), _bf16(v), np.array([0]))
    w0 = 1.0 / (1.0 + math.exp(-3.0 / math.sqrt(D)))
    assert abs(out[0, 5] - w0) < 1e-15 and abs(out[0, 7] - (1 - w0)) < 1e-15
    assert np.count_nonzero(out[0]) == 2


def test_attention_dominant_key_returns_its_value(orc):
    """One logit near 1000 above the rest: the output is that key's value; an
    implementation without the max shift would overflow here."""
    rng = np.random.default_rng(10)
    N = 33
    q = np.zeros((1, N, 1, D), np.float32)
    q[0, :, 0, 0] = 64.0
    k = rng.normal(size=(1, N, 1, D)).astype(np.float32) * 0.01
    k[0, 17, 0, 0] = 152.0                           # 64*152/sqrt(96) ~ 993
    v = rng.normal(size=(1, N, 1, D)).astype(np.float32)
    vb = _bf16(v)
    out = orc.attention_rows(_bf16(q), _bf16(k), vb, np.array([0, 5, 32]))
    for r in range(3):
        np.testing.assert_allclose(out[r], vb.double().numpy()[0, 17, 0], rtol=0, atol=1e-12)


def test_attention_matches_logsumexp_brute_force(orc):
    """A second formulation on tiny grids: weights exp(l - logsumexp(l)) over all keys at once."""
    rng = np.random.default_rng(11)
    for (B, N, heads) in [(1, 64, 2), (2, 8, 3)]:
        q, k, v = (_bf16(rng.normal(size=(B, N, heads, D))) for _ in range(3))
        out = orc.attention_rows(q, k, v, _rows_all(B, heads, N))
        qf, kf, vf = (t.double().numpy() for t in (q, k, v))
        for b in range(B):
            for h in range(heads):
                L = qf[b, :, h] @ kf[b, :, h].T / math.sqrt(D)
                mx = L.max(axis=1, keepdims=True)
                lse = mx + np.log(np.exp(L - mx).sum(axis=1, keepdims=True))
                want = np.exp(L - lse) @ vf[b, :, h]
                got = out[(b * heads + h) * N:(b * heads + h + 1) * N]
                np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_attention_key_permutation_invariance(orc):
    rng = np.random.default_rng(12)
    N = 50
    q, k, v = (rng.normal(size=(1, N, 1, D)).astype(np.float32) for _ in range(3))
    perm = rng.permutation(N)
    a = orc.attention_rows(_bf16(q), _bf16(k), _bf16(v), np.arange(N))
    b = orc.attention_rows(_bf16(q), _bf16(k[:, perm]), _bf16(v[:, perm]), np.arange(N))
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)


def test_sparse_with_every_block_equals_dense_bitwise(orc):
    rng = np.random.default_rng(13)
    block, N, heads = 8, 8 * 5 + 3, 2
    q, k, v = (_bf16(rng.normal(size=(1, N, heads, D))) for _ in range(3))
    nblk = -(-N // block)
    idx, _ = orc.route(q, k, 0.0, block)
    assert idx.shape[-1] == nblk and (idx[0, :, :] == np.arange(nblk)).all()
    rows = _rows_all(1, heads, N)
    dense = orc.attention_rows(q, k, v, rows, None, block)
    sparse = orc.attention_rows(q, k, v, rows, idx, block)
    assert np.array_equal(dense, sparse)


def test_sparse_single_block_is_dense_on_that_block(orc):
    rng = np.random.default_rng(14)
    block, nblk, heads = 8, 6, 1
    N = block * nblk - 5                                # ragged tail block of 3
    q, k, v = (_bf16(rng.normal(size=(1, N, heads, D))) for _ in range(3))
    lists = np.array([[[[5], [0], [2], [5], [1], [3]]]], np.int32)  # one block per query block
    out = orc.attention_rows(q, k, v, np.arange(N), lists, block)
    qf, kf, vf = (t.double().numpy()[0, :, 0] for t in (q, k, v))
    for n in range(N):
        j = lists[0, 0, n // block, 0]
        keys = np.arange(j * block, min(N, (j + 1) * block))
        L = qf[n] @ kf[keys].T / math.sqrt(D)
        w = np.exp(L - L.max())
        np.testing.assert_allclose(out[n], (w / w.sum()) @ vf[keys], rtol=0, atol=1e-12)


def test_round_bf16_nearest_even_from_fp64(orc):
    """Rounding is taken once, straight from fp64: halfway cases go to even, and
    1 + 2^-8 + 2^-30 (just above halfway) rounds up -- a detour through fp32
    would round it to the halfway point first and then down to even."""
    x = np.array([1.0, 1 + 2 ** -8, 1 + 1.5 * 2 ** -8, 1 + 2 ** -9, 1 + 2 ** -8 + 2 ** -30, -3.14159,
                  1e-40, 3.4e38, 3.39e38, 0.0, 1.5 * 2 ** -133])
    got = orc.round_bf16(x).tolist()
    assert got == [0x3F80, 0x3F80, 0x3F81, 0x3F80, 0x3F81, 0xC049, 0x0001, 0x7F80, 0x7F7F, 0x0000, 0x0002]


def test_prologue_variants_agree(orc):
    """The token-subset and bf16-output forms restate the same per-token steps."""
    rng = np.random.default_rng(15)
    grid = (2, 3, 5)
    x = _bf16(rng.normal(size=(2, 30, 3, D)))
    g = (1 + 0.1 * rng.normal(size=D)).astype(np.float32)
    full = orc.qk_norm_rope(x, g, grid)
    toks = np.array([0, 7, 29, 30, 59])
    sub = orc.qk_norm_rope_tokens(x, g, grid, toks)
    np.testing.assert_array_equal(sub, full.reshape(60, 3, D)[toks])
    np.testing.assert_array_equal(orc.qk_norm_rope_bf16(x, g, grid), orc.round_bf16(full))


# ---------------------------------------------------------------- gated residual + AdaLN, SwiGLU

def _zeros(B, C):
    return np.zeros((B, C), dtype=np.float32)


def test_adaln_hand_example(orc):
    """C = 2, x = [1, 3], eps = 0: mean 2, variance 1, so LayerNorm gives [-1, 1];
    with scale [0.5, 0] and shift [0, 10] the update gives [-1.5, 11]."""
    x = _bf16([[[1.0, 3.0]]])
    h, y = orc.residual_adaln(x, None, None, np.array([[0.0, 10.0]], np.float32),
                              np.array([[0.5, 0.0]], np.float32), eps=0.0)
    assert np.array_equal(h, x.view(torch.int16).numpy().view(np.uint16))
    assert np.allclose(y, [[[-1.5, 11.0]]], rtol=0, atol=1e-15)


def test_adaln_normalises_rows(orc):
    """No residual, scale = shift = 0: every row has mean 0 and mean square
    var / (var + eps) (closed form of the normalisation)."""
    x = torch.randn(2, 5, 96, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    eps = 1e-2
    h, y = orc.residual_adaln(x, None, None, _zeros(2, 96), _zeros(2, 96), eps=eps)
    xd = x.double().numpy()
    var = xd.var(axis=-1)
    assert np.allclose(y.mean(axis=-1), 0.0, atol=1e-13)
    assert np.allclose((y ** 2).mean(axis=-1), var / (var + eps), rtol=1e-12)


def test_adaln_modulation_is_affine_per_channel(orc):
    """y(scale, shift) = y(0, 0) * (1 + scale) + shift, channel by channel and per batch."""
    g = torch.Generator().manual_seed(4)
    x = torch.randn(2, 3, 40, generator=g).to(torch.bfloat16)
    sc = torch.randn(2, 40, generator=g).numpy().astype(np.float32)
    sh = torch.randn(2, 40, generator=g).numpy().astype(np.float32)
    _, y0 = orc.residual_adaln(x, None, None, _zeros(2, 40), _zeros(2, 40))
    _, y = orc.residual_adaln(x, None, None, sh, sc)
    want = y0 * (1.0 + sc.astype(np.float64))[:, None, :] + sh.astype(np.float64)[:, None, :]
    assert np.allclose(y, want, rtol=0, atol=1e-12)


def test_adaln_ignores_a_constant_offset(orc):
    """LayerNorm removes the row mean: adding 4 to every channel of integer-valued
    rows (exact in bf16) leaves y unchanged."""
    x = torch.randint(-8, 9, (1, 4, 32), generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    sh = np.linspace(-1, 1, 32, dtype=np.float32)[None]
    sc = np.linspace(0, 2, 32, dtype=np.float32)[None]
    _, y0 = orc.residual_adaln(x, None, None, sh, sc)
    _, y1 = orc.residual_adaln(x + 4, None, None, sh, sc)
    assert np.allclose(y0, y1, rtol=0, atol=1e-13)


def test_gated_residual_terms(orc):
    """h = x + gate * f: gate 0 gives x bit for bit; x = [1, 1], f = [1, -1] and
    gate [2, 2] give [3, -1]; f = x with gate 1 doubles x exactly."""
    g = torch.Generator().manual_seed(6)
    x = torch.randn(2, 3, 16, generator=g).to(torch.bfloat16)
    f = torch.randn(2, 3, 16, generator=g).to(torch.bfloat16)
    xbits = x.view(torch.int16).numpy().view(np.uint16)
    h, _ = orc.residual_adaln(x, f, _zeros(2, 16), _zeros(2, 16), _zeros(2, 16))
    assert np.array_equal(h, xbits)
    h, _ = orc.residual_adaln(x, x, np.ones((2, 16), np.float32), _zeros(2, 16), _zeros(2, 16))
    assert np.array_equal(h, (x * 2).view(torch.int16).numpy().view(np.uint16))
    h, _ = orc.residual_adaln(_bf16([[[1.0, 1.0]]]), _bf16([[[1.0, -1.0]]]), np.full((1, 2), 2.0, np.float32),
                              _zeros(1, 2), _zeros(1, 2))
    assert np.array_equal(h, _bf16([[[3.0, -1.0]]]).view(torch.int16).numpy().view(np.uint16))


def test_gated_residual_gate_is_per_batch(orc):
    """The gate of batch b scales only batch b's branch."""
    x = torch.zeros(2, 1, 8).to(torch.bfloat16)
    f = torch.ones(2, 1, 8).to(torch.bfloat16)
    gate = np.stack([np.full(8, 0.5), np.full(8, -2.0)]).astype(np.float32)
    h, _ = orc.residual_adaln(x, f, gate, _zeros(2, 8), _zeros(2, 8))
    got = torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).float().numpy()
    assert np.array_equal(got[0], np.full((1, 8), 0.5)) and np.array_equal(got[1], np.full((1, 8), -2.0))


def test_swiglu_identities(orc):
    """silu(a) - silu(-a) = a for any a (sigma(a) + sigma(-a) = 1), silu(0) = 0,
    silu(a) -> a for large a and -> 0 for very negative a, b = 0 gives 0;
    the first half of a row is the gated input a, the second half b."""
    a = np.array([0.75, 1.5, 3.0, -2.25, 0.0, 40.0, -40.0], np.float32)
    row = np.concatenate([a, -a, np.ones(7, np.float32), np.ones(7, np.float32)])[None]
    out = orc.swiglu(_bf16(row))[0]
    ab = _bf16(a).double().numpy()
    assert np.allclose(out[:7] - out[7:], ab, rtol=0, atol=1e-14)
    assert out[4] == 0.0
    assert abs(out[5] - 40.0) < 1e-15 * 40 + 1e-14 and abs(out[12]) < 1e-15
    zero_b = np.concatenate([a, np.zeros(7, np.float32)])[None]
    assert np.all(orc.swiglu(_bf16(zero_b)) == 0.0)


def test_swiglu_scales_linearly_in_b(orc):
    """out(a, c * b) = c * out(a, b) for a power-of-two c (exact scaling)."""
    g = torch.Generator().manual_seed(7)
    a = torch.randn(3, 10, generator=g)
    b = torch.randn(3, 10, generator=g)
    o1 = orc.swiglu(torch.cat([a, b], 1).to(torch.bfloat16))
    o2 = orc.swiglu(torch.cat([a, 4 * b], 1).to(torch.bfloat16))
    assert np.allclose(o2, 4 * o1, rtol=1e-15, atol=0)


# ---------------------------------------------------------------- Cache-DiT residual difference

def test_residual_diff_closed_forms(orc):
    """Equal tensors give 0; prev = 2 * cur gives |cur - 2cur| / |2cur| = 1/2 exactly;
    cur = 0 gives 1; cur = -prev gives 2; prev is the base (cur = 2 * prev gives 1,
    not 1/2); all-zero inputs give 0 and a zero base with a nonzero cur gives inf."""
    g = torch.Generator().manual_seed(8)
    b = torch.randn(1000, generator=g).to(torch.bfloat16)
    assert orc.residual_diff(b, b) == 0.0
    assert orc.residual_diff(b, b * 2) == 0.5
    assert orc.residual_diff(b * 2, b) == 1.0
    assert orc.residual_diff(torch.zeros_like(b), b) == 1.0
    assert orc.residual_diff(-b, b) == 2.0
    z = torch.zeros(16, dtype=torch.bfloat16)
    assert orc.residual_diff(z, z) == 0.0
    assert orc.residual_diff(torch.ones(16, dtype=torch.bfloat16), z) == math.inf


def test_residual_diff_hand_example_and_scale_invariance(orc):
    """cur = [1, 2, 3, 4], prev = [1, 1, 4, 2]: |diff| = 0+1+1+2 = 4, |prev| = 8 -> 0.5;
    scaling both by 2^k leaves it unchanged."""
    cur, prev = _bf16([1, 2, 3, 4]), _bf16([1, 1, 4, 2])
    assert orc.residual_diff(cur, prev) == 0.5
    g = torch.Generator().manual_seed(9)
    a = torch.randn(777, generator=g).to(torch.bfloat16)
    c = torch.randn(777, generator=g).to(torch.bfloat16)
    r = orc.residual_diff(a, c)
    assert orc.residual_diff(a * 8, c * 8) == pytest.approx(r, rel=1e-15)


# ---------------------------------------------------------------- full-width QK-RMSNorm

def test_fullnorm_with_one_head_is_the_per_head_prologue(orc):
    """With a single head the hidden state is the head: the full-width prologue
    equals the per-head one bit for bit."""
    g = torch.Generator().manual_seed(10)
    x = torch.randn(1, 60, 1, D, generator=g).to(torch.bfloat16)
    gamma = (1 + 0.1 * torch.randn(D, generator=g)).numpy().astype(np.float32)
    grid = (3, 4, 5)
    assert np.array_equal(orc.qk_fullnorm_rope_bf16(x, gamma, grid), orc.qk_norm_rope_bf16(x, gamma, grid))


def test_fullnorm_couples_the_heads(orc):
    """At the grid origin (RoPE is the identity) with unit gains: every head of a
    token is divided by the same RMS over all its heads.  Head 0 = 1 everywhere,
    head 1 = 3 everywhere: mean square (1 + 9) / 2 = 5, so the outputs are
    1/sqrt(5) and 3/sqrt(5) (eps 0), where the per-head norm would give 1 and 1."""
    x = torch.cat([torch.ones(1, 1, 1, D), 3 * torch.ones(1, 1, 1, D)], dim=2).to(torch.bfloat16)
    out = orc.qk_fullnorm_rope_bf16(x, np.ones(2 * D, np.float32), (1, 1, 1), eps=0.0)
    got = torch.from_numpy(out.view(np.int16)).view(torch.bfloat16).double().numpy()[0, 0]
    want = torch.tensor([1 / math.sqrt(5), 3 / math.sqrt(5)]).to(torch.bfloat16).double().numpy()
    assert np.array_equal(got[0], np.full(D, want[0])) and np.array_equal(got[1], np.full(D, want[1]))


def test_fullnorm_gain_indexes_the_hidden_channel(orc):
    """gamma has one entry per hidden channel: zero gains on head 1 only silence head 1."""
    g = torch.Generator().manual_seed(11)
    x = torch.randn(1, 12, 2, D, generator=g).to(torch.bfloat16)
    gamma = np.ones(2 * D, np.float32)
    gamma[D:] = 0.0
    out = orc.qk_fullnorm_rope_bf16(x, gamma, (1, 3, 4))
    assert np.all((out[:, :, 1] & 0x7FFF) == 0) and np.any(out[:, :, 0] != 0)
