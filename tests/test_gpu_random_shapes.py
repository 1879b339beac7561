"""The whole chain on shapes drawn at random (fixed seed): prologue -> router ->
sparse and dense attention, each stage against the fp64 oracle fed with the
oracle's own inputs to that stage (the prologue's output, the router's lists),
so a mismatch points at one stage.  The shapes cover what hand-picked cases
may miss: ragged tails of every length, odd numbers of query tiles, batch > 1,
head counts that leave a partial head group, and sparsities whose k ranges
from 1 block to all of them."""
import numpy as np
import pytest
import torch

import rope_block_sparse_b200 as h3a
from rope_block_sparse_b200 import synth
from helpers import bits, check_attention, check_prologue, check_router, from_bits, gather_rows

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _shapes(count=10, seed=20260802):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(count):
        B = int(rng.integers(1, 3))
        heads = int(rng.integers(1, 10))
        grid = tuple(int(x) for x in rng.integers(1, 12, size=3))
        grid = (grid[0], grid[1], int(rng.integers(5, 70)))   # N from 5 to ~8k
        s = float(rng.choice([0.0, 0.3, 0.5, 0.75, 0.8, 0.95]))
        out.append((i, B, heads, grid, s))
    return out


@pytest.mark.parametrize("i,B,heads,grid,s", _shapes(), ids=lambda v: str(v))
def test_chain_on_random_shape(orc, i, B, heads, grid, s):
    d = synth.draw(B, heads, grid, "structured", seed=100 + i)
    N = grid[0] * grid[1] * grid[2]
    qn, kn = h3a.qk_norm_rope(d["q"].cuda(), d["k"].cuda(), d["gamma_q"].cuda(), d["gamma_k"].cuda(), grid)
    torch.cuda.synchronize()
    ora_q = orc.qk_norm_rope_bf16(d["q"], d["gamma_q"].numpy(), grid)
    ora_k = orc.qk_norm_rope_bf16(d["k"], d["gamma_k"].numpy(), grid)
    check_prologue(bits(qn), ora_q, f"shape {i} q")
    check_prologue(bits(kn), ora_k, f"shape {i} k")
    # router and attention on the oracle's prologue output
    qd, kd, vd = from_bits(ora_q).cuda(), from_bits(ora_k).cuda(), d["v"].cuda()
    idx = h3a.route(qd, kd, s)
    torch.cuda.synchronize()
    ora_idx, ora_sc = orc.route(ora_q, ora_k, s)
    check_router(idx.cpu().numpy(), ora_idx, ora_sc, f"shape {i} router")
    rows = synth.sample_rows(B, heads, N, 1024, seed=i).numpy()
    o_sparse = h3a.attention(qd, kd, vd, torch.from_numpy(ora_idx).cuda())
    o_dense = h3a.attention(qd, kd, vd)
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0
    check_attention(gather_rows(o_sparse, rows), orc.attention_rows(ora_q, ora_k, d["v"], rows, ora_idx),
                    f"shape {i} sparse")
    check_attention(gather_rows(o_dense, rows), orc.attention_rows(ora_q, ora_k, d["v"], rows), f"shape {i} dense")
