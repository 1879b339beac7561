"""The three stages run back to back on the GPU (prologue -> router ->
attention), as bench.py runs them, compared with the oracle's own chain.

Router rows may differ from the oracle's only inside the tie window; query
blocks whose GPU list differs are left out of the attention comparison (their
key sets differ by construction) and counted."""
import numpy as np
import pytest
import torch

import rope_block_sparse_b200 as h3a
from rope_block_sparse_b200 import synth
from helpers import bits, check_attention, check_prologue, check_router, gather_rows

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _chain(orc, d, grid, sparsity, rows):
    q, k, v = (d[n].cuda() for n in "qkv")
    o, blocks = h3a.attention_core(q, k, v, d["gamma_q"].cuda(), d["gamma_k"].cuda(), grid, sparsity)
    qn, kn = h3a.qk_norm_rope(q, k, d["gamma_q"].cuda(), d["gamma_k"].cuda(), grid)
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0
    ora_q = orc.qk_norm_rope_bf16(d["q"], d["gamma_q"].numpy(), grid)
    ora_k = orc.qk_norm_rope_bf16(d["k"], d["gamma_k"].numpy(), grid)
    check_prologue(bits(qn), ora_q, "chain q")
    check_prologue(bits(kn), ora_k, "chain k")
    B, N, H, _ = d["q"].shape
    ora_idx = None
    keep = np.ones(len(rows), dtype=bool)
    if sparsity is not None:
        ora_idx, ora_sc = orc.route(ora_q, ora_k, sparsity)
        gpu_idx = blocks.cpu().numpy()
        check_router(gpu_idx, ora_idx, ora_sc, "chain router")
        same = (gpu_idx == ora_idx).all(axis=-1)            # [B, H, nblk]
        bh, n = rows // N, rows % N
        keep = same.reshape(B * H, -1)[bh, n // 128]
        assert keep.mean() > 0.9
    want = orc.attention_rows(ora_q.reshape(d["q"].shape), ora_k.reshape(d["k"].shape), d["v"], rows[keep],
                              ora_idx)
    check_attention(gather_rows(o, rows[keep]), want, f"chain s={sparsity}")


@pytest.mark.parametrize("sparsity", [None, 0.75])
def test_chain_tiny_and_layer8k(orc, sparsity):
    for name in ("tiny", "layer8k"):
        w = synth.WORKLOADS[name]
        d = synth.draw_workload(name)
        rows = synth.sample_rows(w.B, w.heads, w.N, 2048).numpy()
        _chain(orc, d, w.grid, sparsity, rows)
