"""GPU parity at the full video sizes, in the launch configuration bench.py
times, on a seeded sample of 4096 query rows across all heads (seed 1234).

video5s : 31x48x84 = 124,992 tokens, 56 heads -- dense, and sparse at 0.75
video10s: 61x48x84 = 245,952 tokens, 56 heads -- sparse at 0.80, and dense

The prologue is checked on sampled tokens, the router on every row; the
attention inputs are the oracle's prologue output and the oracle's block lists.
"""
import numpy as np
import pytest
import torch

import rope_block_sparse_b200 as h3a
from rope_block_sparse_b200 import synth
from helpers import bits, check_attention, check_prologue, check_router, from_bits, gather_rows

pytestmark = [pytest.mark.gpu, pytest.mark.slow,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

SAMPLE = 4096


def _stage(orc, name):
    w = synth.WORKLOADS[name]
    d = synth.draw_workload(name)
    g = w.grid
    q, k = d["q"].cuda(), d["k"].cuda()
    qn, kn = h3a.qk_norm_rope(q, k, d["gamma_q"].cuda(), d["gamma_k"].cuda(), g)
    torch.cuda.synchronize()
    # prologue on sampled tokens
    tok = synth.sample_rows(1, 1, w.N, 2048, seed=99).numpy()
    for x, gam, out in ((d["q"], d["gamma_q"], qn), (d["k"], d["gamma_k"], kn)):
        want = orc.round_bf16(orc.qk_norm_rope_tokens(x, gam.numpy(), g, tok))
        check_prologue(bits(out[0, torch.as_tensor(tok).cuda()]), want, f"{name} prologue")
    del q, k, qn, kn
    ora_q = orc.qk_norm_rope_bf16(d["q"], d["gamma_q"].numpy(), g)
    ora_k = orc.qk_norm_rope_bf16(d["k"], d["gamma_k"].numpy(), g)
    return w, d, ora_q, ora_k


def _attention_checks(orc, w, d, ora_q, ora_k, sparsity):
    qd = from_bits(ora_q).cuda()
    kd = from_bits(ora_k).cuda()
    vd = d["v"].cuda()
    rows = synth.sample_rows(w.B, w.heads, w.N, SAMPLE).numpy()
    # router on the oracle's prologue output
    idx = h3a.route(qd, kd, sparsity)
    torch.cuda.synchronize()
    ora_idx, ora_sc = orc.route(ora_q, ora_k, sparsity)
    check_router(idx.cpu().numpy(), ora_idx, ora_sc, f"{w.name} router")
    del ora_sc
    # sparse attention over the oracle's lists
    o = h3a.attention(qd, kd, vd, torch.from_numpy(ora_idx).cuda())
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0
    want = orc.attention_rows(ora_q, ora_k, d["v"], rows, ora_idx)
    check_attention(gather_rows(o, rows), want, f"{w.name} sparse")
    # dense attention
    o = h3a.attention(qd, kd, vd)
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0
    want = orc.attention_rows(ora_q, ora_k, d["v"], rows)
    check_attention(gather_rows(o, rows), want, f"{w.name} dense")


def test_video5s_dense_and_sparse(orc):
    w, d, ora_q, ora_k = _stage(orc, "video5s_sparse")
    _attention_checks(orc, w, d, ora_q, ora_k, 0.75)


def test_video10s_sparse_and_dense(orc):
    w, d, ora_q, ora_k = _stage(orc, "video10s")
    _attention_checks(orc, w, d, ora_q, ora_k, 0.80)


def test_video5s_fused_prologue_pool_route(orc):
    """The fused prologue + pooling and the pooled router at 124,992 tokens, as
    the bench runs them: bit-identical to the unfused calls (outputs and block
    lists), the lists within the router rule of the oracle's, the outputs by the
    prologue rule on sampled tokens."""
    w = synth.WORKLOADS["video5s_sparse"]
    d = synth.draw_workload("video5s_sparse")
    g = w.grid
    q, k = d["q"].cuda(), d["k"].cuda()
    gq, gk = d["gamma_q"].cuda(), d["gamma_k"].cuda()
    qo, ko, ws = h3a.qk_norm_rope_pool(q, k, gq, gk, g)
    idx = h3a.route_pooled(qo, 0.75, ws)
    qu, ku = h3a.qk_norm_rope(q, k, gq, gk, g)
    idx_u = h3a.route(qu, ku, 0.75)
    torch.cuda.synchronize()
    assert torch.equal(qo.view(torch.int16), qu.view(torch.int16))
    assert torch.equal(ko.view(torch.int16), ku.view(torch.int16))
    assert torch.equal(idx, idx_u)
    del qu, ku, idx_u, q, k
    tok = synth.sample_rows(1, 1, w.N, 2048, seed=7).numpy()
    for x, gam, out in ((d["q"], d["gamma_q"], qo), (d["k"], d["gamma_k"], ko)):
        want = orc.round_bf16(orc.qk_norm_rope_tokens(x, gam.numpy(), g, tok))
        check_prologue(bits(out[0, torch.as_tensor(tok).cuda()]), want, "video5s fused prologue")
    ora_idx, ora_sc = orc.route(bits(qo), bits(ko), 0.75)
    check_router(idx.cpu().numpy(), ora_idx, ora_sc, "video5s pooled router")


def test_video5s_d128_dense_and_sparse(orc):
    """The 124,992-token clip at head_dim 128 (42 heads), as bench.py runs it with
    --workload video5s_d128: router on every row, dense and sparse (0.75)
    attention on the 4096 sampled rows; inputs go to the router as drawn."""
    w = synth.WORKLOADS["video5s_d128"]
    d = synth.draw_workload("video5s_d128")
    q, k, v = (d[n].cuda() for n in "qkv")
    idx = h3a.route(q, k, 0.75)
    torch.cuda.synchronize()
    ora_idx, ora_sc = orc.route(d["q"], d["k"], 0.75)
    check_router(idx.cpu().numpy(), ora_idx, ora_sc, "video5s_d128 router")
    del ora_sc
    rows = synth.sample_rows(w.B, w.heads, w.N, SAMPLE).numpy()
    o = h3a.attention(q, k, v, torch.from_numpy(ora_idx).cuda())
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0
    check_attention(gather_rows(o, rows), orc.attention_rows(d["q"], d["k"], d["v"], rows, ora_idx),
                    "video5s_d128 sparse")
    o = h3a.attention(q, k, v)
    torch.cuda.synchronize()
    assert h3a.last_device_error() == 0
    check_attention(gather_rows(o, rows), orc.attention_rows(d["q"], d["k"], d["v"], rows), "video5s_d128 dense")
