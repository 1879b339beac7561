"""h3a_route_noalloc -- the router for callers that cannot allocate device
memory (a runtime that hands out no allocator after start-up, code inside a
host callback, a fixed memory budget) -- called through the C ABI and checked
against h3a_route with a caller workspace.  Router results are compared bit
for bit, as everywhere in these tests (both calls run the same kernels on the
same inputs).  Two calls in a row with different shapes check that the shared
built-in scratch carries nothing from one call into the next.  Collected last
on purpose, so that a stop-at-first-failure run has executed everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

from rope_block_sparse_b200 import h3a, synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _route_noalloc(q, k, sparsity, out):
    lib = h3a.load()
    d = h3a.desc_of(q)
    kk = ctypes.c_int64(0)
    status = lib.h3a_route_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.byref(d),
                                   float(sparsity), 128, ctypes.c_void_p(out.data_ptr()), ctypes.byref(kk),
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return status, kk.value


def test_noalloc_route_matches_route_on_two_calls_in_a_row():
    cases = [((1, 56, (8, 24, 42), "head_scaled", 0), 0.75),   # 8,064 tokens, 63 blocks
             ((2, 3, (3, 7, 55), "structured", 1), 0.6)]        # 1,155 tokens, ragged tail, B = 2
    for (B, heads, grid, dist, seed), s in cases:
        d = synth.draw(B, heads, grid, dist, seed)
        q, k = d["q"].cuda(), d["k"].cuda()
        want = h3a.route(q, k, s)
        out = torch.full_like(want, -7)
        status, kk = _route_noalloc(q, k, s, out)
        torch.cuda.synchronize()
        assert status == 0, h3a.STATUS_NAMES.get(status, status)
        assert kk == want.shape[-1]
        assert h3a.last_device_error() == 0
        np.testing.assert_array_equal(out.cpu().numpy(), want.cpu().numpy())


def test_noalloc_route_rejects_shapes_beyond_its_scratch():
    """2 x 56 heads x 977 blocks needs 84 MB of pooled means > 64 MiB: refused, nothing launched."""
    B, N, heads = 2, 124992, 56
    q = torch.zeros((B, N, heads, 96), dtype=torch.bfloat16, device="cuda")
    out = torch.full((B, heads, 977, 245), -7, dtype=torch.int32, device="cuda")
    status, _ = _route_noalloc(q, q, 0.75, out)
    torch.cuda.synchronize()
    assert status == 5  # H3A_ERR_WORKSPACE
    assert bool((out == -7).all())
