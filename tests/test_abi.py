"""The C-ABI library without a GPU: it loads, exports every function the
header declares, and its host-side rules (k per sparsity, workspace size,
argument validation) behave as documented.  No call here reaches a kernel:
every call either fails validation or needs no device."""
import ctypes
import os
import re

import pytest
import torch

from rope_block_sparse_b200 import h3a

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "h3a.h")
NO_GPU = pytest.mark.skipif(torch.cuda.is_available(), reason="fake device pointers: CPU-only check")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(h3a_[a-z0-9_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert _declared() == sorted(h3a.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = h3a.load()
    for name in _declared():
        assert hasattr(lib, name), name
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)


def test_status_strings():
    lib = h3a.load()
    for code, name in h3a.STATUS_NAMES.items():
        assert lib.h3a_status_string(code).decode() == name
    assert lib.h3a_status_string(99).decode() == "H3A_ERR_UNKNOWN"


def test_route_k_matches_oracle(orc):
    for nkv in (1, 2, 7, 63, 977, 1922, 5000):
        for s in (0.0, 0.1, 0.5, 0.75, 0.8, 0.9, 0.99):
            assert h3a.route_k(nkv, s) == orc.k_blocks(nkv, s), (nkv, s)
    assert h3a.route_k(10, 1.0) == -1
    assert h3a.route_k(10, -0.1) == -1
    assert h3a.route_k(0, 0.5) == -1


def _desc(B=1, N=8064, heads=56, D=96):
    return h3a.QkvDesc(B, N, heads, D, N * heads * D, heads * D, D)


def test_workspace_size():
    lib = h3a.load()
    n = ctypes.c_size_t()
    d = _desc(N=124992)
    assert lib.h3a_route_workspace_size(ctypes.byref(d), 128, ctypes.byref(n)) == 0
    nblk, nblk4 = 977, 980  # K's means are channel-major, rows of key blocks padded to a multiple of 4
    a256 = lambda x: (x + 255) // 256 * 256
    assert n.value == a256(56 * nblk * 96 * 4) + a256(56 * 96 * nblk4 * 4)
    assert lib.h3a_route_workspace_size(ctypes.byref(d), 64, ctypes.byref(n)) == 2  # block must be 128
    # 42 heads x 128 (the same 5376-wide hidden state): the router takes head_dim 128
    wide = _desc(N=124992, heads=42, D=128)
    assert lib.h3a_route_workspace_size(ctypes.byref(wide), 128, ctypes.byref(n)) == 0
    assert n.value == a256(42 * nblk * 128 * 4) + a256(42 * 128 * nblk4 * 4)
    bad = _desc(D=64)
    assert lib.h3a_route_workspace_size(ctypes.byref(bad), 128, ctypes.byref(n)) == 2


P = ctypes.c_void_p
GOOD = P(0x10000)       # aligned, never dereferenced: every call below fails validation
MISALIGNED = P(0x10008)


@NO_GPU
def test_prologue_validation():
    lib = h3a.load()
    d = _desc(N=8064)
    grid = h3a.Grid(8, 24, 42)
    args = lambda **kw: dict(dict(q=GOOD, k=GOOD, d=ctypes.byref(d), gq=GOOD, gk=GOOD, grid=grid, theta=1e4,
                                  eps=1e-6, qo=GOOD, ko=GOOD, st=None), **kw)

    def call(**kw):
        a = args(**kw)
        return lib.h3a_qk_norm_rope(a["q"], a["k"], a["d"], a["gq"], a["gk"], a["grid"], a["theta"], a["eps"],
                                    a["qo"], a["ko"], a["st"])

    assert call(q=None) == 1
    assert call(ko=None) == 1
    assert call(q=MISALIGNED) == 1
    assert call(grid=h3a.Grid(8, 24, 41)) == 1          # T*H*W != N
    assert call(eps=-1.0) == 1
    assert call(theta=0.0) == 1
    bad = _desc(D=64)
    assert call(d=ctypes.byref(bad)) == 2               # head_dim != 96
    assert call(d=ctypes.byref(_desc(D=128))) == 2     # the prologue is defined for 96 channels
    odd = h3a.QkvDesc(1, 8064, 56, 96, 8064 * 56 * 96, 56 * 96 + 4, 96)
    assert call(d=ctypes.byref(odd)) == 1               # stride not a multiple of 8 elements
    assert lib.h3a_qk_norm_rope(GOOD, GOOD, None, GOOD, GOOD, grid, 1e4, 1e-6, GOOD, GOOD, None) == 1


@NO_GPU
def test_route_validation():
    lib = h3a.load()
    d = _desc(N=8064)
    kk = ctypes.c_int64()
    ws = 2 * ((56 * 63 * 96 * 4 + 255) // 256 * 256)

    def call(s=0.75, block=128, q=GOOD, idx=GOOD, w=GOOD, wsb=ws, desc=None):
        return lib.h3a_route(q, GOOD, ctypes.byref(desc or d), s, block, idx, ctypes.byref(kk), w, wsb, None)

    assert call(s=1.0) == 1
    assert call(s=-0.5) == 1
    assert call(block=64) == 2
    assert call(q=None) == 1
    assert call(idx=P(0x10002)) == 1
    assert call(w=None) == 5
    assert call(wsb=ws - 1) == 5
    assert call(w=MISALIGNED) == 5
    # the score kernel keeps a CTA's 8 query-block rows of fp32 scores against
    # every key block in shared memory: 6,048 key blocks at head_dim 96 and
    # 6,016 at 128 (200 KB); past that the call is refused before any launch
    for D, most in ((96, 6048), (128, 6016)):
        assert call(desc=_desc(N=most * 128, heads=1, D=D), wsb=0) == 5      # shape accepted, workspace short
        assert call(desc=_desc(N=most * 128 + 1, heads=1, D=D), wsb=0) == 2
    assert call(desc=_desc(B=65536, N=128, heads=1)) == 2                  # B * heads beyond the grid's y range


@NO_GPU
def test_fused_prologue_and_pooled_route_validation():
    lib = h3a.load()
    d = _desc(N=8064)
    grid = h3a.Grid(8, 24, 42)
    ws = 2 * ((56 * 63 * 96 * 4 + 255) // 256 * 256)
    kk = ctypes.c_int64()

    def pro(q=GOOD, gq=GOOD, grid=grid, eps=1e-6, w=GOOD, wsb=ws, desc=None):
        return lib.h3a_qk_norm_rope_pool(q, GOOD, ctypes.byref(desc or d), gq, GOOD, grid, 1e4, eps, GOOD, GOOD,
                                         w, wsb, None)

    assert pro(q=None) == 1
    assert pro(q=MISALIGNED) == 1
    assert pro(gq=None) == 1
    assert pro(grid=h3a.Grid(8, 24, 41)) == 1          # T*H*W != N
    assert pro(eps=-1.0) == 1
    assert pro(desc=_desc(D=64)) == 2                   # head_dim != 96
    assert pro(w=None) == 5
    assert pro(wsb=ws - 1) == 5
    assert pro(w=MISALIGNED) == 5

    def rp(s=0.75, block=128, idx=GOOD, w=GOOD, wsb=ws, desc=None):
        return lib.h3a_route_pooled(ctypes.byref(desc or d), s, block, idx, ctypes.byref(kk), w, wsb, None)

    assert rp(s=1.0) == 1
    assert rp(s=-0.1) == 1
    assert rp(block=64) == 2
    assert rp(idx=None) == 1
    assert rp(idx=P(0x10002)) == 1
    assert rp(w=None) == 5
    assert rp(wsb=ws - 1) == 5
    assert rp(desc=_desc(D=128)) == 2


@NO_GPU
def test_attention_validation():
    lib = h3a.load()
    d = _desc(N=8064)

    def call(blocks=None, kb=0, block=128, scale=0.0, o=GOOD, desc=None):
        return lib.h3a_attention(GOOD, GOOD, GOOD, ctypes.byref(desc or d), blocks, kb, block, scale, o, None)

    assert call(block=64) == 2
    assert call(o=None) == 1
    assert call(o=MISALIGNED) == 1
    assert call(blocks=GOOD, kb=0) == 1               # sparse mode needs 1 <= k <= nblk
    assert call(blocks=GOOD, kb=64) == 1              # nblk = 63
    assert call(scale=-1.0) == 1
    assert call(scale=float("inf")) == 1
    assert call(desc=_desc(D=64)) == 2
    wide = _desc(N=8064, heads=42, D=128)                # head_dim 128 passes the shape check
    assert call(desc=wide, o=None) == 1
    assert call(desc=wide, block=64) == 2


@NO_GPU
def test_dit_ops_validation():
    lib = h3a.load()

    def ad(x=GOOD, f=GOOD, gate=GOOD, h=GOOD, y=GOOD, B=1, R=4, C=5376, eps=1e-6):
        return lib.h3a_residual_adaln(x, f, gate, GOOD, GOOD, B, R, C, eps, h, y, None)

    assert ad(C=12) == 1                    # not a multiple of 8
    assert ad(C=0) == 1
    assert ad(C=14336 + 8) == 2             # wider than a CTA's registers hold
    assert ad(x=None) == 1
    assert ad(gate=None) == 1               # a residual needs its gate
    assert ad(h=None) == 1                  # ... and an h output
    assert ad(y=MISALIGNED) == 1
    assert ad(eps=-1.0) == 1
    assert ad(B=0) == 1
    assert lib.h3a_swiglu(GOOD, 4, 12, GOOD, None) == 1
    assert lib.h3a_swiglu(None, 4, 16, GOOD, None) == 1
    assert lib.h3a_swiglu(GOOD, 4, 16, MISALIGNED, None) == 1
    assert lib.h3a_swiglu(GOOD, -1, 16, GOOD, None) == 1

    def rd(cur=GOOD, n=4096, thr=0.04, w=GOOD, wsb=32768, rel=GOOD, reuse=GOOD):
        return lib.h3a_residual_diff(cur, GOOD, n, thr, w, wsb, rel, reuse, None)

    assert rd(n=12) == 1
    assert rd(n=0) == 1
    assert rd(cur=None) == 1
    assert rd(rel=P(0x10004)) == 1          # fp64 output must be 8-byte aligned
    assert rd(thr=-1.0) == 1
    assert rd(thr=float("nan")) == 1
    assert rd(w=None) == 5
    assert rd(wsb=32767) == 5


def test_step_schedule_follows_the_page():
    """The router works from the 10th denoising step on (tests/golden/page_facts.txt):
    steps 1..9 dense, 10 onward at the given sparsity; bad arguments give -1."""
    lib = h3a.load()
    facts = open(os.path.join(ROOT, "tests", "golden", "page_facts.txt")).read().split()
    first = int(facts[facts.index("subblock_first_sparse_step") + 1])
    assert first == h3a.FIRST_SPARSE_STEP == 10
    for step in range(1, first):
        assert lib.h3a_step_sparsity(step, first, 0.75) == 0.0
    for step in (first, first + 1, 50):
        assert lib.h3a_step_sparsity(step, first, 0.8) == 0.8
    assert lib.h3a_step_sparsity(0, first, 0.75) == -1.0
    assert lib.h3a_step_sparsity(5, 0, 0.75) == -1.0
    assert lib.h3a_step_sparsity(12, first, 1.0) == -1.0
    assert h3a.step_sparsity(9) == 0.0 and h3a.step_sparsity(10) == 0.75


def test_python_binding_refuses_cpu_tensors():
    q = torch.zeros(1, 128, 2, 96, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        h3a.attention(q, q, q)
    with pytest.raises(ValueError, match="CUDA"):
        h3a.route(q, q, 0.5)
