"""ctypes front end of the fp64 CPU oracle (``oracle/oracle.cpp``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py``.  The product package
never imports it, and it imports nothing from the product package.  Inputs
are plain numpy arrays (bf16 tensors as their uint16 bit patterns).

Each wrapper states what it computes and the passage it follows; the C source
carries the same citations.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so with g++ (IEEE fp64, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-pthread", "-shared", "-fPIC",
                               "-fno-fast-math", _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.oracle_abi_version.restype = i32
        lib.oracle_threads.argtypes = [i32]
        lib.oracle_threads.restype = i32
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_double.restype = f64
        lib.oracle_rmsnorm.argtypes = [P, i32, P, f64, P]
        lib.oracle_rope3d.argtypes = [P, i32, P, f64]
        lib.oracle_token_position.argtypes = [i64, i32, i32, i32, P]
        lib.oracle_qk_norm_rope.argtypes = [P, i32, i64, i32, i32, P, i32, i32, i32, f64, f64, P, i32]
        lib.oracle_qk_norm_rope.restype = i32
        lib.oracle_qk_norm_rope_tokens.argtypes = [P, i32, i64, i32, i32, P, i32, i32, i32, f64, f64, P, i64, P,
                                                   i32]
        lib.oracle_qk_norm_rope_tokens.restype = i32
        lib.oracle_round_bf16.argtypes = [P, i64, P]
        lib.oracle_qk_norm_rope_bf16.argtypes = [P, i32, i64, i32, i32, P, i32, i32, i32, f64, f64, P, i32]
        lib.oracle_qk_norm_rope_bf16.restype = i32
        lib.oracle_num_blocks.argtypes = [i64, i32]
        lib.oracle_num_blocks.restype = i64
        lib.oracle_k_blocks.argtypes = [i64, f64]
        lib.oracle_k_blocks.restype = i64
        lib.oracle_pool.argtypes = [P, i32, i64, i32, i32, i32, P, i32]
        lib.oracle_pool.restype = i32
        lib.oracle_block_scores.argtypes = [P, P, i64, i64, i32, P, i32]
        lib.oracle_block_scores.restype = i32
        lib.oracle_topk.argtypes = [P, i64, i64, i64, P, i32]
        lib.oracle_topk.restype = i32
        lib.oracle_route.argtypes = [P, P, i32, i64, i32, i32, f64, i32, P, P, i32]
        lib.oracle_route.restype = i64
        lib.oracle_attention_rows.argtypes = [P, P, P, i32, i64, i32, i32, P, i64, i32, f64, P, i64, P, i32]
        lib.oracle_attention_rows.restype = i32
        lib.oracle_residual_adaln.argtypes = [P, P, P, P, P, i32, i64, i32, f64, P, P, i32]
        lib.oracle_residual_adaln.restype = i32
        lib.oracle_swiglu.argtypes = [P, i64, i32, P, i32]
        lib.oracle_swiglu.restype = i32
        lib.oracle_residual_diff.argtypes = [P, P, i64]
        lib.oracle_residual_diff.restype = f64
        lib.oracle_qk_fullnorm_rope_bf16.argtypes = [P, i32, i64, i32, i32, P, i32, i32, i32, f64, f64, P, i32]
        lib.oracle_qk_fullnorm_rope_bf16.restype = i32
        assert lib.oracle_abi_version() == 1
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _bits(x) -> np.ndarray:
    """bf16 data as a C-contiguous uint16 array (accepts uint16 arrays or bf16 torch tensors)."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch  # plumbing only: view the bf16 bits

    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def threads(n: int = 0) -> int:
    """Threads the oracle uses for n (0 = all hardware threads)."""
    return _load().oracle_threads(n)


def bf16_to_double(bits: int) -> float:
    return _load().oracle_bf16_to_double(bits)


def rmsnorm(x: np.ndarray, gamma: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """RMSNorm of one head vector: x / sqrt(mean(x^2) + eps) * gamma."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    g = np.ascontiguousarray(gamma, dtype=np.float64)
    y = np.empty_like(x)
    _load().oracle_rmsnorm(_ptr(x), x.size, _ptr(g), eps, _ptr(y))
    return y


def rope3d(y: np.ndarray, pos, theta: float = 10000.0) -> np.ndarray:
    """3D RoPE of one head vector at grid position pos = (t, h, w); returns a copy."""
    out = np.array(y, dtype=np.float64, copy=True)
    p = np.ascontiguousarray(pos, dtype=np.int32)
    _load().oracle_rope3d(_ptr(out), out.size, _ptr(p), theta)
    return out


def token_position(n: int, grid) -> tuple:
    p = np.zeros(3, dtype=np.int32)
    _load().oracle_token_position(n, grid[0], grid[1], grid[2], _ptr(p))
    return tuple(int(v) for v in p)


def qk_norm_rope(x, gamma: np.ndarray, grid, theta: float = 10000.0, eps: float = 1e-6,
                 nthreads: int = 0) -> np.ndarray:
    """Fused RMSNorm + 3D RoPE of a [B, N, heads, d] bf16 tensor, fp64 result."""
    xb = _bits(x)
    B, N, heads, d = xb.shape
    g = np.ascontiguousarray(gamma, dtype=np.float32)
    out = np.empty(xb.shape, dtype=np.float64)
    rc = _load().oracle_qk_norm_rope(_ptr(xb), B, N, heads, d, _ptr(g), grid[0], grid[1], grid[2],
                                     theta, eps, _ptr(out), nthreads)
    if rc != 0:
        raise ValueError("oracle_qk_norm_rope: bad sizes")
    return out


def qk_norm_rope_tokens(x, gamma: np.ndarray, grid, tokens, theta: float = 10000.0, eps: float = 1e-6,
                        nthreads: int = 0) -> np.ndarray:
    """The fused prologue at flattened tokens tok = b*N + n only -> fp64 [len(tokens), heads, d]."""
    xb = _bits(x)
    B, N, heads, d = xb.shape
    g = np.ascontiguousarray(gamma, dtype=np.float32)
    tok = np.ascontiguousarray(tokens, dtype=np.int64)
    out = np.empty((tok.size, heads, d), dtype=np.float64)
    rc = _load().oracle_qk_norm_rope_tokens(_ptr(xb), B, N, heads, d, _ptr(g), grid[0], grid[1], grid[2], theta,
                                            eps, _ptr(tok), tok.size, _ptr(out), nthreads)
    if rc != 0:
        raise ValueError("oracle_qk_norm_rope_tokens: bad sizes")
    return out


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (nearest-even, straight from fp64); returns uint16 bit patterns."""
    xa = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(xa.shape, dtype=np.uint16)
    _load().oracle_round_bf16(_ptr(xa), xa.size, _ptr(out))
    return out


def qk_norm_rope_bf16(x, gamma: np.ndarray, grid, theta: float = 10000.0, eps: float = 1e-6,
                      nthreads: int = 0) -> np.ndarray:
    """The fused prologue with its one rounding to bf16 applied -> uint16 bits, layout of x."""
    xb = _bits(x)
    B, N, heads, d = xb.shape
    g = np.ascontiguousarray(gamma, dtype=np.float32)
    out = np.empty(xb.shape, dtype=np.uint16)
    rc = _load().oracle_qk_norm_rope_bf16(_ptr(xb), B, N, heads, d, _ptr(g), grid[0], grid[1], grid[2], theta,
                                          eps, _ptr(out), nthreads)
    if rc != 0:
        raise ValueError("oracle_qk_norm_rope_bf16: bad sizes")
    return out


def num_blocks(N: int, block: int = 128) -> int:
    return _load().oracle_num_blocks(N, block)


def k_blocks(nkv: int, sparsity: float) -> int:
    return _load().oracle_k_blocks(nkv, sparsity)


def pool(x, block: int = 128, nthreads: int = 0) -> np.ndarray:
    """Block means of a [B, N, heads, d] bf16 tensor -> fp32 [B, heads, nblk, d]."""
    xb = _bits(x)
    B, N, heads, d = xb.shape
    nblk = num_blocks(N, block)
    out = np.empty((B, heads, nblk, d), dtype=np.float32)
    rc = _load().oracle_pool(_ptr(xb), B, N, heads, d, block, _ptr(out), nthreads)
    if rc != 0:
        raise ValueError("oracle_pool: bad sizes")
    return out


def block_scores(qp: np.ndarray, kp: np.ndarray, nthreads: int = 0) -> np.ndarray:
    """fp32 block scores (qbar . kbar) / sqrt(d) for pooled [B, heads, nblk, d] inputs."""
    qp = np.ascontiguousarray(qp, dtype=np.float32)
    kp = np.ascontiguousarray(kp, dtype=np.float32)
    B, heads, nblk, d = qp.shape
    out = np.empty((B, heads, nblk, nblk), dtype=np.float32)
    _load().oracle_block_scores(_ptr(qp), _ptr(kp), B * heads, nblk, d, _ptr(out), nthreads)
    return out


def topk(scores: np.ndarray, k: int, nthreads: int = 0) -> np.ndarray:
    """Per row: the k highest scores (ties to the lower index), indices ascending."""
    s = np.ascontiguousarray(scores, dtype=np.float32)
    rows = int(np.prod(s.shape[:-1]))
    out = np.empty(s.shape[:-1] + (k,), dtype=np.int32)
    rc = _load().oracle_topk(_ptr(s), rows, s.shape[-1], k, _ptr(out), nthreads)
    if rc != 0:
        raise ValueError("oracle_topk: bad k")
    return out


def route(q, k, sparsity: float, block: int = 128, nthreads: int = 0):
    """The blockwise router: returns (idx int32 [B, heads, nblk, k], scores fp32 [B, heads, nblk, nblk])."""
    qb, kb = _bits(q), _bits(k)
    B, N, heads, d = qb.shape
    nblk = num_blocks(N, block)
    kk = k_blocks(nblk, sparsity)
    idx = np.empty((B, heads, nblk, kk), dtype=np.int32)
    sc = np.empty((B, heads, nblk, nblk), dtype=np.float32)
    got = _load().oracle_route(_ptr(qb), _ptr(kb), B, N, heads, d, sparsity, block, _ptr(idx), _ptr(sc),
                               nthreads)
    if got != kk:
        raise ValueError("oracle_route: bad arguments")
    return idx, sc


def attention_rows(q, k, v, rows, block_idx: np.ndarray | None = None, block: int = 128,
                   scale: float | None = None, nthreads: int = 0) -> np.ndarray:
    """fp64 attention output of the given rows r = (b*heads + h)*N + n -> [len(rows), d]."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, N, heads, d = qb.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    r = np.ascontiguousarray(rows, dtype=np.int64)
    out = np.empty((r.size, d), dtype=np.float64)
    if block_idx is None:
        bp, kbl = None, 0
    else:
        bi = np.ascontiguousarray(block_idx, dtype=np.int32)
        bp, kbl = _ptr(bi), bi.shape[-1]
    rc = _load().oracle_attention_rows(_ptr(qb), _ptr(kb), _ptr(vb), B, N, heads, d, bp, kbl, block, scale,
                                       _ptr(r), r.size, _ptr(out), nthreads)
    if rc != 0:
        raise ValueError("oracle_attention_rows: bad sizes")
    return out


def residual_adaln(x, f, gate: np.ndarray, shift: np.ndarray, scale: np.ndarray, eps: float = 1e-6,
                   nthreads: int = 0):
    """Gated residual + AdaLN update of bf16 [B, R, C] rows (f None: the AdaLN update alone).

    gate, shift, scale: fp32 [B, C].  Returns (h bf16 bits [B, R, C], y fp64 [B, R, C])."""
    xb = _bits(x)
    B, R, C = xb.shape
    fb = None if f is None else _bits(f)
    if fb is not None and fb.shape != xb.shape:
        raise ValueError("x and f must have the same shape")
    g = np.ascontiguousarray(gate if gate is not None else np.zeros((B, C)), dtype=np.float32)
    sh = np.ascontiguousarray(shift, dtype=np.float32)
    sc = np.ascontiguousarray(scale, dtype=np.float32)
    for a in (g, sh, sc):
        if a.shape != (B, C):
            raise ValueError("gate, shift, scale must be [B, C]")
    h = np.empty(xb.shape, dtype=np.uint16)
    y = np.empty(xb.shape, dtype=np.float64)
    rc = _load().oracle_residual_adaln(_ptr(xb), None if fb is None else _ptr(fb), _ptr(g), _ptr(sh), _ptr(sc),
                                       B, R, C, eps, _ptr(h), _ptr(y), nthreads)
    if rc != 0:
        raise ValueError("oracle_residual_adaln: bad sizes")
    return h, y


def swiglu(x, nthreads: int = 0) -> np.ndarray:
    """silu(a) * b for bf16 [R, 2F] rows with halves a | b -> fp64 [R, F]."""
    xb = _bits(x)
    R, F2 = xb.shape
    if F2 % 2:
        raise ValueError("last dimension must be even (a | b halves)")
    out = np.empty((R, F2 // 2), dtype=np.float64)
    rc = _load().oracle_swiglu(_ptr(xb), R, F2 // 2, _ptr(out), nthreads)
    if rc != 0:
        raise ValueError("oracle_swiglu: bad sizes")
    return out


def residual_diff(cur, prev) -> float:
    """Relative L1 difference sum|cur - prev| / sum|prev| of two bf16 tensors (fp64)."""
    a, b = _bits(cur).reshape(-1), _bits(prev).reshape(-1)
    if a.size != b.size:
        raise ValueError("cur and prev must have the same number of elements")
    return float(_load().oracle_residual_diff(_ptr(np.ascontiguousarray(a)), _ptr(np.ascontiguousarray(b)), a.size))


def qk_fullnorm_rope_bf16(x, gamma: np.ndarray, grid, theta: float = 10000.0, eps: float = 1e-6,
                          nthreads: int = 0) -> np.ndarray:
    """The prologue with the RMSNorm over the token's whole hidden state (all heads;
    gamma fp32 [heads * d]), then per-head 3D RoPE, rounded to bf16 -> uint16 bits."""
    xb = _bits(x)
    B, N, heads, d = xb.shape
    g = np.ascontiguousarray(gamma, dtype=np.float32).reshape(-1)
    if g.size != heads * d:
        raise ValueError("gamma must have heads * d entries")
    out = np.empty(xb.shape, dtype=np.uint16)
    rc = _load().oracle_qk_fullnorm_rope_bf16(_ptr(xb), B, N, heads, d, _ptr(g), grid[0], grid[1], grid[2], theta,
                                              eps, _ptr(out), nthreads)
    if rc != 0:
        raise ValueError("oracle_qk_fullnorm_rope_bf16: bad sizes")
    return out
