"""Thin ctypes binding of libh3a (include/h3a.h) over torch tensors.

Argument marshalling only: shapes, strides and pointers are read from the
tensors and passed to the C ABI, which validates them and launches the CUDA
kernels on torch's current stream.  Every step of the attention core runs in
libh3a; if the library is missing or the tensors are not on a CUDA device the
calls raise -- there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libh3a.so")
HEAD_DIM = 96
BLOCK = 128

H3A_OK = 0
STATUS_NAMES = {0: "H3A_OK", 1: "H3A_ERR_INVALID_ARG", 2: "H3A_ERR_UNSUPPORTED", 3: "H3A_ERR_CUDA",
                4: "H3A_ERR_TIMEOUT", 5: "H3A_ERR_WORKSPACE"}

# Every function the header declares; checked by the ABI test.
EXPORTS = ("h3a_qk_norm_rope", "h3a_route_k", "h3a_route_workspace_size", "h3a_route", "h3a_attention",
           "h3a_status_string", "h3a_last_cuda_error_string", "h3a_last_device_error",
           "h3a_selftest_wait_timeout", "h3a_selftest_mma", "h3a_selftest_exp2", "h3a_route_noalloc",
           "h3a_qk_norm_rope_pool", "h3a_route_pooled", "h3a_residual_adaln", "h3a_swiglu",
           "h3a_residual_diff", "h3a_step_sparsity", "h3a_qk_fullnorm_rope")
ROUTE_NOALLOC_MAX_BYTES = 64 << 20  # H3A_ROUTE_NOALLOC_MAX_BYTES
RESIDUAL_DIFF_WORKSPACE_BYTES = 32768  # H3A_RESIDUAL_DIFF_WORKSPACE_BYTES


class H3AError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str = ""):
        self.status = status
        msg = f"{fn} failed: {STATUS_NAMES.get(status, status)}"
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


class Grid(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("W", ctypes.c_int32)]


class QkvDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("N", ctypes.c_int32), ("heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("stride_b", ctypes.c_int64), ("stride_n", ctypes.c_int64),
                ("stride_h", ctypes.c_int64)]


_lib = None


def load() -> ctypes.CDLL:
    """Load libh3a.so from the package directory (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libh3a.so not found at {LIB_PATH}; build it with "
                           "`python -m rope_block_sparse_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, i32, i64, f32, f64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_double
    st = ctypes.c_int
    lib.h3a_qk_norm_rope.argtypes = [P, P, ctypes.POINTER(QkvDesc), P, P, Grid, f64, f32, P, P, P]
    lib.h3a_qk_norm_rope.restype = st
    lib.h3a_route_k.argtypes = [i64, f64]
    lib.h3a_route_k.restype = i64
    lib.h3a_route_workspace_size.argtypes = [ctypes.POINTER(QkvDesc), i32, ctypes.POINTER(ctypes.c_size_t)]
    lib.h3a_route_workspace_size.restype = st
    lib.h3a_route.argtypes = [P, P, ctypes.POINTER(QkvDesc), f64, i32, P, ctypes.POINTER(ctypes.c_int64), P,
                              ctypes.c_size_t, P]
    lib.h3a_route.restype = st
    lib.h3a_attention.argtypes = [P, P, P, ctypes.POINTER(QkvDesc), P, i32, i32, f32, P, P]
    lib.h3a_attention.restype = st
    lib.h3a_status_string.argtypes = [st]
    lib.h3a_status_string.restype = ctypes.c_char_p
    lib.h3a_last_cuda_error_string.argtypes = []
    lib.h3a_last_cuda_error_string.restype = ctypes.c_char_p
    lib.h3a_last_device_error.argtypes = [P]
    lib.h3a_last_device_error.restype = st
    lib.h3a_selftest_wait_timeout.argtypes = [ctypes.c_uint32, P]
    lib.h3a_selftest_wait_timeout.restype = st
    lib.h3a_selftest_mma.argtypes = [P, P, P, P, P]
    lib.h3a_selftest_mma.restype = st
    lib.h3a_selftest_exp2.argtypes = [P, P, i32, P]
    lib.h3a_selftest_exp2.restype = st
    lib.h3a_route_noalloc.argtypes = [P, P, ctypes.POINTER(QkvDesc), f64, i32, P, ctypes.POINTER(ctypes.c_int64), P]
    lib.h3a_route_noalloc.restype = st
    lib.h3a_qk_norm_rope_pool.argtypes = [P, P, ctypes.POINTER(QkvDesc), P, P, Grid, f64, f32, P, P, P,
                                          ctypes.c_size_t, P]
    lib.h3a_qk_norm_rope_pool.restype = st
    lib.h3a_route_pooled.argtypes = [ctypes.POINTER(QkvDesc), f64, i32, P, ctypes.POINTER(ctypes.c_int64), P,
                                     ctypes.c_size_t, P]
    lib.h3a_route_pooled.restype = st
    lib.h3a_residual_adaln.argtypes = [P, P, P, P, P, i32, i64, i32, f32, P, P, P]
    lib.h3a_residual_adaln.restype = st
    lib.h3a_swiglu.argtypes = [P, i64, i32, P, P]
    lib.h3a_swiglu.restype = st
    lib.h3a_residual_diff.argtypes = [P, P, i64, f64, P, ctypes.c_size_t, P, P, P]
    lib.h3a_residual_diff.restype = st
    lib.h3a_step_sparsity.argtypes = [i32, i32, f64]
    lib.h3a_step_sparsity.restype = f64
    lib.h3a_qk_fullnorm_rope.argtypes = [P, P, ctypes.POINTER(QkvDesc), P, P, Grid, f64, f32, P, P, P]
    lib.h3a_qk_fullnorm_rope.restype = st
    _lib = lib
    return lib


def _check(fn: str, status: int):
    if status != H3A_OK:
        detail = load().h3a_last_cuda_error_string().decode() if status == 3 else ""
        raise H3AError(fn, status, detail)


def _stream_handle():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t: torch.Tensor | None):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def desc_of(t: torch.Tensor) -> QkvDesc:
    """Descriptor of a [B, N, heads, head_dim] tensor whose last dimension is contiguous."""
    if t.dim() != 4:
        raise ValueError(f"expected a [B, N, heads, head_dim] tensor, got shape {tuple(t.shape)}")
    if t.stride(3) != 1:
        raise ValueError("head_dim must be the contiguous dimension")
    B, N, H, D = t.shape
    return QkvDesc(B, N, H, D, t.stride(0), t.stride(1), t.stride(2))


def _check_qkv(*ts: torch.Tensor):
    ref = ts[0]
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must be on a CUDA device (libh3a has no CPU path)")
        if t.dtype != torch.bfloat16:
            raise ValueError(f"tensors must be bfloat16, got {t.dtype}")
        if t.shape != ref.shape or t.stride() != ref.stride():
            raise ValueError("q, k, v (and outputs) must share shape and strides")


def _prologue_outputs(q, k, gamma_q, gamma_k, inplace, out):
    _check_qkv(q, k)
    for g in (gamma_q, gamma_k):
        if not g.is_cuda or g.dtype != torch.float32 or g.numel() != HEAD_DIM or not g.is_contiguous():
            raise ValueError("gammas must be contiguous fp32 [96] CUDA tensors")
    if inplace:
        return q, k
    if out is not None:
        qo, ko = out
        _check_qkv(q, qo, ko)
        return qo, ko
    return torch.empty_like(q), torch.empty_like(k)


def qk_norm_rope(q: torch.Tensor, k: torch.Tensor, gamma_q: torch.Tensor, gamma_k: torch.Tensor, grid,
                 theta: float = 10000.0, eps: float = 1e-6, inplace: bool = False, out=None):
    """Fused QK-RMSNorm + 3D RoPE over [B, N, heads, 96] bf16 q and k; returns (q_out, k_out).

    inplace=True overwrites q and k; out=(q_out, k_out) writes into given tensors."""
    lib = load()
    qo, ko = _prologue_outputs(q, k, gamma_q, gamma_k, inplace, out)
    d = desc_of(q)
    _check("h3a_qk_norm_rope", lib.h3a_qk_norm_rope(_ptr(q), _ptr(k), ctypes.byref(d), _ptr(gamma_q),
                                                    _ptr(gamma_k), Grid(*grid), float(theta), float(eps),
                                                    _ptr(qo), _ptr(ko), _stream_handle()))
    return qo, ko


def qk_fullnorm_rope(q: torch.Tensor, k: torch.Tensor, gamma_q: torch.Tensor, gamma_k: torch.Tensor, grid,
                     theta: float = 10000.0, eps: float = 1e-6, inplace: bool = False, out=None):
    """qk_norm_rope with the RMSNorm over each token's whole hidden state (all heads);
    gamma_q, gamma_k: fp32 [heads * 96].  Returns (q_out, k_out)."""
    lib = load()
    _check_qkv(q, k)
    heads = q.shape[2]
    for g in (gamma_q, gamma_k):
        if not g.is_cuda or g.dtype != torch.float32 or g.numel() != heads * HEAD_DIM or not g.is_contiguous():
            raise ValueError("gammas must be contiguous fp32 [heads * 96] CUDA tensors")
    if inplace:
        qo, ko = q, k
    elif out is not None:
        qo, ko = out
        _check_qkv(q, qo, ko)
    else:
        qo, ko = torch.empty_like(q), torch.empty_like(k)
    d = desc_of(q)
    _check("h3a_qk_fullnorm_rope", lib.h3a_qk_fullnorm_rope(_ptr(q), _ptr(k), ctypes.byref(d), _ptr(gamma_q),
                                                            _ptr(gamma_k), Grid(*grid), float(theta), float(eps),
                                                            _ptr(qo), _ptr(ko), _stream_handle()))
    return qo, ko


def _workspace(q: torch.Tensor, workspace: torch.Tensor | None, block: int = BLOCK) -> torch.Tensor:
    need = route_workspace_size(q, block)
    if workspace is None:
        return torch.empty(need, dtype=torch.uint8, device=q.device)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return workspace


def qk_norm_rope_pool(q: torch.Tensor, k: torch.Tensor, gamma_q: torch.Tensor, gamma_k: torch.Tensor, grid,
                      theta: float = 10000.0, eps: float = 1e-6, workspace: torch.Tensor | None = None,
                      inplace: bool = False, out=None):
    """qk_norm_rope that also leaves the router's fp32 block means in `workspace`
    (as route() would compute them); returns (q_out, k_out, workspace) for route_pooled()."""
    lib = load()
    qo, ko = _prologue_outputs(q, k, gamma_q, gamma_k, inplace, out)
    workspace = _workspace(q, workspace)
    d = desc_of(q)
    _check("h3a_qk_norm_rope_pool",
           lib.h3a_qk_norm_rope_pool(_ptr(q), _ptr(k), ctypes.byref(d), _ptr(gamma_q), _ptr(gamma_k), Grid(*grid),
                                     float(theta), float(eps), _ptr(qo), _ptr(ko), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream_handle()))
    return qo, ko, workspace


def route_pooled(q: torch.Tensor, sparsity: float, workspace: torch.Tensor, block: int = BLOCK,
                 out: torch.Tensor | None = None) -> torch.Tensor:
    """Scores + top-k from the block means qk_norm_rope_pool left in `workspace`
    (q only supplies the shape); same result as route() on the prologue outputs."""
    lib = load()
    if not q.is_cuda:
        raise ValueError("tensors must be on a CUDA device (libh3a has no CPU path)")
    B, N, H, _ = q.shape
    nblk = (N + block - 1) // block
    kk = route_k(nblk, sparsity)
    if kk < 0:
        raise ValueError(f"sparsity {sparsity} outside [0, 1)")
    out = _route_out(q, nblk, kk, out)
    k_out = ctypes.c_int64(0)
    d = desc_of(q)
    _check("h3a_route_pooled", lib.h3a_route_pooled(ctypes.byref(d), float(sparsity), block, _ptr(out),
                                                    ctypes.byref(k_out), _ptr(workspace),
                                                    workspace.numel() * workspace.element_size(),
                                                    _stream_handle()))
    return out


def _route_out(q: torch.Tensor, nblk: int, kk: int, out: torch.Tensor | None) -> torch.Tensor:
    B, _, H, _ = q.shape
    if out is None:
        return torch.empty((B, H, nblk, kk), dtype=torch.int32, device=q.device)
    if out.shape != (B, H, nblk, kk) or out.dtype != torch.int32 or not out.is_contiguous():
        raise ValueError("out must be a contiguous int32 [B, heads, nblk, k] tensor")
    return out


FIRST_SPARSE_STEP = 10  # the router works from the 10th denoising step on


def step_sparsity(step: int, sparsity: float = 0.75, first_sparse_step: int = FIRST_SPARSE_STEP) -> float:
    """Sparsity at denoising step `step` (from 1): 0.0 (dense) before first_sparse_step."""
    s = float(load().h3a_step_sparsity(int(step), int(first_sparse_step), float(sparsity)))
    if s < 0:
        raise ValueError(f"bad step schedule: step={step}, first_sparse_step={first_sparse_step}, sparsity={sparsity}")
    return s


def route_k(nkv: int, sparsity: float) -> int:
    return int(load().h3a_route_k(nkv, sparsity))


def route_workspace_size(q: torch.Tensor, block: int = BLOCK) -> int:
    lib = load()
    d = desc_of(q)
    n = ctypes.c_size_t(0)
    _check("h3a_route_workspace_size", lib.h3a_route_workspace_size(ctypes.byref(d), block, ctypes.byref(n)))
    return n.value


def route(q: torch.Tensor, k: torch.Tensor, sparsity: float, block: int = BLOCK,
          workspace: torch.Tensor | None = None, out: torch.Tensor | None = None) -> torch.Tensor:
    """Blockwise KV-block router: int32 [B, heads, nblk, k] ascending block lists."""
    lib = load()
    _check_qkv(q, k)
    B, N, H, _ = q.shape
    nblk = (N + block - 1) // block
    kk = route_k(nblk, sparsity)
    if kk < 0:
        raise ValueError(f"sparsity {sparsity} outside [0, 1)")
    workspace = _workspace(q, workspace, block)
    out = _route_out(q, nblk, kk, out)
    k_out = ctypes.c_int64(0)
    d = desc_of(q)
    _check("h3a_route", lib.h3a_route(_ptr(q), _ptr(k), ctypes.byref(d), float(sparsity), block, _ptr(out),
                                      ctypes.byref(k_out), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                      _stream_handle()))
    return out


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block_idx: torch.Tensor | None = None,
              scale: float = 0.0, block: int = BLOCK, out: torch.Tensor | None = None) -> torch.Tensor:
    """Bidirectional attention, dense (block_idx None) or over routed KV blocks."""
    lib = load()
    if out is None:
        out = torch.empty_like(q)
    _check_qkv(q, k, v, out)
    kb = 0
    if block_idx is not None:
        B, N, H, _ = q.shape
        nblk = (N + block - 1) // block
        if (block_idx.dtype != torch.int32 or not block_idx.is_contiguous() or block_idx.dim() != 4
                or tuple(block_idx.shape[:3]) != (B, H, nblk) or not block_idx.is_cuda):
            raise ValueError("block_idx must be a contiguous int32 CUDA tensor [B, heads, nblk, k]")
        kb = block_idx.shape[3]
    d = desc_of(q)
    _check("h3a_attention", lib.h3a_attention(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(d), _ptr(block_idx), kb,
                                              block, float(scale), _ptr(out), _stream_handle()))
    return out


def residual_adaln(x: torch.Tensor, f: torch.Tensor | None, gate: torch.Tensor | None, shift: torch.Tensor,
                   scale: torch.Tensor, eps: float = 1e-6, out=None):
    """Gated residual + AdaLN update of bf16 [B, rows, C] rows: h = x + gate*f (bf16),
    y = LayerNorm(h) * (1 + scale) + shift.  gate/shift/scale: fp32 [B, C].
    f None: the AdaLN update of x alone.  Returns (h or None, y); out=(h, y) writes in place."""
    lib = load()
    if x.dim() != 3 or not x.is_cuda or x.dtype != torch.bfloat16 or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 [B, rows, C] CUDA tensor")
    B, R, C = x.shape
    for t in ([f] if f is not None else []):
        if t.shape != x.shape or t.dtype != torch.bfloat16 or not t.is_contiguous() or not t.is_cuda:
            raise ValueError("f must match x")
    for name, t in (("shift", shift), ("scale", scale)) + ((("gate", gate),) if f is not None else ()):
        if t is None or t.shape != (B, C) or t.dtype != torch.float32 or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"{name} must be a contiguous fp32 [B, C] CUDA tensor")
    if out is not None:
        h, y = out
    else:
        h = torch.empty_like(x) if f is not None else None
        y = torch.empty_like(x)
    _check("h3a_residual_adaln", lib.h3a_residual_adaln(_ptr(x), _ptr(f), _ptr(gate if f is not None else None),
                                                        _ptr(shift), _ptr(scale), B, R, C, float(eps), _ptr(h),
                                                        _ptr(y), _stream_handle()))
    return h, y


def swiglu(x: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """silu(a) * b for bf16 [rows, 2F] rows laid out [a | b] -> bf16 [rows, F]."""
    lib = load()
    if x.dim() != 2 or not x.is_cuda or x.dtype != torch.bfloat16 or not x.is_contiguous() or x.shape[1] % 2:
        raise ValueError("x must be a contiguous bf16 [rows, 2F] CUDA tensor")
    R, F = x.shape[0], x.shape[1] // 2
    if out is None:
        out = torch.empty((R, F), dtype=torch.bfloat16, device=x.device)
    _check("h3a_swiglu", lib.h3a_swiglu(_ptr(x), R, F, _ptr(out), _stream_handle()))
    return out


def residual_diff(cur: torch.Tensor, prev: torch.Tensor, threshold: float = 0.04,
                  workspace: torch.Tensor | None = None, out=None):
    """Cache-DiT reuse decision: rel = sum|cur - prev| / sum|prev| over two bf16 tensors of
    the same size, reuse = rel < threshold.  Returns device tensors (rel fp64 [1], reuse int32 [1])."""
    lib = load()
    for t in (cur, prev):
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("cur and prev must be contiguous bf16 CUDA tensors")
    if cur.numel() != prev.numel():
        raise ValueError("cur and prev must have the same number of values")
    if workspace is None:
        workspace = torch.empty(RESIDUAL_DIFF_WORKSPACE_BYTES, dtype=torch.uint8, device=cur.device)
    if out is None:
        rel = torch.empty(1, dtype=torch.float64, device=cur.device)
        reuse = torch.empty(1, dtype=torch.int32, device=cur.device)
    else:
        rel, reuse = out
    _check("h3a_residual_diff", lib.h3a_residual_diff(_ptr(cur), _ptr(prev), cur.numel(), float(threshold),
                                                      _ptr(workspace), workspace.numel() * workspace.element_size(),
                                                      _ptr(rel), _ptr(reuse), _stream_handle()))
    return rel, reuse


def last_device_error() -> int:
    """Synchronise the current stream and read/clear the device status word (H3A_OK or H3A_ERR_TIMEOUT)."""
    return int(load().h3a_last_device_error(_stream_handle()))


def selftest_wait_timeout(limit_us: int = 1000) -> int:
    return int(load().h3a_selftest_wait_timeout(limit_us, _stream_handle()))


def selftest_mma(a: torch.Tensor, b: torch.Tensor):
    """Tensor-core self-check: returns (S = A B^T fp32 [128,128], R = bf16(S) B fp32 [128,96])."""
    lib = load()
    for t in (a, b):
        if t.shape != (128, HEAD_DIM) or t.dtype != torch.bfloat16 or not t.is_contiguous() or not t.is_cuda:
            raise ValueError("a, b must be contiguous bf16 [128, 96] CUDA tensors")
    s = torch.empty((128, 128), dtype=torch.float32, device=a.device)
    r = torch.empty((128, HEAD_DIM), dtype=torch.float32, device=a.device)
    _check("h3a_selftest_mma", lib.h3a_selftest_mma(_ptr(a), _ptr(b), _ptr(s), _ptr(r), _stream_handle()))
    return s, r


def selftest_exp2(x: torch.Tensor) -> torch.Tensor:
    """2^x by the softmax's exponential (ex2.approx): fp32 CUDA tensor in and out."""
    lib = load()
    if not x.is_cuda or x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("x must be a contiguous fp32 CUDA tensor")
    y = torch.empty_like(x)
    _check("h3a_selftest_exp2", lib.h3a_selftest_exp2(_ptr(x), _ptr(y), x.numel(), _stream_handle()))
    return y


def attention_core(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, gamma_q: torch.Tensor,
                   gamma_k: torch.Tensor, grid, sparsity: float | None = None, theta: float = 10000.0,
                   eps: float = 1e-6, workspace: torch.Tensor | None = None, step: int | None = None):
    """The whole per-layer core: prologue over Q/K, then dense attention
    (sparsity None) or router + block-sparse attention.  With `step` (denoising
    step, from 1) the sparsity applies only from step 10 on, dense before.
    Returns (o, block_idx or None)."""
    if sparsity is not None and step is not None:
        sparsity = step_sparsity(step, sparsity) or None
    if sparsity is None:
        qn, kn = qk_norm_rope(q, k, gamma_q, gamma_k, grid, theta, eps)
        return attention(qn, kn, v), None
    qn, kn, ws = qk_norm_rope_pool(q, k, gamma_q, gamma_k, grid, theta, eps, workspace=workspace)
    blocks = route_pooled(qn, sparsity, ws)
    return attention(qn, kn, v, blocks), blocks
