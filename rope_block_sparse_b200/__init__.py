"""B200-native (sm_100a) attention core for H3-style video DiTs.

Public API (CUDA tensors, bf16 [B, N, heads, 96]):
    qk_norm_rope(q, k, gamma_q, gamma_k, grid, theta, eps) -> (q', k')
    route(q, k, sparsity) -> int32 [B, heads, nblk, k] KV-block lists
    qk_norm_rope_pool(...) -> (q', k', workspace), then route_pooled(q', sparsity, workspace):
        the prologue with the router's block pooling folded in
    residual_adaln(x, f, gate, shift, scale) -> (h, y), swiglu(x) -> out:
        the other fused DiT operators (gated residual + AdaLN update, SwiGLU)
    residual_diff(cur, prev, threshold) -> (rel, reuse): the Cache-DiT reuse decision
    attention(q, k, v, block_idx=None) -> o
    attention_core(q, k, v, gamma_q, gamma_k, grid, sparsity=None) -> (o, block_idx)

All compute runs in libh3a.so (include/h3a.h); the Python layer only marshals
arguments.  ``synth`` holds the seeded synthetic input generators.
"""
from .h3a import (H3AError, attention, attention_core, last_device_error, load, qk_fullnorm_rope, qk_norm_rope,
                  qk_norm_rope_pool,
                  residual_adaln, residual_diff, route, route_k, route_pooled, route_workspace_size, selftest_exp2,
                  selftest_mma, selftest_wait_timeout, step_sparsity, swiglu)

__all__ = ["H3AError", "attention", "attention_core", "last_device_error", "load", "qk_fullnorm_rope", "qk_norm_rope",
           "qk_norm_rope_pool", "residual_adaln", "residual_diff", "route", "route_k", "route_pooled", "route_workspace_size",
           "selftest_exp2", "selftest_mma", "selftest_wait_timeout", "step_sparsity", "swiglu"]
