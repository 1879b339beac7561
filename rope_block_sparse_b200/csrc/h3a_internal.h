// Launchers shared between the C-ABI front end (h3a_api.cu) and the kernel
// translation units.  Not part of the public interface.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace h3a {

constexpr int kHeadDim = 96;       // every call
constexpr int kHeadDimWide = 128;  // the router and attention also take it (SubBlock's head size)
constexpr int kBlock = 128;

// Status word bits set by kernels (read back by h3a_last_device_error).
constexpr int kDevTimeout = 1;

struct Shape {
    int B, N, heads;
    int d;               // head_dim: 96, or 128 (router and attention)
    int64_t sb, sn, sh;  // element strides; head_dim contiguous
};

// QK-RMSNorm + 3D RoPE (prologue.cu).
cudaError_t launch_qk_norm_rope(const void* q, const void* k, void* q_out, void* k_out, const float* gamma_q,
                                const float* gamma_k, const Shape& s, int T, int H, int W, double theta,
                                float eps, cudaStream_t st);

// Prologue whose RMSNorm spans all heads of a token (gains [heads * 96]).
cudaError_t launch_qk_fullnorm_rope(const void* q, const void* k, void* q_out, void* k_out, const float* gamma_q,
                                    const float* gamma_k, const Shape& s, int H, int W, double theta, float eps,
                                    cudaStream_t st);

// Prologue that also writes the fp32 means of its rounded outputs over
// 128-token blocks into pool_q / pool_k (the router's layouts, below)
// (prologue.cu).  Q and K are read through tensor maps made by
// make_head_slice_tensor_map; a bounded wait that expires sets `status`.
cudaError_t launch_qk_norm_rope_pool(const CUtensorMap& tq, const CUtensorMap& tk, void* q_out, void* k_out,
                                     const float* gamma_q, const float* gamma_k, const Shape& s, int H, int W,
                                     double theta, float eps, float* pool_q, float* pool_k, int* status,
                                     uint64_t timeout_ns, cudaStream_t st);
// Heads per slice of the tensor map the prologue with pooling reads.
constexpr int kPrologueSliceHeads = 28;

// The router's fp32 block means: Q's as [B, heads, nblk, d]; K's channel-major,
// [B, heads, d, pooled_k_stride(nblk)] (one 16-byte-aligned row of key blocks
// per channel, so that the score kernel reads consecutive key blocks).
__host__ __device__ inline int pooled_k_stride(int nblk) { return (nblk + 3) & ~3; }

// Router (router.cu): block means of q and k into pooled_q / pooled_k (the
// layouts above), then scores and top-k into idx.
cudaError_t launch_route(const void* q, const void* k, const Shape& s, int nblk, int kk, float* pooled_q,
                         float* pooled_k, int32_t* idx, cudaStream_t st);
// Scores and top-k only, from block means already in pooled_q / pooled_k.
cudaError_t launch_route_scores(const float* pooled_q, const float* pooled_k, const Shape& s, int nblk, int kk,
                                int32_t* idx, cudaStream_t st);
// Largest nblk the score/top-k kernel supports (shared-memory bound).
int route_max_blocks(int d);

// Attention (attention.cu).  blocks == nullptr: dense.
cudaError_t launch_attention(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* o,
                             const Shape& s, const int32_t* blocks, int k_blocks, float scale, int* status,
                             uint64_t timeout_ns, cudaStream_t st);

// Gated residual + AdaLN update and SwiGLU (dit_ops.cu).
cudaError_t launch_residual_adaln(const void* x, const void* f, const float* gate, const float* shift,
                                  const float* scale, int B, int64_t rows, int width, float eps, void* h_out,
                                  void* y_out, cudaStream_t st);
int residual_adaln_max_width();
cudaError_t launch_swiglu(const void* in, int64_t rows, int ffn_width, void* out, cudaStream_t st);
// Cache-DiT residual difference (dit_ops.cu): rel = sum|cur - prev| / sum|prev|.
size_t residual_diff_workspace_bytes();
cudaError_t launch_residual_diff(const void* cur, const void* prev, int64_t n, double threshold, void* workspace,
                                 double* rel_out, int32_t* reuse_out, cudaStream_t st);

// Self-checks (selftest.cu).
cudaError_t launch_selftest_wait(uint64_t limit_ns, int* status, cudaStream_t st);
cudaError_t launch_selftest_exp2(const float* x, float* y, int n, cudaStream_t st);
cudaError_t launch_selftest_mma(const CUtensorMap& ta, const CUtensorMap& tb, float* s_out, float* r_out,
                                int* status, uint64_t timeout_ns, cudaStream_t st);

// Tensor map over a [B, N, heads, 96] bf16 tensor with a {32, 1, 128, 1} box,
// 64-byte swizzle (h3a_api.cu).
cudaError_t make_qkv_tensor_map(CUtensorMap* map, const void* base, const Shape& s);
// Tensor map over the same tensor with a {96, kPrologueSliceHeads, 1, 1} box:
// one token's slice of consecutive heads, no swizzle, heads past the tensor
// read as zero (h3a_api.cu).
cudaError_t make_head_slice_tensor_map(CUtensorMap* map, const void* base, const Shape& s);

}  // namespace h3a
