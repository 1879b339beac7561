// The other fused DiT operators of the news.cocoloop.cn MiniMax-H3 SGLang
// report (section "Erst drei übereinandergelegte Beschleunigungsebenen",
// fused-operator paragraph: the AdaLN update, the gated residual path and the
// SwiGLU activation are fused like QK-RMSNorm + 3D RoPE, to cut trips through
// device memory, without changing any result).  The page gives no formulas;
// these are the DiT block's:
//
//   residual_adaln_kernel   h = x + gate[b] * f   (rounded once to bf16: the
//                           tensor the block passes on), then the AdaLN update
//                           y = LayerNorm(h) * (1 + scale[b]) + shift[b], with
//                           LayerNorm without affine over the rounded h.  One
//                           pass over HBM: x and f read once, h and y written
//                           once.  f == null gives the AdaLN update alone.
//   swiglu_kernel           out = silu(a) * b for rows [a | b] of width 2F.
//   residual_diff_*         the Cache-DiT reuse decision (same page, next
//                           paragraph: a residual-difference threshold of 0.04
//                           or 0.08 decides reuse between adjacent denoising
//                           steps), read as rel = sum|cur - prev| / sum|prev|.
//
// All are HBM-bound.  residual_adaln: one 224-thread CTA per token row, each
// thread holding up to VPT 16-byte vectors of the row in registers, so the
// mean and the variance (exact two-pass, in fp32) need no second read; the
// two reductions go through warp shuffles and shared memory.  swiglu: a
// grid-stride loop over 16-byte output vectors, two per iteration.
// residual_diff: a grid-stride pass writing one fp64 partial pair per CTA to a
// caller workspace, then one CTA adding them in index order (deterministic).
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>

#include "h3a_internal.h"

namespace h3a {
namespace {

constexpr int kRowThreads = 224;
constexpr int kRowWarps = kRowThreads / 32;

struct AdalnArgs {
    const __nv_bfloat16* x;
    const __nv_bfloat16* f;  // null: no residual
    const float* gate;
    const float* shift;
    const float* scale;
    __nv_bfloat16* h;        // may be null when f is null
    __nv_bfloat16* y;
    int64_t rows;            // rows per batch
    int width;
    float eps;
};

__device__ __forceinline__ void unpack8(uint4 v, float (&o)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        o[2 * i] = __uint_as_float(w[i] << 16);
        o[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void load8f(const float* p, float (&o)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    o[0] = a.x, o[1] = a.y, o[2] = a.z, o[3] = a.w, o[4] = b.x, o[5] = b.y, o[6] = b.z, o[7] = b.w;
}

// Sum over the CTA (every thread receives it).
__device__ __forceinline__ float cta_sum(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[warp] = v;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kRowWarps; ++w) t += red[w];
    __syncthreads();  // red is reused by the next reduction
    return t;
}

template <int VPT>
__global__ void __launch_bounds__(kRowThreads) residual_adaln_kernel(const AdalnArgs a) {
    __shared__ float red[kRowWarps];
    const int64_t row = blockIdx.x;  // over B * rows
    const int b = static_cast<int>(row / a.rows);
    const int nvec = a.width / 8;
    const int64_t base = row * a.width;
    const float* gate = a.gate + static_cast<int64_t>(b) * a.width;
    float h[VPT][8];
    float sum = 0.f;
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
        const int v = threadIdx.x + u * kRowThreads;
        if (v < nvec) {
            float xv[8];
            unpack8(__ldg(reinterpret_cast<const uint4*>(a.x + base) + v), xv);
            if (a.f) {
                float fv[8], gv[8];
                unpack8(__ldg(reinterpret_cast<const uint4*>(a.f + base) + v), fv);
                load8f(gate + 8 * v, gv);
#pragma unroll
                for (int i = 0; i < 8; ++i) xv[i] = fmaf(gv[i], fv[i], xv[i]);
            }
            // round h once to bf16; the statistics use the rounded values
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                w[i] = pack2(xv[2 * i], xv[2 * i + 1]);
                h[u][2 * i] = __uint_as_float(w[i] << 16);
                h[u][2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
                sum += h[u][2 * i] + h[u][2 * i + 1];
            }
            if (a.h) reinterpret_cast<uint4*>(a.h + base)[v] = make_uint4(w[0], w[1], w[2], w[3]);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) h[u][i] = 0.f;
        }
    }
    const float inv_c = 1.0f / static_cast<float>(a.width);
    const float mean = cta_sum(sum, red) * inv_c;
    float sq = 0.f;
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
        if (threadIdx.x + u * kRowThreads < nvec) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float dlt = h[u][i] - mean;
                sq = fmaf(dlt, dlt, sq);
            }
        }
    }
    const float rstd = rsqrtf(cta_sum(sq, red) * inv_c + a.eps);
    const float* shift = a.shift + static_cast<int64_t>(b) * a.width;
    const float* scale = a.scale + static_cast<int64_t>(b) * a.width;
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
        const int v = threadIdx.x + u * kRowThreads;
        if (v < nvec) {
            float sv[8], tv[8];
            load8f(scale + 8 * v, sv);
            load8f(shift + 8 * v, tv);
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float y0 = fmaf((h[u][2 * i] - mean) * rstd, 1.0f + sv[2 * i], tv[2 * i]);
                const float y1 = fmaf((h[u][2 * i + 1] - mean) * rstd, 1.0f + sv[2 * i + 1], tv[2 * i + 1]);
                w[i] = pack2(y0, y1);
            }
            reinterpret_cast<uint4*>(a.y + base)[v] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

struct SwigluArgs {
    const __nv_bfloat16* in;
    __nv_bfloat16* out;
    int64_t vectors;  // rows * F / 8
    int fvec;         // F / 8
};

__device__ __forceinline__ float silu(float v) { return v / (1.0f + expf(-v)); }

__device__ __forceinline__ uint4 swiglu8(uint4 av, uint4 bv) {
    float a8[8], b8[8];
    unpack8(av, a8);
    unpack8(bv, b8);
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = pack2(silu(a8[2 * i]) * b8[2 * i], silu(a8[2 * i + 1]) * b8[2 * i + 1]);
    return make_uint4(w[0], w[1], w[2], w[3]);
}

__global__ void __launch_bounds__(256) swiglu_kernel(const SwigluArgs a) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const uint4* in = reinterpret_cast<const uint4*>(a.in);
    uint4* out = reinterpret_cast<uint4*>(a.out);
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < a.vectors; i += 2 * stride) {
        const int64_t i1 = i + stride;
        const bool two = i1 < a.vectors;
        // output vector i of row r = i / fvec, column block j: a at [2F*r + 8j], b at +F
        const int64_t r0 = i / a.fvec, r1 = i1 / a.fvec;
        const int64_t s0 = 2 * r0 * a.fvec + (i - r0 * a.fvec), s1 = 2 * r1 * a.fvec + (i1 - r1 * a.fvec);
        const uint4 a0 = __ldg(in + s0), b0 = __ldg(in + s0 + a.fvec);
        uint4 a1 = make_uint4(0, 0, 0, 0), b1 = a1;
        if (two) {
            a1 = __ldg(in + s1);
            b1 = __ldg(in + s1 + a.fvec);
        }
        out[i] = swiglu8(a0, b0);
        if (two) out[i1] = swiglu8(a1, b1);
    }
}

// Relative L1 difference, stage 1: CTA c writes (sum|cur - prev|, sum|prev|)
// over its grid-stride share of 16-byte vectors to partial[2c], [2c + 1].
// Each 8-element vector is summed in fp32 (|a - b| and |b| of bf16 values)
// and added to fp64 accumulators; the CTA total goes through fp64 shuffles.
constexpr int kDiffThreads = 256;
constexpr int kDiffMaxCtas = 2048;

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// CTA-wide fp64 sums of (x, y), deterministic; valid in thread 0.
__device__ __forceinline__ void cta_sum2_d(double& x, double& y) {
    __shared__ double red[2][kDiffThreads / 32];
    x = warp_sum_d(x);
    y = warp_sum_d(y);
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
        red[0][warp] = x;
        red[1][warp] = y;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        x = y = 0.0;
        for (int w = 0; w < kDiffThreads / 32; ++w) {
            x += red[0][w];
            y += red[1][w];
        }
    }
}

__global__ void __launch_bounds__(kDiffThreads) residual_diff_partial_kernel(const uint4* cur, const uint4* prev,
                                                                             int64_t nvec, double* partial) {
    double num = 0.0, den = 0.0;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kDiffThreads;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kDiffThreads + threadIdx.x; i < nvec; i += stride) {
        float a[8], b[8];
        unpack8(__ldg(cur + i), a);
        unpack8(__ldg(prev + i), b);
        float n8 = 0.f, d8 = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            n8 += fabsf(a[e] - b[e]);
            d8 += fabsf(b[e]);
        }
        num += static_cast<double>(n8);
        den += static_cast<double>(d8);
    }
    cta_sum2_d(num, den);
    if (threadIdx.x == 0) {
        partial[2 * blockIdx.x] = num;
        partial[2 * blockIdx.x + 1] = den;
    }
}

// Stage 2: one CTA adds the partials in index order and decides reuse.
__global__ void __launch_bounds__(kDiffThreads) residual_diff_final_kernel(const double* partial, int nparts,
                                                                           double threshold, double* rel_out,
                                                                           int32_t* reuse_out) {
    double num = 0.0, den = 0.0;
    for (int p = threadIdx.x; p < nparts; p += kDiffThreads) {
        num += partial[2 * p];
        den += partial[2 * p + 1];
    }
    cta_sum2_d(num, den);
    if (threadIdx.x == 0) {
        const double rel = den == 0.0 ? (num == 0.0 ? 0.0 : INFINITY) : num / den;
        *rel_out = rel;
        if (reuse_out) *reuse_out = rel < threshold ? 1 : 0;
    }
}

template <int VPT>
cudaError_t adaln(const AdalnArgs& a, int64_t total_rows, cudaStream_t st) {
    residual_adaln_kernel<VPT><<<static_cast<unsigned>(total_rows), kRowThreads, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

int residual_adaln_max_width() { return 8 * kRowThreads * 8; }  // 14,336 channels

cudaError_t launch_residual_adaln(const void* x, const void* f, const float* gate, const float* shift,
                                  const float* scale, int B, int64_t rows, int width, float eps, void* h_out,
                                  void* y_out, cudaStream_t st) {
    AdalnArgs a;
    a.x = static_cast<const __nv_bfloat16*>(x);
    a.f = static_cast<const __nv_bfloat16*>(f);
    a.gate = gate;
    a.shift = shift;
    a.scale = scale;
    a.h = static_cast<__nv_bfloat16*>(h_out);
    a.y = static_cast<__nv_bfloat16*>(y_out);
    a.rows = rows;
    a.width = width;
    a.eps = eps;
    const int64_t total = static_cast<int64_t>(B) * rows;
    if (total == 0) return cudaSuccess;
    const int vpt = (width / 8 + kRowThreads - 1) / kRowThreads;
    switch (vpt) {
        case 1: return adaln<1>(a, total, st);
        case 2: return adaln<2>(a, total, st);
        case 3: return adaln<3>(a, total, st);
        case 4: return adaln<4>(a, total, st);
        case 5: return adaln<5>(a, total, st);
        case 6: return adaln<6>(a, total, st);
        case 7: return adaln<7>(a, total, st);
        default: return adaln<8>(a, total, st);
    }
}

size_t residual_diff_workspace_bytes() { return sizeof(double) * 2 * kDiffMaxCtas; }

cudaError_t launch_residual_diff(const void* cur, const void* prev, int64_t n, double threshold, void* workspace,
                                 double* rel_out, int32_t* reuse_out, cudaStream_t st) {
    const int64_t nvec = n / 8;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t ctas = (nvec + 4 * kDiffThreads - 1) / (4 * kDiffThreads);
    ctas = std::max<int64_t>(1, std::min<int64_t>(ctas, std::min<int64_t>(static_cast<int64_t>(sms) * 8, kDiffMaxCtas)));
    double* partial = static_cast<double*>(workspace);
    residual_diff_partial_kernel<<<static_cast<unsigned>(ctas), kDiffThreads, 0, st>>>(
        static_cast<const uint4*>(cur), static_cast<const uint4*>(prev), nvec, partial);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    residual_diff_final_kernel<<<1, kDiffThreads, 0, st>>>(partial, static_cast<int>(ctas), threshold, rel_out,
                                                          reuse_out);
    return cudaGetLastError();
}

cudaError_t launch_swiglu(const void* in, int64_t rows, int ffn_width, void* out, cudaStream_t st) {
    SwigluArgs a;
    a.in = static_cast<const __nv_bfloat16*>(in);
    a.out = static_cast<__nv_bfloat16*>(out);
    a.fvec = ffn_width / 8;
    a.vectors = rows * a.fvec;
    if (a.vectors == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t blocks = (a.vectors + 2 * 256 - 1) / (2 * 256);
    const int64_t cap = static_cast<int64_t>(sms) * 8;
    if (blocks > cap) blocks = cap;
    swiglu_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace h3a
