// Fused QK-RMSNorm + 3D RoPE prologue (news.cocoloop.cn MiniMax-H3 SGLang
// report, fused-operator paragraph: QK-RMSNorm with 3D RoPE in one kernel, no
// change to the result; 3D multimodal RoPE from the 52hbtv.com H3-Image page,
// section 二, model table).
//
// HBM-bound: every element of Q and K is read once and written once (4 bytes
// per element, 43,008 bytes per token at 56 heads).  One warp owns one token at
// a time and walks its heads four at a time: 8 lanes per head, 12 contiguous
// channels (six rotation pairs) per lane, so a warp touches 768 contiguous
// bytes per head group and every 32-byte sector is used whole.  The RMS sum is
// reduced with three xor shuffles inside each 8-lane group.  The rotation of a
// lane's six pairs depends only on the token, so cos/sin are computed once per
// token (fp32 sincos of a two-float angle) and reused for all heads of Q and K.
#include <cuda_bf16.h>

#include <cmath>

#include "h3a_internal.h"

namespace h3a {
namespace {

constexpr int kThreads = 256;
constexpr int kLanesPerHead = 8;
constexpr int kChanPerLane = kHeadDim / kLanesPerHead;  // 12
constexpr int kPairsPerLane = kChanPerLane / 2;          // 6
constexpr int kPairsPerSection = kHeadDim / 6;           // 16

struct PrologueArgs {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    __nv_bfloat16* qo;
    __nv_bfloat16* ko;
    const float* gq;
    const float* gk;
    int64_t tokens;  // B * N
    int N, heads, H, W;
    int64_t sb, sn, sh;
    float eps;
    // theta^(-2j/32) as an unevaluated sum hi + lo of two floats
    float freq_hi[kPairsPerSection];
    float freq_lo[kPairsPerSection];
};

__device__ __forceinline__ void unpack4(uint2 v, float* x) {
    x[0] = __uint_as_float(v.x << 16);
    x[1] = __uint_as_float(v.x & 0xFFFF0000u);
    x[2] = __uint_as_float(v.y << 16);
    x[3] = __uint_as_float(v.y & 0xFFFF0000u);
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Normalise, scale, rotate and store one lane's 12 channels of one head.
__device__ __forceinline__ void norm_rope_store(const uint2 (&raw)[3], const float (&g)[kChanPerLane],
                                                const float (&cs)[kPairsPerLane], const float (&sn)[kPairsPerLane],
                                                float eps, bool active, __nv_bfloat16* dst) {
    float x[kChanPerLane];
    unpack4(raw[0], x);
    unpack4(raw[1], x + 4);
    unpack4(raw[2], x + 8);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < kChanPerLane; ++i) ss = fmaf(x[i], x[i], ss);
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    ss += __shfl_xor_sync(0xffffffffu, ss, 4);
    const float r = rsqrtf(ss * (1.0f / kHeadDim) + eps);
    uint32_t out[kPairsPerLane];
#pragma unroll
    for (int p = 0; p < kPairsPerLane; ++p) {
        const float y0 = x[2 * p] * r * g[2 * p];
        const float y1 = x[2 * p + 1] * r * g[2 * p + 1];
        const float z0 = y0 * cs[p] - y1 * sn[p];
        const float z1 = y0 * sn[p] + y1 * cs[p];
        out[p] = pack2(z0, z1);
    }
    if (active) {
        uint2* d = reinterpret_cast<uint2*>(dst);
        d[0] = make_uint2(out[0], out[1]);
        d[1] = make_uint2(out[2], out[3]);
        d[2] = make_uint2(out[4], out[5]);
    }
}

__device__ __forceinline__ void load3(const __nv_bfloat16* src, bool active, uint2 (&raw)[3]) {
    if (active) {
        const uint2* s = reinterpret_cast<const uint2*>(src);
        raw[0] = s[0];
        raw[1] = s[1];
        raw[2] = s[2];
    } else {
        raw[0] = raw[1] = raw[2] = make_uint2(0u, 0u);
    }
}

__global__ void __launch_bounds__(kThreads, 3) qk_norm_rope_kernel(const PrologueArgs a) {
    const int lane = threadIdx.x & 31;
    const int grp = lane >> 3;  // head within a group of four
    const int sub = lane & 7;   // 12-channel slice within the head
    const int c0 = sub * kChanPerLane;

    float gq[kChanPerLane], gk[kChanPerLane];
#pragma unroll
    for (int i = 0; i < kChanPerLane; ++i) {
        gq[i] = __ldg(a.gq + c0 + i);
        gk[i] = __ldg(a.gk + c0 + i);
    }

    const int64_t warps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
    const int head_groups = (a.heads + 3) >> 2;
    for (int64_t tok = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5); tok < a.tokens;
         tok += warps) {
        const int b = static_cast<int>(tok / a.N);
        const int n = static_cast<int>(tok - static_cast<int64_t>(b) * a.N);
        const int pos[3] = {n / (a.H * a.W), (n / a.W) % a.H, n % a.W};

        // rotation of this lane's six pairs at this token
        float cs[kPairsPerLane], sn[kPairsPerLane];
#pragma unroll
        for (int p = 0; p < kPairsPerLane; ++p) {
            const int pair = sub * kPairsPerLane + p;  // 0..47 within the head
            const int axis = pair / kPairsPerSection;
            const int j = pair % kPairsPerSection;
            const float ps = static_cast<float>(pos[axis]);
            const float hi = a.freq_hi[j];
            const float a_hi = ps * hi;
            const float a_lo = fmaf(ps, hi, -a_hi) + ps * a.freq_lo[j];
            float s, c;
            sincosf(a_hi, &s, &c);
            cs[p] = fmaf(-a_lo, s, c);
            sn[p] = fmaf(a_lo, c, s);
        }

        const int64_t tok_off = static_cast<int64_t>(b) * a.sb + static_cast<int64_t>(n) * a.sn + c0;
        for (int hg = 0; hg < head_groups; hg += 2) {
            const int h0 = hg * 4 + grp, h1 = h0 + 4;
            const bool act0 = h0 < a.heads, act1 = h1 < a.heads;
            const int64_t off0 = tok_off + static_cast<int64_t>(h0) * a.sh;
            const int64_t off1 = tok_off + static_cast<int64_t>(h1) * a.sh;
            uint2 rq0[3], rk0[3], rq1[3], rk1[3];
            load3(a.q + off0, act0, rq0);
            load3(a.k + off0, act0, rk0);
            load3(a.q + off1, act1, rq1);
            load3(a.k + off1, act1, rk1);
            norm_rope_store(rq0, gq, cs, sn, a.eps, act0, a.qo + off0);
            norm_rope_store(rk0, gk, cs, sn, a.eps, act0, a.ko + off0);
            norm_rope_store(rq1, gq, cs, sn, a.eps, act1, a.qo + off1);
            norm_rope_store(rk1, gk, cs, sn, a.eps, act1, a.ko + off1);
        }
    }
}

}  // namespace

cudaError_t launch_qk_norm_rope(const void* q, const void* k, void* q_out, void* k_out, const float* gamma_q,
                                const float* gamma_k, const Shape& s, int T, int H, int W, double theta,
                                float eps, cudaStream_t st) {
    (void)T;
    PrologueArgs a;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.k = static_cast<const __nv_bfloat16*>(k);
    a.qo = static_cast<__nv_bfloat16*>(q_out);
    a.ko = static_cast<__nv_bfloat16*>(k_out);
    a.gq = gamma_q;
    a.gk = gamma_k;
    a.tokens = static_cast<int64_t>(s.B) * s.N;
    a.N = s.N;
    a.heads = s.heads;
    a.H = H;
    a.W = W;
    a.sb = s.sb;
    a.sn = s.sn;
    a.sh = s.sh;
    a.eps = eps;
    for (int j = 0; j < kPairsPerSection; ++j) {
        const double f = std::pow(theta, -2.0 * j / (kHeadDim / 3));
        a.freq_hi[j] = static_cast<float>(f);
        a.freq_lo[j] = static_cast<float>(f - static_cast<double>(a.freq_hi[j]));
    }
    if (a.tokens == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t warps_needed = a.tokens;
    int64_t blocks = (warps_needed + (kThreads / 32) - 1) / (kThreads / 32);
    const int64_t cap = static_cast<int64_t>(sms) * 3 * 8;
    if (blocks > cap) blocks = cap;
    qk_norm_rope_kernel<<<static_cast<unsigned>(blocks), kThreads, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace h3a
