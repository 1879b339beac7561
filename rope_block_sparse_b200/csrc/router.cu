// Blockwise KV-block router (news.cocoloop.cn MiniMax-H3 SGLang report,
// SubBlock paragraph: a blockwise sparse router prunes the KV blocks taking
// part in attention, sparsity 0.75 or 0.80).  Pooling, scoring and selection
// follow the problem statement: mean-pooled 128-token blocks, fp32 scores,
// per-query-block top-k with ties to the lower block index.
//
// Two kernels:
//   block_pool_kernel   HBM-bound: one CTA per (batch, block, tensor) streams the
//                       block's 128 token rows (all heads) once and writes fp32
//                       means: Q's [B, heads, nblk, D], K's channel-major
//                       [B, heads, D, nblk rounded up to 4].
//   score_topk_kernel   one CTA per (batch*head, 8 query blocks): fp32 scores of
//                       its query blocks against every key block into shared
//                       memory (8 x 4 register tiles over the channel-major K
//                       means), then one warp per query block selects the top k
//                       -- 256 buckets linear in the score and an exact ranking
//                       of the bucket holding the cut, or a 4-pass 8-bit radix
//                       select over order-preserving 32-bit keys when that
//                       bucket is crowded -- and emits the indices ascending.
#include <cuda_bf16.h>

#include <cmath>

#include "h3a_internal.h"

namespace h3a {
namespace {

constexpr int kPoolThreads = 224;    // 672 16-byte vectors per CTA row: 56 heads of 96 or 42 of 128
constexpr int kVecPerThread = 3;
template <int D>
constexpr int heads_per_pool_cta() { return kPoolThreads * kVecPerThread / (D / 8); }
// Eight query blocks per score CTA (one warp each in the selection), four
// CTAs per SM: half-size CTAs keep more of them resident at large nblk and
// overlap one CTA's scores with another's selection (16-block CTAs, two per
// SM, took 0.444 against 0.413 ms at 977 blocks and 2.28 against 1.74 ms at
// 1,922, with identical lists).
constexpr int kScoreThreads = 256;   // 8 warps
constexpr int kRowsPerCta = 8;       // query blocks per score CTA
static_assert(kScoreThreads / 256 * 8 == kRowsPerCta && kScoreThreads / 32 == kRowsPerCta,
              "8 x 4 score tiles over 256 key groups; one selecting warp per query block");
constexpr int kScoreSmemLimit = 200 * 1024;

struct PoolArgs {
    const __nv_bfloat16* x[2];
    float* out[2];
    int N, heads, nblk;
    int64_t sb, sn, sh;
};

__device__ __forceinline__ void acc8(float* acc, uint4 v) {
    acc[0] += __uint_as_float(v.x << 16);
    acc[1] += __uint_as_float(v.x & 0xFFFF0000u);
    acc[2] += __uint_as_float(v.y << 16);
    acc[3] += __uint_as_float(v.y & 0xFFFF0000u);
    acc[4] += __uint_as_float(v.z << 16);
    acc[5] += __uint_as_float(v.z & 0xFFFF0000u);
    acc[6] += __uint_as_float(v.w << 16);
    acc[7] += __uint_as_float(v.w & 0xFFFF0000u);
}

// grid: (nblk, B, 2 tensors x head chunks).  Thread t covers 16-byte vectors
// t, t+224, t+448 of the chunk's part of a token row (vector v = head
// HC*chunk + v/(D/8), channels 8*(v%(D/8)) .. +7, HC = 56 heads at D = 96,
// 42 at D = 128).
template <int D>
__global__ void __launch_bounds__(kPoolThreads) block_pool_kernel(const PoolArgs a) {
    constexpr int kHeadsPerPoolCta = heads_per_pool_cta<D>();
    constexpr int kVecPerHead = D / 8;
    const int blk = blockIdx.x, b = blockIdx.y, which = blockIdx.z & 1, chunk = blockIdx.z >> 1;
    const __nv_bfloat16* x = a.x[which];
    const int n0 = blk * kBlock;
    const int n1 = min(a.N, n0 + kBlock);
    const int h_base = chunk * kHeadsPerPoolCta;
    const int vec_per_row = min(kHeadsPerPoolCta, a.heads - h_base) * kVecPerHead;

    int64_t off[kVecPerThread];
    bool act[kVecPerThread];
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
        const int v = threadIdx.x + u * kPoolThreads;
        act[u] = v < vec_per_row;
        const int h = h_base + v / kVecPerHead, c = (v % kVecPerHead) * 8;
        off[u] = static_cast<int64_t>(b) * a.sb + static_cast<int64_t>(h) * a.sh + c;
    }
    float acc[kVecPerThread][8];
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;

    int n = n0;
    for (; n + 4 <= n1; n += 4) {
        uint4 v[4][kVecPerThread];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int u = 0; u < kVecPerThread; ++u)
                v[r][u] = act[u] ? __ldg(reinterpret_cast<const uint4*>(x + off[u] + static_cast<int64_t>(n + r) * a.sn))
                                 : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int u = 0; u < kVecPerThread; ++u) acc8(acc[u], v[r][u]);
    }
    for (; n < n1; ++n) {
#pragma unroll
        for (int u = 0; u < kVecPerThread; ++u)
            if (act[u]) acc8(acc[u], __ldg(reinterpret_cast<const uint4*>(x + off[u] + static_cast<int64_t>(n) * a.sn)));
    }
    const float inv_len = 1.0f / static_cast<float>(n1 - n0);
    const int kstride = pooled_k_stride(a.nblk);
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
        if (!act[u]) continue;
        const int v = threadIdx.x + u * kPoolThreads;
        const int h = h_base + v / kVecPerHead, c = (v % kVecPerHead) * 8;
        const int64_t bh = static_cast<int64_t>(b) * a.heads + h;
        if (which == 0) {  // Q: [B, heads, nblk, D]
            float* dst = a.out[0] + (bh * a.nblk + blk) * D + c;
            reinterpret_cast<float4*>(dst)[0] =
                make_float4(acc[u][0] * inv_len, acc[u][1] * inv_len, acc[u][2] * inv_len, acc[u][3] * inv_len);
            reinterpret_cast<float4*>(dst)[1] =
                make_float4(acc[u][4] * inv_len, acc[u][5] * inv_len, acc[u][6] * inv_len, acc[u][7] * inv_len);
        } else {  // K: channel-major [B, heads, D, kstride]
            float* dst = a.out[1] + (bh * D + c) * kstride + blk;
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[static_cast<int64_t>(i) * kstride] = acc[u][i] * inv_len;
        }
    }
}

struct ScoreArgs {
    const float* qp;
    const float* kp;
    int32_t* idx;
    int nblk, kk;
    float inv_sqrt_d;
};

// Order-preserving map of a finite float to uint32 (-0 folded onto +0).
__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f == 0.f ? 0.f : f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Given a 256-bin histogram h (bin 255 the largest values) and a rank
// 1 <= r <= total, finds the bin holding the r-th largest value and the
// number of values in the bins above it.  Warp-collective; lane l reads bins
// 255-8l .. 248-8l and the counts are prefix-summed across the warp.
__device__ __forceinline__ void select_digit(const uint32_t* h, int lane, uint32_t r, uint32_t& bin,
                                             uint32_t& above) {
    uint32_t cnt[8];
    uint32_t local = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        cnt[i] = h[255 - (lane * 8 + i)];
        local += cnt[i];
    }
    uint32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    const uint32_t excl = incl - local;  // values in larger bins, from lanes before
    const bool mine = excl < r && r <= incl;
    const uint32_t owner = __ballot_sync(0xffffffffu, mine);
    const int src = __ffs(owner) - 1;
    uint32_t b = 0, ab = 0;
    if (mine) {
        uint32_t run = excl;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (run < r && r <= run + cnt[i]) {
                b = 255 - (lane * 8 + i);
                ab = run;
                break;
            }
            run += cnt[i];
        }
    }
    bin = __shfl_sync(0xffffffffu, b, src);
    above = __shfl_sync(0xffffffffu, ab, src);
}

// grid: (ceil(nblk / 8), B*heads), 256 threads.  Dynamic shared memory:
// qbar[D][8] fp32 (the CTA's 8 query-block means, channel-major),
// scores[8][nblk4] fp32 (nblk4 = nblk rounded up to 4), histograms[8][256] u32.
//
// Scores: thread t computes the CTA's 8 query blocks against key blocks
// j0 + 4*t .. +3, j0 = 0, 1024, ...: an 8 x 4 register tile.  Per
// channel it reads its four key means with one 16-byte load -- the K means are
// channel-major, so a warp's loads are 512 contiguous bytes -- and two 16-byte
// broadcasts of the query means.  Every dot product adds q_c * k_c in channel
// order c = 0..D-1 with one fmaf per channel, then scales by 1/sqrt(D).
template <int D>
__global__ void __launch_bounds__(kScoreThreads, 4) score_topk_kernel(const ScoreArgs a) {
    extern __shared__ __align__(16) float smem[];
    const int nblk4 = pooled_k_stride(a.nblk);
    float* qbar = smem;                                                  // [D][8]
    float* scores = qbar + kRowsPerCta * D;                              // [8][nblk4]
    uint32_t* hist = reinterpret_cast<uint32_t*>(scores + kRowsPerCta * nblk4);  // [8][256]

    const int bh = blockIdx.y;
    const int i0 = blockIdx.x * kRowsPerCta;
    const int rows = min(kRowsPerCta, a.nblk - i0);
    const float* qsrc = a.qp + (static_cast<int64_t>(bh) * a.nblk + i0) * D;
    const float* ksrc = a.kp + static_cast<int64_t>(bh) * D * nblk4;

    for (int e = threadIdx.x; e < kRowsPerCta * D; e += kScoreThreads) {
        const int r = e / D, c = e - r * D;
        qbar[c * kRowsPerCta + r] = (r < rows) ? qsrc[e] : 0.f;
    }
    __syncthreads();

    const int rh = threadIdx.x >> 8;   // query blocks 8*rh .. 8*rh+7 of the CTA
    const int kt = threadIdx.x & 255;  // key blocks j0 + 4*kt .. +3
    for (int j0 = 0; j0 < nblk4; j0 += 1024) {
        const int j = j0 + 4 * kt;
        if (j >= nblk4) break;
        float acc[8][4];
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[r][i] = 0.f;
        const float* kc = ksrc + j;
#pragma unroll 4
        for (int c = 0; c < D; ++c) {
            const float4 kv = __ldg(reinterpret_cast<const float4*>(kc + static_cast<int64_t>(c) * nblk4));
            const float4 qa = reinterpret_cast<const float4*>(qbar + c * kRowsPerCta + 8 * rh)[0];
            const float4 qb = reinterpret_cast<const float4*>(qbar + c * kRowsPerCta + 8 * rh)[1];
            const float q[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                acc[r][0] = fmaf(q[r], kv.x, acc[r][0]);
                acc[r][1] = fmaf(q[r], kv.y, acc[r][1]);
                acc[r][2] = fmaf(q[r], kv.z, acc[r][2]);
                acc[r][3] = fmaf(q[r], kv.w, acc[r][3]);
            }
        }
        // key blocks past nblk (the padding of the last group of four) are
        // stored too and never read
#pragma unroll
        for (int r = 0; r < 8; ++r)
            reinterpret_cast<float4*>(scores + (8 * rh + r) * nblk4 + j)[0] =
                make_float4(acc[r][0] * a.inv_sqrt_d, acc[r][1] * a.inv_sqrt_d, acc[r][2] * a.inv_sqrt_d,
                            acc[r][3] * a.inv_sqrt_d);
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp >= rows) return;
    const float* s = scores + warp * nblk4;
    uint32_t* h = hist + warp * 256;
    int32_t* out = a.idx + (static_cast<int64_t>(bh) * a.nblk + i0 + warp) * a.kk;
    const uint32_t lt_mask = (1u << lane) - 1u;

    // Selection of the kk highest scores of the row, ties to the lower index,
    // emitted ascending.  Fast path: 256 buckets linear in the score between
    // the row's min and max.  The bucket index is a non-decreasing function of
    // the value, so every key in a higher bucket is strictly larger than every
    // key in a lower one and equal values share a bucket; the buckets above
    // the one holding the kk-th largest are taken whole, and the `need` best
    // of that bucket by (score descending, index ascending) are ranked exactly
    // -- the same set the radix select below finds.  The radix select runs
    // when that bucket holds more than 32 keys or the row is constant.
    float smax = -INFINITY, smin = INFINITY;
    for (int j = lane; j < a.nblk; j += 32) {
        const float v = s[j];
        smax = fmaxf(smax, v);
        smin = fminf(smin, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, o));
        smin = fminf(smin, __shfl_xor_sync(0xffffffffu, smin, o));
    }
    const float scale = 256.0f / (smax - smin);
    if (smax > smin && scale < INFINITY) {
        auto bucket = [&](float v) { return min(255, static_cast<int>((v - smin) * scale)); };
#pragma unroll
        for (int i = 0; i < 8; ++i) h[lane * 8 + i] = 0u;
        __syncwarp();
        for (int j = lane; j < a.nblk; j += 32) atomicAdd(&h[bucket(s[j])], 1u);
        __syncwarp();
        uint32_t bstar, above;
        select_digit(h, lane, static_cast<uint32_t>(a.kk), bstar, above);
        const int need = a.kk - static_cast<int>(above);  // 1 .. size of bucket bstar
        __syncwarp();
        // the bucket's keys, in index order, into h[0 .. 31]
        int cnt = 0;
        for (int base = 0; base < a.nblk; base += 32) {
            const int j = base + lane;
            const bool c = j < a.nblk && bucket(s[j]) == static_cast<int>(bstar);
            const uint32_t m = __ballot_sync(0xffffffffu, c);
            const int pos = cnt + __popc(m & lt_mask);
            if (c && pos < 32) h[pos] = static_cast<uint32_t>(j);
            cnt += __popc(m);
        }
        __syncwarp();
        if (cnt <= 32) {
            const int cj = lane < cnt ? static_cast<int>(h[lane]) : 0;
            const float cs = lane < cnt ? s[cj] : -INFINITY;
            int rank = 0;  // candidates ahead of this one in (score desc, index asc)
            for (int m = 0; m < cnt; ++m) {
                const float sm = __shfl_sync(0xffffffffu, cs, m);
                const int jm = __shfl_sync(0xffffffffu, cj, m);
                rank += (sm > cs || (sm == cs && jm < cj)) ? 1 : 0;
            }
            const uint32_t take = __ballot_sync(0xffffffffu, lane < cnt && rank < need);
            int written = 0, eq_seen = 0;
            for (int base = 0; base < a.nblk; base += 32) {
                const int j = base + lane;
                const int bk = j < a.nblk ? bucket(s[j]) : -1;
                const bool eq = bk == static_cast<int>(bstar);
                const uint32_t eq_mask = __ballot_sync(0xffffffffu, eq);
                const bool sel = bk > static_cast<int>(bstar) ||
                                 (eq && ((take >> (eq_seen + __popc(eq_mask & lt_mask))) & 1u));
                const uint32_t sel_mask = __ballot_sync(0xffffffffu, sel);
                if (sel) out[written + __popc(sel_mask & lt_mask)] = j;
                written += __popc(sel_mask);
                eq_seen += __popc(eq_mask);
            }
            return;
        }
    }

    // radix select of the kk-th largest key, 8 bits per pass, most significant first
    uint32_t prefix = 0;
    int remaining = a.kk;
    for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i) h[lane * 8 + i] = 0u;
        __syncwarp();
        const uint32_t hi_mask = (shift == 24) ? 0u : (0xFFFFFFFFu << (shift + 8));
        for (int j = lane; j < a.nblk; j += 32) {
            const uint32_t u = order_key(s[j]);
            if ((u & hi_mask) == (prefix & hi_mask)) atomicAdd(&h[(u >> shift) & 255u], 1u);
        }
        __syncwarp();
        uint32_t digit, above;
        select_digit(h, lane, static_cast<uint32_t>(remaining), digit, above);
        prefix |= digit << shift;
        remaining -= static_cast<int>(above);
        __syncwarp();
    }

    // emit: every key above the threshold, plus the first `remaining` keys equal
    // to it (lowest indices first), in ascending index order
    int written = 0, eq_seen = 0;
    for (int base = 0; base < a.nblk; base += 32) {
        const int j = base + lane;
        const bool in = j < a.nblk;
        const uint32_t u = in ? order_key(s[j]) : 0u;
        const bool gt = in && u > prefix;
        const bool eq = in && u == prefix;
        const uint32_t eq_mask = __ballot_sync(0xffffffffu, eq);
        const int eq_rank = eq_seen + __popc(eq_mask & lt_mask);
        const bool sel = gt || (eq && eq_rank < remaining);
        const uint32_t sel_mask = __ballot_sync(0xffffffffu, sel);
        if (sel) out[written + __popc(sel_mask & lt_mask)] = j;
        written += __popc(sel_mask);
        eq_seen += __popc(eq_mask);
    }
}

size_t score_smem_bytes(int nblk, int d) {
    return (static_cast<size_t>(kRowsPerCta) * d + static_cast<size_t>(kRowsPerCta) * pooled_k_stride(nblk)) *
               sizeof(float) +
           static_cast<size_t>(kRowsPerCta) * 256 * sizeof(uint32_t);
}

template <int D>
cudaError_t scores(const float* pooled_q, const float* pooled_k, const Shape& s, int nblk, int kk, int32_t* idx,
                   cudaStream_t st) {
    ScoreArgs a;
    a.qp = pooled_q;
    a.kp = pooled_k;
    a.idx = idx;
    a.nblk = nblk;
    a.kk = kk;
    a.inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
    const size_t smem = score_smem_bytes(nblk, D);
    cudaError_t e = cudaFuncSetAttribute(score_topk_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    score_topk_kernel<D><<<dim3((nblk + kRowsPerCta - 1) / kRowsPerCta, s.B * s.heads), kScoreThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <int D>
cudaError_t pool(const void* q, const void* k, const Shape& s, int nblk, float* pooled_q, float* pooled_k,
                 cudaStream_t st) {
    PoolArgs p;
    p.x[0] = static_cast<const __nv_bfloat16*>(q);
    p.x[1] = static_cast<const __nv_bfloat16*>(k);
    p.out[0] = pooled_q;
    p.out[1] = pooled_k;
    p.N = s.N;
    p.heads = s.heads;
    p.nblk = nblk;
    p.sb = s.sb;
    p.sn = s.sn;
    p.sh = s.sh;
    constexpr int hc = heads_per_pool_cta<D>();
    const int chunks = (s.heads + hc - 1) / hc;
    block_pool_kernel<D><<<dim3(nblk, s.B, 2 * chunks), kPoolThreads, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

int route_max_blocks(int d) {
    // largest nblk whose score tile fits the shared-memory budget
    return static_cast<int>((kScoreSmemLimit - score_smem_bytes(0, d)) / (kRowsPerCta * sizeof(float))) & ~3;
}

cudaError_t launch_route_scores(const float* pooled_q, const float* pooled_k, const Shape& s, int nblk, int kk,
                                int32_t* idx, cudaStream_t st) {
    if (s.d == kHeadDimWide) return scores<kHeadDimWide>(pooled_q, pooled_k, s, nblk, kk, idx, st);
    return scores<kHeadDim>(pooled_q, pooled_k, s, nblk, kk, idx, st);
}

cudaError_t launch_route(const void* q, const void* k, const Shape& s, int nblk, int kk, float* pooled_q,
                         float* pooled_k, int32_t* idx, cudaStream_t st) {
    cudaError_t e = s.d == kHeadDimWide ? pool<kHeadDimWide>(q, k, s, nblk, pooled_q, pooled_k, st)
                                        : pool<kHeadDim>(q, k, s, nblk, pooled_q, pooled_k, st);
    if (e != cudaSuccess) return e;
    return launch_route_scores(pooled_q, pooled_k, s, nblk, kk, idx, st);
}

}  // namespace h3a
