// Fused QK-RMSNorm + 3D RoPE prologue (news.cocoloop.cn MiniMax-H3 SGLang
// report, fused-operator paragraph: QK-RMSNorm with 3D RoPE in one kernel, no
// change to the result; 3D multimodal RoPE from the 52hbtv.com H3-Image page,
// section 二, model table), the same prologue with the router's block
// pooling folded in (qk_norm_rope_pool_kernel), and the variant whose RMSNorm
// spans the token's whole hidden state (qk_fullnorm_rope_kernel, at the end).
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

#include "fastmath.cuh"
#include "h3a_internal.h"
#include "sm100.cuh"

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
    // block pooling (qk_norm_rope_pool_kernel only): the router's fp32 means
    float* pool_q;
    float* pool_k;
    int nblk;
    int* status;          // device status word (bounded-wait timeouts)
    uint64_t timeout_ns;  // limit of one pipeline wait
};

// Two packed bf16 (low half first) as an fp32 pair.
__device__ __forceinline__ uint64_t unpack2(uint32_t v) {
    return f2(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Normalise, scale and rotate one lane's 12 channels of one head; out[p] holds
// the rounded pair p as packed bf16.  A rotation pair (x0, x1) is one packed
// fp32 register pair throughout: the sum of squares, the gains g2[p] = (g0, g1)
// and the rotation rot[p] = (cos, sin) scaled by the RMS factor each take one
// f32x2 instruction per pair.  Every lane of the warp must take part (the RMS
// sum is reduced across each 8-lane group).
__device__ __forceinline__ void norm_rope(const uint2 (&raw)[3], const uint64_t (&g2)[kPairsPerLane],
                                          const uint64_t (&rot)[kPairsPerLane], float eps,
                                          uint32_t (&out)[kPairsPerLane]) {
    uint64_t x[kPairsPerLane];
#pragma unroll
    for (int q = 0; q < 3; ++q) {
        x[2 * q] = unpack2(raw[q].x);
        x[2 * q + 1] = unpack2(raw[q].y);
    }
    uint64_t ss2 = f2_mul(x[0], x[0]);
#pragma unroll
    for (int p = 1; p < kPairsPerLane; ++p) ss2 = f2_fma(x[p], x[p], ss2);
    float s0, s1;
    f2_split(ss2, s0, s1);
    float ss = s0 + s1;
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    ss += __shfl_xor_sync(0xffffffffu, ss, 4);
    const float r = rsqrtf(ss * (1.0f / kHeadDim) + eps);
    const uint64_t r2 = f2(r, r);
#pragma unroll
    for (int p = 0; p < kPairsPerLane; ++p) {
        float u0, u1, c, sn;
        f2_split(f2_mul(x[p], g2[p]), u0, u1);  // gains
        f2_split(f2_mul(rot[p], r2), c, sn);    // rotation scaled by 1 / RMS
        out[p] = pack2(fmaf(u0, c, -u1 * sn), fmaf(u0, sn, u1 * c));
    }
}

__device__ __forceinline__ void store3(const uint32_t (&out)[kPairsPerLane], bool active, __nv_bfloat16* dst) {
    if (active) {
        uint2* d = reinterpret_cast<uint2*>(dst);
        d[0] = make_uint2(out[0], out[1]);
        d[1] = make_uint2(out[2], out[3]);
        d[2] = make_uint2(out[4], out[5]);
    }
}

__device__ __forceinline__ void norm_rope_store(const uint2 (&raw)[3], const uint64_t (&g2)[kPairsPerLane],
                                                const uint64_t (&rot)[kPairsPerLane], float eps, bool active,
                                                __nv_bfloat16* dst) {
    uint32_t out[kPairsPerLane];
    norm_rope(raw, g2, rot, eps, out);
    store3(out, active, dst);
}

// The lane's gains as pairs (g[c0 + 2p], g[c0 + 2p + 1]).
__device__ __forceinline__ void load_gain_pairs(const float* g, int c0, uint64_t (&g2)[kPairsPerLane]) {
#pragma unroll
    for (int p = 0; p < kPairsPerLane; ++p) g2[p] = f2(__ldg(g + c0 + 2 * p), __ldg(g + c0 + 2 * p + 1));
}

// cos / sin of the angle pos * theta^(-2j/32) of pair j of a section at axis
// position `pos`: fp32 sincos of the high part of the angle, corrected to
// first order by its low part (the frequency is an unevaluated sum hi + lo of
// two floats).
__device__ __forceinline__ void rotation_at(int pos, int j, const float* freq_hi, const float* freq_lo,
                                            float& c_out, float& s_out) {
    const float ps = static_cast<float>(pos);
    const float hi = freq_hi[j];
    const float a_hi = ps * hi;
    const float a_lo = fmaf(ps, hi, -a_hi) + ps * freq_lo[j];
    float s, c;
    sincosf(a_hi, &s, &c);
    c_out = fmaf(-a_lo, s, c);
    s_out = fmaf(a_lo, c, s);
}

// The rotation of pair `pair` (0..47 within a head: section pair / 16 --
// t, h, w -- index j = pair % 16) at grid position (pt, ph, pw).
__device__ __forceinline__ void rotation(int pt, int ph, int pw, int pair, const float* freq_hi,
                                         const float* freq_lo, float& c_out, float& s_out) {
    const int axis = pair / kPairsPerSection;
    // selects, not an indexed array: axis depends on the lane
    rotation_at(axis == 0 ? pt : (axis == 1 ? ph : pw), pair % kPairsPerSection, freq_hi, freq_lo, c_out, s_out);
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

// Two CTAs per SM: the 128 registers that allows hold two head groups' loads
// of Q and K without spilling (at three CTAs, 80 registers, the kernel
// spilled and ran 5% slower).
__global__ void __launch_bounds__(kThreads, 2) qk_norm_rope_kernel(const PrologueArgs a) {
    const int lane = threadIdx.x & 31;
    const int grp = lane >> 3;  // head within a group of four
    const int sub = lane & 7;   // 12-channel slice within the head
    const int c0 = sub * kChanPerLane;

    uint64_t gq[kPairsPerLane], gk[kPairsPerLane];
    load_gain_pairs(a.gq, c0, gq);
    load_gain_pairs(a.gk, c0, gk);

    const int64_t warps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
    const int head_groups = (a.heads + 3) >> 2;
    for (int64_t tok = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5); tok < a.tokens;
         tok += warps) {
        const int b = static_cast<int>(tok / a.N);
        const int n = static_cast<int>(tok - static_cast<int64_t>(b) * a.N);
        const int pt = n / (a.H * a.W), ph = (n / a.W) % a.H, pw = n % a.W;

        // rotation of this lane's six pairs at this token
        uint64_t rot[kPairsPerLane];
#pragma unroll
        for (int p = 0; p < kPairsPerLane; ++p) {
            float c, sn;
            rotation(pt, ph, pw, sub * kPairsPerLane + p, a.freq_hi, a.freq_lo, c, sn);
            rot[p] = f2(c, sn);
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
            norm_rope_store(rq0, gq, rot, a.eps, act0, a.qo + off0);
            norm_rope_store(rk0, gk, rot, a.eps, act0, a.ko + off0);
            norm_rope_store(rq1, gq, rot, a.eps, act1, a.qo + off1);
            norm_rope_store(rk1, gk, rot, a.eps, act1, a.ko + off1);
        }
    }
}

// ---------------------------------------------------------------------------
// Prologue + block pooling.  The router pools the prologue's outputs over
// 128-token blocks (news.cocoloop.cn MiniMax-H3 SGLang report, SubBlock
// paragraph; block means as fixed by the problem statement); this kernel
// produces those means while the rounded outputs are still in registers, so
// the router need not read Q and K back from HBM.
//
// One CTA per (batch, 128-token block, chunk of 28 heads).  Warp 7 streams the
// block's token rows into a ring of kPoolRing slots in shared memory with TMA
// (one 28-head x 96-channel slice of Q and one of K per token, 5,376 bytes
// each, through a tensor map, so any head and token stride works), so the
// loads in flight hold no registers.  Warps 0-6 own four heads each with the
// prologue's lane layout (8 lanes per head, 12 channels per lane): per token a
// warp reads its slice from the slot, releases the slot, normalises, rotates,
// stores the rounded outputs and adds them to its block sums.  Each (head,
// channel) sum lives in one lane and adds the bf16-rounded outputs in token
// order, exactly as the separate pooling kernel does, so the means are
// bit-identical to it.  The rotations are computed once per CTA into shared
// memory (while the first tokens load): a pair's angle depends on one axis
// position only, so the block needs one row of 16 (cos, sin) per distinct w,
// per distinct (t, h) row and per distinct t of its tokens -- some 90 rows for
// the clip grids instead of 128 tokens x 48 pairs -- and each warp steps its
// tokens' (w, h, t) indices with counters instead of divisions.
// Every barrier wait is bounded; an expired wait sets the device status word.
constexpr int kPoolWarps = 7;                              // consumer warps
constexpr int kPoolThreads = 32 * (kPoolWarps + 1);        // + the TMA producer warp
constexpr int kPoolConsumers = 32 * kPoolWarps;            // 224
constexpr int kPoolHeadsPerCta = 4 * kPoolWarps;           // 28
constexpr int kPairsPerHead = kHeadDim / 2;                // 48
constexpr int kPoolRing = 5;                               // tokens in flight per CTA
constexpr int kSliceBytes = kPoolHeadsPerCta * kHeadDim * 2;  // 5,376
static_assert(kSliceBytes % 128 == 0, "slots stay 128-byte aligned");

// Rows of 16 (cos, sin) pairs the block's rotation tables can need: at most
// 128 distinct w values plus two more rows of (t, h) for a 128-token block
// (nw + nr <= 130 for any W), and at most 128 distinct t values.
constexpr int kRotRows = 130 + kBlock;
struct PoolSmem {
    uint8_t ring[kPoolRing][2][kSliceBytes];     // [slot][Q, K][28 heads x 96 bf16]
    float2 rot[kRotRows * kPairsPerSection];     // (cos, sin): w rows, then (t, h) rows, then t rows
    uint64_t full[kPoolRing], empty[kPoolRing];
    int abort_flag;
    int never;  // stays 0: abort flag for the producer's final drain
};
constexpr size_t kPoolSmemBytes = sizeof(PoolSmem) + 1024;  // + alignment slack

// acc[p] += the rounded pair p (one f32x2 add: the same fp32 sums, in the same
// token order, as two scalar adds).
__device__ __forceinline__ void add_rounded(const uint32_t (&out)[kPairsPerLane], uint64_t (&acc)[kPairsPerLane]) {
#pragma unroll
    for (int p = 0; p < kPairsPerLane; ++p) acc[p] = f2_add(acc[p], unpack2(out[p]));
}

__device__ __forceinline__ void pool_timeout(const PrologueArgs& a, volatile int* abort_flag) {
    *abort_flag = 1;
    atomicOr(a.status, kDevTimeout);
}

__global__ void __launch_bounds__(kPoolThreads, 2)
    qk_norm_rope_pool_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                             const PrologueArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base_addr = smem_u32(smem_raw);
    PoolSmem& sm = *reinterpret_cast<PoolSmem*>(smem_raw + (((base_addr + 1023u) & ~1023u) - base_addr));
    const int blk = blockIdx.x, b = blockIdx.y, chunk = blockIdx.z;
    const int n0 = blk * kBlock;
    const int len = min(a.N - n0, kBlock);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort_flag = &sm.abort_flag;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kPoolRing; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], kPoolWarps);  // one arrival per consumer warp
        }
        sm.abort_flag = 0;
        sm.never = 0;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == kPoolWarps) {
        // TMA producer: token t goes to slot t % kPoolRing once the consumers
        // have released that slot's previous token
        if (lane == 0) {
            prefetch_tensor_map(&tq);
            prefetch_tensor_map(&tk);
            const int h0 = chunk * kPoolHeadsPerCta;
            int issued = 0;
            for (int t = 0; t < len; ++t) {
                const int slot = t % kPoolRing;
                const uint32_t ph = static_cast<uint32_t>(t / kPoolRing) & 1u;
                if (t >= kPoolRing && !mbar_wait(&sm.empty[slot], ph ^ 1u, abort_flag, a.timeout_ns)) {
                    pool_timeout(a, abort_flag);
                    break;
                }
                // the consumers read the slot's previous token with ordinary
                // shared-memory loads; the TMA refill below writes through the
                // async proxy, which the barrier alone does not order after them
                fence_proxy_async_shared();
                mbar_arrive_expect_tx(&sm.full[slot], 2 * kSliceBytes);
                tma_load_4d(sm.ring[slot][0], &tq, &sm.full[slot], 0, h0, n0 + t, b);
                tma_load_4d(sm.ring[slot][1], &tk, &sm.full[slot], 0, h0, n0 + t, b);
                issued = t + 1;
            }
            // every load issued must have landed before the CTA exits (normally
            // the consumers have already waited for each of them)
            for (int t = max(0, issued - kPoolRing); t < issued; ++t)
                mbar_wait(&sm.full[t % kPoolRing], static_cast<uint32_t>(t / kPoolRing) & 1u, &sm.never,
                          a.timeout_ns);
        }
        return;
    }

    // consumers: the block's rotation tables first, while the first tokens load
    const int HW = a.H * a.W;
    const int w0 = n0 % a.W, r0 = n0 / a.W, t0 = n0 / HW;
    const int nw = min(len, a.W);                       // w rows: w = (w0 + k) mod W
    const int nr = (n0 + len - 1) / a.W - r0 + 1;       // (t, h) rows r0 .. : h = r mod H
    const int nt = (n0 + len - 1) / HW - t0 + 1;        // t rows t0 ..
    for (int e = threadIdx.x; e < (nw + nr + nt) * kPairsPerSection; e += kPoolConsumers) {
        const int row = e / kPairsPerSection, j = e - row * kPairsPerSection;
        int pos;
        if (row < nw) {
            pos = w0 + row;
            if (pos >= a.W) pos -= a.W;
        } else if (row < nw + nr) {
            pos = (r0 + row - nw) % a.H;
        } else {
            pos = t0 + row - nw - nr;
        }
        float c, sn;
        rotation_at(pos, j, a.freq_hi, a.freq_lo, c, sn);
        sm.rot[e] = make_float2(c, sn);
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kPoolConsumers) : "memory");  // the consumer warps only

    const int sub = lane & 7;
    const int c0 = sub * kChanPerLane;
    const int hl = warp * 4 + (lane >> 3);  // head within the chunk
    const int h = chunk * kPoolHeadsPerCta + hl;
    const bool active = h < a.heads;
    uint64_t gq[kPairsPerLane], gk[kPairsPerLane];
    load_gain_pairs(a.gq, c0, gq);
    load_gain_pairs(a.gk, c0, gk);
    uint64_t accq[kPairsPerLane], acck[kPairsPerLane];
#pragma unroll
    for (int p = 0; p < kPairsPerLane; ++p) accq[p] = acck[p] = f2(0.f, 0.f);

    const int64_t base = static_cast<int64_t>(b) * a.sb + static_cast<int64_t>(h) * a.sh + c0;
    const int lane_off = hl * kHeadDim * 2 + sub * kChanPerLane * 2;  // byte offset of the lane's 12 channels
    // the lane's six pairs: section (0 t, 1 h, 2 w) and index within it
    int axis[kPairsPerLane], jj[kPairsPerLane];
#pragma unroll
    for (int p = 0; p < kPairsPerLane; ++p) {
        axis[p] = (sub * kPairsPerLane + p) / kPairsPerSection;
        jj[p] = (sub * kPairsPerLane + p) % kPairsPerSection;
    }
    // table rows of the current token, stepped token by token
    int kw = 0, mh = 0, mt = 0, wcur = w0, hcur = r0 % a.H;
    bool ok = true;
    for (int t = 0; t < len; ++t) {
        const int slot = t % kPoolRing;
        const uint32_t ph = static_cast<uint32_t>(t / kPoolRing) & 1u;
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.full[slot], ph, abort_flag, a.timeout_ns))) {
            ok = false;
            break;
        }
        const uint2* sq = reinterpret_cast<const uint2*>(sm.ring[slot][0] + lane_off);
        const uint2* sk = reinterpret_cast<const uint2*>(sm.ring[slot][1] + lane_off);
        const uint2 rq[3] = {sq[0], sq[1], sq[2]};
        const uint2 rk[3] = {sk[0], sk[1], sk[2]};
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[slot]);  // the slice is in registers
        uint64_t rot[kPairsPerLane];
        const int row_t = nw + nr + mt, row_h = nw + mh, row_w = kw;
#pragma unroll
        for (int p = 0; p < kPairsPerLane; ++p) {
            const int row = axis[p] == 0 ? row_t : (axis[p] == 1 ? row_h : row_w);
            rot[p] = *reinterpret_cast<const uint64_t*>(&sm.rot[row * kPairsPerSection + jj[p]]);  // (cos, sin)
        }
        // next token: w advances; a wrap of w moves to the next (t, h) row, a
        // wrap of h to the next t
        if (++kw == a.W) kw = 0;
        if (++wcur == a.W) {
            wcur = 0;
            ++mh;
            if (++hcur == a.H) {
                hcur = 0;
                ++mt;
            }
        }
        const int64_t off = base + static_cast<int64_t>(n0 + t) * a.sn;
        uint32_t oq[kPairsPerLane], ok_[kPairsPerLane];
        norm_rope(rq, gq, rot, a.eps, oq);
        norm_rope(rk, gk, rot, a.eps, ok_);
        store3(oq, active, a.qo + off);
        store3(ok_, active, a.ko + off);
        add_rounded(oq, accq);
        add_rounded(ok_, acck);
    }
    if (!ok) {
        pool_timeout(a, abort_flag);
        return;
    }
    if (!active) return;
    const float inv_len = 1.0f / static_cast<float>(len);
    // Q's means row-major [B, heads, nblk, 96]; K's channel-major
    // [B, heads, 96, stride], the router's layouts
    const int64_t bh = static_cast<int64_t>(b) * a.heads + h;
    float mq[kChanPerLane], mk[kChanPerLane];
#pragma unroll
    for (int p = 0; p < kPairsPerLane; ++p) {
        f2_split(accq[p], mq[2 * p], mq[2 * p + 1]);
        f2_split(acck[p], mk[2 * p], mk[2 * p + 1]);
    }
    float4* dq = reinterpret_cast<float4*>(a.pool_q + (bh * a.nblk + blk) * kHeadDim + c0);
#pragma unroll
    for (int u = 0; u < kChanPerLane / 4; ++u)
        dq[u] = make_float4(mq[4 * u] * inv_len, mq[4 * u + 1] * inv_len, mq[4 * u + 2] * inv_len,
                            mq[4 * u + 3] * inv_len);
    const int kstride = pooled_k_stride(a.nblk);
    float* dk = a.pool_k + (bh * kHeadDim + c0) * kstride + blk;
#pragma unroll
    for (int i = 0; i < kChanPerLane; ++i) dk[static_cast<int64_t>(i) * kstride] = mk[i] * inv_len;
}

// ---------------------------------------------------------------------------
// RMSNorm over the whole hidden state (all heads x 96 channels of a token, one
// gain per hidden channel), then the same per-head 3D RoPE: the other reading
// of "QK-RMSNorm" in the fused-operator paragraph.  One 224-thread CTA per
// token keeps the token's Q and K rows in registers (16-byte vector v of a row
// = head v / 12, channels 8 * (v % 12) .. + 7; three vectors per thread per
// tensor at 56 heads), so each row is read from HBM once: sums of squares of
// Q and of K reduced over the CTA, the token's 48 rotations computed once into
// shared memory, then scale, rotate and store.
constexpr int kFullThreads = 224;
constexpr int kFullWarps = kFullThreads / 32;
constexpr int kVecPerHead = kHeadDim / 8;  // 12

template <int VPT>
__global__ void __launch_bounds__(kFullThreads) qk_fullnorm_rope_kernel(const PrologueArgs a) {
    __shared__ float2 rot[kPairsPerHead];
    __shared__ float red[2][kFullWarps];
    const int64_t tok = blockIdx.x;
    const int b = static_cast<int>(tok / a.N);
    const int n = static_cast<int>(tok - static_cast<int64_t>(b) * a.N);
    if (threadIdx.x < kPairsPerHead) {
        float c, sn;
        rotation(n / (a.H * a.W), (n / a.W) % a.H, n % a.W, threadIdx.x, a.freq_hi, a.freq_lo, c, sn);
        rot[threadIdx.x] = make_float2(c, sn);
    }
    const int nvec = a.heads * kVecPerHead;
    const int64_t tok_off = static_cast<int64_t>(b) * a.sb + static_cast<int64_t>(n) * a.sn;
    uint4 xq[VPT], xk[VPT];
    float ssq = 0.f, ssk = 0.f;
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
        const int v = threadIdx.x + u * kFullThreads;
        xq[u] = xk[u] = make_uint4(0, 0, 0, 0);
        if (v < nvec) {
            const int64_t off = tok_off + static_cast<int64_t>(v / kVecPerHead) * a.sh + (v % kVecPerHead) * 8;
            xq[u] = __ldg(reinterpret_cast<const uint4*>(a.q + off));
            xk[u] = __ldg(reinterpret_cast<const uint4*>(a.k + off));
        }
        const uint32_t wq[4] = {xq[u].x, xq[u].y, xq[u].z, xq[u].w};
        const uint32_t wk[4] = {xk[u].x, xk[u].y, xk[u].z, xk[u].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float q0 = __uint_as_float(wq[i] << 16), q1 = __uint_as_float(wq[i] & 0xFFFF0000u);
            const float k0 = __uint_as_float(wk[i] << 16), k1 = __uint_as_float(wk[i] & 0xFFFF0000u);
            ssq = fmaf(q0, q0, fmaf(q1, q1, ssq));
            ssk = fmaf(k0, k0, fmaf(k1, k1, ssk));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
        ssk += __shfl_xor_sync(0xffffffffu, ssk, o);
    }
    if ((threadIdx.x & 31) == 0) {
        red[0][threadIdx.x >> 5] = ssq;
        red[1][threadIdx.x >> 5] = ssk;
    }
    __syncthreads();  // also publishes rot[]
    ssq = ssk = 0.f;
#pragma unroll
    for (int w = 0; w < kFullWarps; ++w) {
        ssq += red[0][w];
        ssk += red[1][w];
    }
    const float inv_width = 1.0f / static_cast<float>(a.heads * kHeadDim);
    const float rq = rsqrtf(ssq * inv_width + a.eps);
    const float rk = rsqrtf(ssk * inv_width + a.eps);
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
        const int v = threadIdx.x + u * kFullThreads;
        if (v >= nvec) continue;
        const int h = v / kVecPerHead, c0 = (v % kVecPerHead) * 8;
        const int64_t off = tok_off + static_cast<int64_t>(h) * a.sh + c0;
        float gq[8], gk[8];
        const float4* pq = reinterpret_cast<const float4*>(a.gq + h * kHeadDim + c0);
        const float4* pk = reinterpret_cast<const float4*>(a.gk + h * kHeadDim + c0);
        const float4 gq0 = __ldg(pq), gq1 = __ldg(pq + 1), gk0 = __ldg(pk), gk1 = __ldg(pk + 1);
        gq[0] = gq0.x, gq[1] = gq0.y, gq[2] = gq0.z, gq[3] = gq0.w, gq[4] = gq1.x, gq[5] = gq1.y, gq[6] = gq1.z,
        gq[7] = gq1.w;
        gk[0] = gk0.x, gk[1] = gk0.y, gk[2] = gk0.z, gk[3] = gk0.w, gk[4] = gk1.x, gk[5] = gk1.y, gk[6] = gk1.z,
        gk[7] = gk1.w;
        const uint32_t wq[4] = {xq[u].x, xq[u].y, xq[u].z, xq[u].w};
        const uint32_t wk[4] = {xk[u].x, xk[u].y, xk[u].z, xk[u].w};
        uint32_t oq[4], ok[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 cs = rot[c0 / 2 + i];  // pair (c0 + 2i, c0 + 2i + 1) of the head
            const float q0 = __uint_as_float(wq[i] << 16) * rq * gq[2 * i];
            const float q1 = __uint_as_float(wq[i] & 0xFFFF0000u) * rq * gq[2 * i + 1];
            const float k0 = __uint_as_float(wk[i] << 16) * rk * gk[2 * i];
            const float k1 = __uint_as_float(wk[i] & 0xFFFF0000u) * rk * gk[2 * i + 1];
            oq[i] = pack2(q0 * cs.x - q1 * cs.y, q0 * cs.y + q1 * cs.x);
            ok[i] = pack2(k0 * cs.x - k1 * cs.y, k0 * cs.y + k1 * cs.x);
        }
        *reinterpret_cast<uint4*>(a.qo + off) = make_uint4(oq[0], oq[1], oq[2], oq[3]);
        *reinterpret_cast<uint4*>(a.ko + off) = make_uint4(ok[0], ok[1], ok[2], ok[3]);
    }
}

}  // namespace

namespace {

// theta^(-2j/32), j = 0..15, split into an unevaluated sum hi + lo of two floats.
void set_frequencies(double theta, PrologueArgs& a) {
    for (int j = 0; j < kPairsPerSection; ++j) {
        const double f = std::pow(theta, -2.0 * j / (kHeadDim / 3));
        a.freq_hi[j] = static_cast<float>(f);
        a.freq_lo[j] = static_cast<float>(f - static_cast<double>(a.freq_hi[j]));
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
    set_frequencies(theta, a);
    a.pool_q = a.pool_k = nullptr;
    a.nblk = 0;
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

cudaError_t launch_qk_norm_rope_pool(const CUtensorMap& tq, const CUtensorMap& tk, void* q_out, void* k_out,
                                     const float* gamma_q, const float* gamma_k, const Shape& s, int H, int W,
                                     double theta, float eps, float* pool_q, float* pool_k, int* status,
                                     uint64_t timeout_ns, cudaStream_t st) {
    PrologueArgs a;
    a.q = nullptr;  // read through the tensor maps
    a.k = nullptr;
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
    set_frequencies(theta, a);
    a.pool_q = pool_q;
    a.pool_k = pool_k;
    a.nblk = (s.N + kBlock - 1) / kBlock;
    a.status = status;
    a.timeout_ns = timeout_ns;
    const int chunks = (s.heads + kPoolHeadsPerCta - 1) / kPoolHeadsPerCta;
    cudaError_t e = cudaFuncSetAttribute(qk_norm_rope_pool_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kPoolSmemBytes));
    if (e != cudaSuccess) return e;
    qk_norm_rope_pool_kernel<<<dim3(a.nblk, s.B, chunks), kPoolThreads, kPoolSmemBytes, st>>>(tq, tk, a);
    return cudaGetLastError();
}

cudaError_t launch_qk_fullnorm_rope(const void* q, const void* k, void* q_out, void* k_out, const float* gamma_q,
                                    const float* gamma_k, const Shape& s, int H, int W, double theta, float eps,
                                    cudaStream_t st) {
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
    set_frequencies(theta, a);
    a.pool_q = a.pool_k = nullptr;
    a.nblk = 0;
    if (a.tokens == 0) return cudaSuccess;
    const unsigned grid = static_cast<unsigned>(a.tokens);
    switch ((s.heads * kVecPerHead + kFullThreads - 1) / kFullThreads) {
        case 1: qk_fullnorm_rope_kernel<1><<<grid, kFullThreads, 0, st>>>(a); break;
        case 2: qk_fullnorm_rope_kernel<2><<<grid, kFullThreads, 0, st>>>(a); break;
        case 3: qk_fullnorm_rope_kernel<3><<<grid, kFullThreads, 0, st>>>(a); break;
        case 4: qk_fullnorm_rope_kernel<4><<<grid, kFullThreads, 0, st>>>(a); break;
        default: return cudaErrorNotSupported;  // more than 74 heads
    }
    return cudaGetLastError();
}

}  // namespace h3a
