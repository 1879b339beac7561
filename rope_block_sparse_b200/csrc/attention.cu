// Bidirectional flash attention for sm_100a, dense or over routed KV blocks.
//
// Dense lossless path and SubBlock sparse attention: news.cocoloop.cn
// MiniMax-H3 SGLang report (opening quote: dense path with no approximation;
// SubBlock paragraph: a blockwise router prunes KV blocks; "Ein paar Grenzen":
// long non-causal attention in BF16).
//
// One CTA owns two 128-row query tiles of one (batch, head) -- query blocks
// 2p and 2p+1, i.e. the router's query blocks -- and streams 128-row K/V tiles
// through shared memory: every KV block for dense attention, or each tile's
// own routed list in sparse mode (a KV tile both lists name at the same step is
// loaded once and shared).  Each 128-key block is processed as two 64-key
// half-steps u = 2j + h.  Warp roles (384 threads):
//   warp 0      TMA producer: Q tiles once, then a 3-stage K ring and a 3-stage
//               V ring (64-byte swizzled 128 x 32 chunks, 3 per 128 x 96 tile).
//   warp 1      owns tensor memory (512 columns) and issues tcgen05.mma from one
//               thread: S_t[h] = Q_t K_h^T (M=128, N=64, K=96 as 6 steps of 16)
//               into one of two S buffers per tile, O_t += P_t[h] V_h (M=128,
//               N=96, K=64 as 4 steps; P read from TMEM, V as an MN-major
//               operand).  Order per half-step u and tile t: wait P_t(u),
//               PV_t(u), then QK_t(u+2) into the buffer PV_t(u) just read, so
//               the next S of every tile is computed while its softmax runs.
//   warps 4-7   softmax of tile 0, warps 8-11 softmax of tile 1: thread r owns
//               query row r (TMEM lane r); it reads its 64 S values from TMEM,
//               keeps the running max / sum in fp32 (log2 domain), computes
//               exponentials on the MUFU unit and, for three pairs in eight, as
//               a polynomial on the FMA pipe, writes P as packed bf16 over the
//               first 32 columns of the S buffer, and rescales its O row in TMEM
//               only when the max grew by more than 2^8 (the final division by
//               the row sum keeps this exact).  At the end it divides O by the
//               row sum, rounds once to bf16 and stores the row.
// TMEM columns: S_0[0..1] [0,128), S_1[0..1] [128,256), O_0 [256,352),
// O_1 [352,448).  Every mbarrier wait is bounded (timeout + CTA abort flag); a
// timeout sets the device status word instead of hanging or trapping.
#include <cuda_bf16.h>

#include "h3a_internal.h"
#include "fastmath.cuh"
#include "sm100.cuh"

namespace h3a {
namespace {

constexpr int kThreads = 384;
constexpr int kStages = 3;
constexpr int kChunkBytes = 128 * 64;        // 128 rows x 32 bf16, 64-byte swizzle
constexpr int kTileBytes = 3 * kChunkBytes;  // 128 x 96 bf16
constexpr int kHalf = 64;                     // keys per half-step (half a 128-token KV block)
constexpr uint32_t kTmemCols = 512;
// TMEM columns: S_t[h] (64 fp32 columns; P_t[h] as packed bf16 over its first
// 32) at 128t + 64h, O_t (96 fp32 columns) at 256 + 96t.
__host__ __device__ constexpr uint32_t col_s(int t, int h) { return 128u * t + 64u * h; }
__host__ __device__ constexpr uint32_t col_o(int t) { return 256u + 96u * t; }
constexpr uint32_t kSwizzle64 = 4;

struct AttnSmem {
    uint8_t q[2][kTileBytes];
    uint8_t k[kStages][kTileBytes];
    uint8_t v[kStages][kTileBytes];
    uint64_t q_full[2];
    uint64_t k_full[kStages], k_empty[kStages];
    uint64_t v_full[kStages], v_empty[kStages];
    uint64_t s_full[2][2], p_full[2][2];  // [tile][S buffer]
    uint64_t pv_done[2], o_done[2];
    uint64_t mma_drain;
    uint32_t tmem_base;
    int abort_flag;
    int never;  // stays 0: abort flag for waits that must ignore an abort
};

constexpr size_t kSmemBytes = sizeof(AttnSmem) + 1024;  // + alignment slack

struct AttnArgs {
    __nv_bfloat16* o;
    const int32_t* blocks;  // [B, heads, nblk, n_iter] or null
    int N, heads, nblk, npairs, n_iter;
    int64_t sb, sn, sh;
    float scale_log2;  // logit scale * log2(e)
    int* status;
    uint64_t timeout_ns;
};

__device__ __forceinline__ void raise_timeout(const AttnArgs& a, volatile int* abort_flag) {
    *abort_flag = 1;
    atomicOr(a.status, kDevTimeout);
}

// K-major operand from a 128 x 96 tile (three swizzled 32-column chunks of
// 64-byte rows): k-step s covers columns [16s, 16s + 16), starting at row0.
__device__ __forceinline__ uint64_t kmajor_desc(const uint8_t* tile, int s, int row0) {
    return smem_desc(smem_u32(tile) + (s >> 1) * kChunkBytes + (s & 1) * 32 + row0 * 64, 16, 512, kSwizzle64);
}

// The same [128 kv rows x 96] tile read as an MN-major operand (N = 96 along
// the contiguous dimension, K = kv rows): 16 rows from row0.
__device__ __forceinline__ uint64_t mnmajor_desc(const uint8_t* tile, int row0) {
    return smem_desc(smem_u32(tile) + row0 * 64, kChunkBytes, 512, kSwizzle64);
}

struct KvPlan {
    int kv0, kv1;
    bool shared;  // tile 1 exists and reads the same KV block as tile 0 at this step
};

__device__ __forceinline__ KvPlan kv_plan(const int32_t* l0, const int32_t* l1, bool has1, int j) {
    KvPlan p;
    p.kv0 = l0 ? __ldg(l0 + j) : j;
    p.kv1 = has1 ? (l1 ? __ldg(l1 + j) : j) : p.kv0;
    p.shared = has1 && p.kv1 == p.kv0;
    return p;
}

__device__ void producer(AttnSmem& sm, const AttnArgs& a, const CUtensorMap* tq, const CUtensorMap* tk,
                         const CUtensorMap* tv, int b, int h, int qb0, bool has1, const int32_t* l0,
                         const int32_t* l1, volatile int* abort_flag) {
    prefetch_tensor_map(tq);
    prefetch_tensor_map(tk);
    prefetch_tensor_map(tv);
    const int ntiles = has1 ? 2 : 1;
    for (int t = 0; t < ntiles; ++t) {
        mbar_arrive_expect_tx(&sm.q_full[t], kTileBytes);
        for (int c = 0; c < 3; ++c)
            tma_load_4d(sm.q[t] + c * kChunkBytes, tq, &sm.q_full[t], 32 * c, h, (qb0 + t) * 128, b);
    }
    uint32_t ks = 0, kph = 0, vs = 0, vph = 0;
    // per stage: bit s of *_issued = a load was issued, bit s of *_par = its phase parity
    uint32_t k_issued = 0, k_par = 0, v_issued = 0, v_par = 0;
    bool ok = true;
    for (int j = 0; j < a.n_iter && ok; ++j) {
        const KvPlan p = kv_plan(l0, l1, has1, j);
        const int nld = (has1 && !p.shared) ? 2 : 1;
        for (int u = 0; u < nld && ok; ++u) {
            if (!mbar_wait(&sm.k_empty[ks], kph ^ 1u, abort_flag, a.timeout_ns)) {
                ok = false;
                break;
            }
            const int kv = u ? p.kv1 : p.kv0;
            mbar_arrive_expect_tx(&sm.k_full[ks], kTileBytes);
            for (int c = 0; c < 3; ++c)
                tma_load_4d(sm.k[ks] + c * kChunkBytes, tk, &sm.k_full[ks], 32 * c, h, kv * 128, b);
            k_issued |= 1u << ks;
            k_par = (k_par & ~(1u << ks)) | (kph << ks);
            if (++ks == kStages) {
                ks = 0;
                kph ^= 1u;
            }
        }
        for (int u = 0; u < nld && ok; ++u) {
            if (!mbar_wait(&sm.v_empty[vs], vph ^ 1u, abort_flag, a.timeout_ns)) {
                ok = false;
                break;
            }
            const int kv = u ? p.kv1 : p.kv0;
            mbar_arrive_expect_tx(&sm.v_full[vs], kTileBytes);
            for (int c = 0; c < 3; ++c)
                tma_load_4d(sm.v[vs] + c * kChunkBytes, tv, &sm.v_full[vs], 32 * c, h, kv * 128, b);
            v_issued |= 1u << vs;
            v_par = (v_par & ~(1u << vs)) | (vph << vs);
            if (++vs == kStages) {
                vs = 0;
                vph ^= 1u;
            }
        }
    }
    if (!ok) raise_timeout(a, abort_flag);
    // Drain: every load issued must have landed before the CTA may exit.
    volatile int* never = &sm.never;
    for (int t = 0; t < ntiles; ++t) mbar_wait(&sm.q_full[t], 0u, never, a.timeout_ns);
    for (int s = 0; s < kStages; ++s) {
        if ((k_issued >> s) & 1u) mbar_wait(&sm.k_full[s], (k_par >> s) & 1u, never, a.timeout_ns);
        if ((v_issued >> s) & 1u) mbar_wait(&sm.v_full[s], (v_par >> s) & 1u, never, a.timeout_ns);
    }
}

// ---------------------------------------------------------------- MMA issue

struct MmaState {
    uint32_t ks = 0, kph = 0, vs = 0, vph = 0;  // ring positions
    uint32_t kst[2] = {0, 0}, vst[2] = {0, 0};  // stage each tile reads for the current block
};

// S_t[h] = Q_t K_half^T for half h of the step's KV block (M=128, N=64, K=96).
__device__ __forceinline__ bool issue_qk(AttnSmem& sm, const AttnArgs& a, MmaState& st, uint32_t tmem, int t,
                                         int u, const KvPlan& p, volatile int* abort_flag) {
    const int h = u & 1;
    if (h == 0) {
        if (t == 0 || !p.shared) {
            if (!mbar_wait(&sm.k_full[st.ks], st.kph, abort_flag, a.timeout_ns)) return false;
            st.kst[t] = st.ks;
            if (++st.ks == kStages) {
                st.ks = 0;
                st.kph ^= 1u;
            }
        } else {
            st.kst[1] = st.kst[0];
        }
    }
    const uint32_t stage = st.kst[t];
    tc_fence_after_sync();
    constexpr uint32_t idesc = idesc_bf16_f32(128, kHalf, 0, 0);
#pragma unroll
    for (int s = 0; s < 6; ++s)
        mma_ss(tmem + col_s(t, h), kmajor_desc(sm.q[t], s, 0), kmajor_desc(sm.k[stage], s, kHalf * h), idesc,
               s > 0 ? 1u : 0u);
    tc_commit(&sm.s_full[t][h]);
    if (h == 1 && (t == 1 || !p.shared)) tc_commit(&sm.k_empty[stage]);
    return true;
}

// O_t += P_t[h] V_half (M=128, N=96, K=64), P read from TMEM.
__device__ __forceinline__ bool issue_pv(AttnSmem& sm, const AttnArgs& a, MmaState& st, uint32_t tmem, int t,
                                         int u, const KvPlan& p, volatile int* abort_flag) {
    const int h = u & 1;
    if (h == 0) {
        if (t == 0 || !p.shared) {
            if (!mbar_wait(&sm.v_full[st.vs], st.vph, abort_flag, a.timeout_ns)) return false;
            st.vst[t] = st.vs;
            if (++st.vs == kStages) {
                st.vs = 0;
                st.vph ^= 1u;
            }
        } else {
            st.vst[1] = st.vst[0];
        }
    }
    const uint32_t stage = st.vst[t];
    tc_fence_after_sync();
    constexpr uint32_t idesc = idesc_bf16_f32(128, 96, 0, 1);
#pragma unroll
    for (int s = 0; s < kHalf / 16; ++s)
        mma_ts(tmem + col_o(t), tmem + col_s(t, h) + 8 * s, mnmajor_desc(sm.v[stage], kHalf * h + 16 * s), idesc,
               (u == 0 && s == 0) ? 0u : 1u);
    tc_commit(&sm.pv_done[t]);
    if (h == 1 && (t == 1 || !p.shared)) tc_commit(&sm.v_empty[stage]);
    return true;
}

// Issue order over half-steps u = 2j + h: QK for u = 0, 1 of both tiles, then
// per u and tile: wait P_t(u), PV_t(u), QK_t(u + 2) into the S buffer PV_t(u)
// has just consumed (tcgen05.mma from one thread executes in issue order).
// Each tile therefore always has the next S ready while its softmax runs.
__device__ void mma_issuer(AttnSmem& sm, const AttnArgs& a, uint32_t tmem, bool has1, const int32_t* l0,
                           const int32_t* l1, volatile int* abort_flag) {
    const int ntiles = has1 ? 2 : 1;
    const int nsub = 2 * a.n_iter;
    bool ok = true;
    for (int t = 0; t < ntiles && ok; ++t) ok = mbar_wait(&sm.q_full[t], 0u, abort_flag, a.timeout_ns);
    MmaState st;
    KvPlan cur = kv_plan(l0, l1, has1, 0);
    for (int u = 0; u < 2 && ok; ++u)
        for (int t = 0; t < ntiles && ok; ++t) ok = issue_qk(sm, a, st, tmem, t, u, cur, abort_flag);
    KvPlan next = cur;
    for (int u = 0; u < nsub && ok; ++u) {
        const int h = u & 1;
        if (h == 0) {
            cur = (u == 0) ? cur : next;
            if (u + 2 < nsub) next = kv_plan(l0, l1, has1, (u >> 1) + 1);
        }
        for (int t = 0; t < ntiles && ok; ++t) {
            if (!mbar_wait(&sm.p_full[t][h], static_cast<uint32_t>((u >> 1) & 1), abort_flag, a.timeout_ns)) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            if (!issue_pv(sm, a, st, tmem, t, u, cur, abort_flag)) {
                ok = false;
                break;
            }
            if (u + 2 < nsub) {
                if (!issue_qk(sm, a, st, tmem, t, u + 2, next, abort_flag)) ok = false;
            } else if (u == nsub - 1) {
                tc_commit(&sm.o_done[t]);
            }
        }
    }
    if (!ok) raise_timeout(a, abort_flag);
    // Drain: every MMA issued must have completed before TMEM is released.
    tc_commit(&sm.mma_drain);
    volatile int* never = &sm.never;
    mbar_wait(&sm.mma_drain, 0u, never, a.timeout_ns);
}

// ---------------------------------------------------------------- softmax

// Pairs i (mod 8) whose exponentials take the polynomial path; the rest use
// ex2.approx on the MUFU unit.  Three of eight pairs splits the exponentials
// between the two pipes so that neither bounds the step before the tensor core.
#ifndef H3A_POLY_PAIRS
#define H3A_POLY_PAIRS 0x94u
#endif
constexpr uint32_t kPolyPairs = H3A_POLY_PAIRS;

__device__ void softmax_group(AttnSmem& sm, const AttnArgs& a, uint32_t tmem, int t, int b, int h, int qb,
                              const int32_t* list, volatile int* abort_flag) {
    const int lane = threadIdx.x & 31;
    const int quarter = (threadIdx.x >> 5) & 3;  // TMEM lanes [32*quarter, 32*quarter + 32)
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tO = tmem + lane_addr + col_o(t);
    const float c = a.scale_log2;
    const uint64_t c2 = f2(c, c);
    const int nsub = 2 * a.n_iter;
    float m_used = -INFINITY;  // running max of scaled logits (log2 units) used for P
    uint64_t l2 = f2(0.f, 0.f);  // running sum of P, two partial lanes
    int kv = 0;
    bool ok = true;
    for (int u = 0; u < nsub; ++u) {
        const int hh = u & 1;
        const uint32_t tS = tmem + lane_addr + col_s(t, hh);
        // warp-uniform outcome: the tcgen05.ld/st below are warp-collective
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[t][hh], static_cast<uint32_t>((u >> 1) & 1), abort_flag,
                                               a.timeout_ns))) {
            ok = false;
            break;
        }
        tc_fence_after_sync();
        uint32_t s[2][32];
        tmem_ld_x32(tS + 0, s[0]);
        tmem_ld_x32(tS + 32, s[1]);
        tmem_wait_ld_x32(s[0]);
        tmem_wait_ld_x32(s[1]);

        if (hh == 0) kv = list ? __ldg(list + (u >> 1)) : (u >> 1);
        const int valid = (kv == a.nblk - 1) ? a.N - kv * 128 - kHalf * hh : kHalf;
        if (valid < kHalf) {
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2)
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (q2 * 32 + i >= valid) s[q2][i] = __float_as_uint(-INFINITY);
        }
        // row max: four independent chains of 3-input max
        float pm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2)
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
                pm[(i >> 3) & 3] = max3(pm[(i >> 3) & 3], __uint_as_float(s[q2][i]), __uint_as_float(s[q2][i + 1]));
                pm[(i >> 3) & 3] = max3(pm[(i >> 3) & 3], __uint_as_float(s[q2][i + 2]), __uint_as_float(s[q2][i + 3]));
                pm[(i >> 3) & 3] = max3(pm[(i >> 3) & 3], __uint_as_float(s[q2][i + 4]), __uint_as_float(s[q2][i + 5]));
                pm[(i >> 3) & 3] = max3(pm[(i >> 3) & 3], __uint_as_float(s[q2][i + 6]), __uint_as_float(s[q2][i + 7]));
            }
        const float mx = fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3]));
        const float m_new = fmaxf(m_used, mx * c);
        // A row whose max grew by more than 2^8 rescales: P uses the new max and
        // O is multiplied by alpha once PV of the previous half-step is done.
        float alpha = 1.0f;
        bool rescale_warp = false;
        if (u == 0) {
            m_used = m_new;
        } else {
            const bool need = m_new - m_used > 8.0f;
            rescale_warp = __any_sync(0xffffffffu, need);
            if (need) {
                alpha = ex2_approx(m_used - m_new);
                m_used = m_new;
            }
        }
        const uint64_t negm2 = f2(-m_used, -m_used);
        uint64_t ps = f2(0.f, 0.f);
        // P over the first 32 columns of this S buffer: keys 32q2..32q2+31 -> columns 16q2..16q2+15
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint64_t x = f2_fma(f2(__uint_as_float(s[q2][2 * i]), __uint_as_float(s[q2][2 * i + 1])), c2, negm2);
                uint64_t pp;
                if ((kPolyPairs >> (i & 7)) & 1u) {
                    pp = exp2_poly_pair(x);
                } else {
                    float x0, x1;
                    f2_split(x, x0, x1);
                    pp = f2(ex2_approx(x0), ex2_approx(x1));
                }
                ps = f2_add(ps, pp);
                float p0, p1;
                f2_split(pp, p0, p1);
                pk[i] = pack_bf16x2(p0, p1);
            }
            tmem_st_x16(tS + 16 * q2, pk);
        }
        if (rescale_warp) {
            float l0, l1;
            f2_split(l2, l0, l1);
            l2 = f2(l0 * alpha, l1 * alpha);
            // O_t must hold PV(u-1) before it is rescaled
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.pv_done[t], static_cast<uint32_t>((u - 1) & 1), abort_flag,
                                                   a.timeout_ns))) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
#pragma unroll
            for (int q3 = 0; q3 < 3; ++q3) {
                uint32_t o[32];
                tmem_ld_x32(tO + 32 * q3, o);
                tmem_wait_ld_x32(o);
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                tmem_st_x32(tO + 32 * q3, o);
            }
        }
        l2 = f2_add(l2, ps);
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(&sm.p_full[t][hh]);
    }
    if (!ok) {
        raise_timeout(a, abort_flag);
        return;
    }
    if (!__all_sync(0xffffffffu, mbar_wait(&sm.o_done[t], 0u, abort_flag, a.timeout_ns))) {
        raise_timeout(a, abort_flag);
        return;
    }
    tc_fence_after_sync();
    float l0, l1;
    f2_split(l2, l0, l1);
    const float inv_l = 1.0f / (l0 + l1);
    const int n = qb * 128 + row;
    __nv_bfloat16* dst = a.o + static_cast<int64_t>(b) * a.sb + static_cast<int64_t>(n) * a.sn +
                         static_cast<int64_t>(h) * a.sh;
#pragma unroll
    for (int q3 = 0; q3 < 3; ++q3) {
        uint32_t o[32];
        tmem_ld_x32(tO + 32 * q3, o);
        tmem_wait_ld_x32(o);
        if (n < a.N) {
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
            uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * q3);
#pragma unroll
            for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const AttnArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = smem_u32(smem_raw);
    AttnSmem& sm = *reinterpret_cast<AttnSmem*>(smem_raw + (((base + 1023u) & ~1023u) - base));

    const int warp = threadIdx.x >> 5;
    const int pair = blockIdx.x % a.npairs;
    const int bh = blockIdx.x / a.npairs;
    const int b = bh / a.heads, h = bh % a.heads;
    const int qb0 = 2 * pair;
    const bool has1 = qb0 + 1 < a.nblk;
    const int32_t* l0 = a.blocks ? a.blocks + (static_cast<int64_t>(bh) * a.nblk + qb0) * a.n_iter : nullptr;
    const int32_t* l1 = (a.blocks && has1) ? l0 + a.n_iter : nullptr;

    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(&sm.q_full[t], 1);
            for (int hh = 0; hh < 2; ++hh) {
                mbar_init(&sm.s_full[t][hh], 1);
                mbar_init(&sm.p_full[t][hh], 128);
            }
            mbar_init(&sm.pv_done[t], 1);
            mbar_init(&sm.o_done[t], 1);
        }
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.k_full[s], 1);
            mbar_init(&sm.k_empty[s], 1);
            mbar_init(&sm.v_full[s], 1);
            mbar_init(&sm.v_empty[s], 1);
        }
        mbar_init(&sm.mma_drain, 1);
        sm.abort_flag = 0;
        sm.never = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = sm.tmem_base;
    volatile int* abort_flag = &sm.abort_flag;

    if (warp == 0) {
        if ((threadIdx.x & 31) == 0) producer(sm, a, &tq, &tk, &tv, b, h, qb0, has1, l0, l1, abort_flag);
    } else if (warp == 1) {
        if ((threadIdx.x & 31) == 0) mma_issuer(sm, a, tmem, has1, l0, l1, abort_flag);
    } else if (warp >= 4 && warp < 8) {
        softmax_group(sm, a, tmem, 0, b, h, qb0, l0, abort_flag);
    } else if (warp >= 8 && has1) {
        softmax_group(sm, a, tmem, 1, b, h, qb0 + 1, l1, abort_flag);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

cudaError_t launch_attention(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* o,
                             const Shape& s, const int32_t* blocks, int k_blocks, float scale, int* status,
                             uint64_t timeout_ns, cudaStream_t st) {
    AttnArgs a;
    a.o = static_cast<__nv_bfloat16*>(o);
    a.blocks = blocks;
    a.N = s.N;
    a.heads = s.heads;
    a.nblk = (s.N + kBlock - 1) / kBlock;
    a.npairs = (a.nblk + 1) / 2;
    a.n_iter = blocks ? k_blocks : a.nblk;
    a.sb = s.sb;
    a.sn = s.sn;
    a.sh = s.sh;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.status = status;
    a.timeout_ns = timeout_ns;
    cudaError_t e = cudaFuncSetAttribute(attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    const int64_t grid = static_cast<int64_t>(s.B) * s.heads * a.npairs;
    attention_kernel<<<static_cast<unsigned>(grid), kThreads, kSmemBytes, st>>>(tq, tk, tv, a);
    return cudaGetLastError();
}

}  // namespace h3a
