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
// loaded once and shared).  Warp roles (384 threads, 12 warps):
//   warps 0-7   softmax: warpgroup t = warp / 4 handles query tile t; thread r
//               owns row r (TMEM lane r) and all 128 key columns of every
//               block, so the row max and row sum never leave the thread.  It
//               loads the row of S from TMEM in two 64-column halves, taking
//               the first half's max while the second half loads, then the
//               block max, computes exp2 in fp32 (log2 domain, packed f32x2
//               FMAs and adds) against the row's reference max and packs P to
//               bf16 in place over the same registers.  The reference is fixed
//               by the first block; a later block moves it up and rescales O
//               (in TMEM) only when the row max grew by more than 2^8 (the
//               final division by the row sum keeps this exact).  At the end
//               the thread divides its O row by the row sum, rounds once to
//               bf16 and stores it.
//   warp 8      TMA producer: Q tiles once, then a K ring and a V ring
//               (64-byte swizzled 128 x 32 chunks, D/32 per 128 x D tile).
//   warp 9      owns tensor memory (512 columns) and issues S_t = Q_t K^T
//               (M=128, N=128, K=D as D/16 steps of 16) into TMEM.
//   warp 10     (head_dim 96) issues O_t += P_t V (M=128, N=D, K=128 as 8
//               steps, P read from TMEM, V as an MN-major operand).
//   warp 11     idle: it completes the third warpgroup, whose registers
//               (setmaxnreg) go to the softmax warpgroups (200 each).
// Head_dim 96 (TMEM: S_0 [0,128), S_1 [128,256), O_0 [256,352), O_1
// [352,448), P [448,512)): P goes to its own 64-column buffer, which the two
// tiles take in turn, so S_t is released as soon as the softmax has read it
// and QK_t(j+1) runs during the exponentials of block j; QK and PV have
// separate issuing threads (warps 9 and 10), since they touch disjoint TMEM
// and one thread's barrier latency would otherwise hold up the other's MMAs.
// Head_dim 128 (O_0 [256,384), O_1 [384,512): no columns left): P_t is
// written over S_t, 16 columns at a time, and warp 9 issues both MMAs in the
// order PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1), so each softmax group waits
// only on its own tile's chain; four 32-channel chunks per tile, 2-stage
// rings.  Every mbarrier wait is bounded (timeout + CTA abort flag); a timeout
// sets the device status word instead of hanging or trapping.
#include <cuda_bf16.h>

#include "h3a_internal.h"
#include "fastmath.cuh"
#include "sm100.cuh"

namespace h3a {
namespace {

constexpr int kSoftmaxWarps = 8;                   // 2 warpgroups: one per query tile
constexpr int kProducerWarp = 8, kMmaWarp = 9, kPvWarp = 10;
constexpr int kThreads = 32 * (kSoftmaxWarps + 4);  // 384: a full third warpgroup (warp 11 idle)
// Register split (setmaxnreg, per warpgroup): the launch gives every thread
// 168 registers (65,536 / 384 rounded down to 8); the third warpgroup
// (producer, MMA issuers, an idle warp) drops to 80 and the two softmax
// warpgroups rise to 200, so a softmax thread holds its 128-value row without
// spilling.  The new total must fit in what the block was launched with.
constexpr uint32_t kRegsLaunch = (65536 / kThreads) / 8 * 8;
constexpr uint32_t kRegsSoftmax = 200, kRegsOther = 80;
static_assert(kSoftmaxWarps * 32 * kRegsSoftmax + 128 * kRegsOther <= kThreads * kRegsLaunch, "register split");
constexpr int kChunkBytes = 128 * 64;        // 128 rows x 32 bf16, 64-byte swizzle
constexpr uint32_t kTmemCols = 512;
// TMEM column of S_t
__host__ __device__ constexpr uint32_t col_s(int t) { return t ? 128u : 0u; }
constexpr uint32_t kSwizzle64 = 4;

// Geometry per head dimension D (96, or 128 -- SubBlock's stated head size):
// a 128-row tile is D/32 swizzled 32-channel chunks; O_t takes D TMEM columns
// (O_0 [256, 256+D), O_1 [256+D, 256+2D)); at D = 128 the K and V rings keep
// two stages each so that Q tiles and rings fit in 227 KB of shared memory.
template <int D>
struct Geo {
    static_assert(D == 96 || D == 128, "head_dim 96 or 128");
    static constexpr int kChunks = D / 32;
    static constexpr int kTileBytes = kChunks * kChunkBytes;
    static constexpr int kStages = D == 96 ? 3 : 2;
    static constexpr int kKSteps = D / 16;  // QK^T k-steps of 16
    __host__ __device__ static constexpr uint32_t col_o(int t) { return 256u + (t ? D : 0); }
    // At D = 96 the 64 columns after O_1 hold one bf16 P buffer that both
    // tiles take in turn, so S_t is free as soon as its softmax has read it
    // and QK_t(j+1) runs during the exponentials of block j.  At D = 128 no
    // columns are left: P_t is written over S_t and QK_t(j+1) follows PV_t(j).
    static constexpr bool kSepP = D == 96;
    static constexpr uint32_t kColP = 256u + 2 * D;
    static_assert(!kSepP || kColP + 64 <= kTmemCols, "P buffer inside the allocation");
};

template <int D>
struct AttnSmem {
    static constexpr int kStages = Geo<D>::kStages;
    static constexpr int kTileBytes = Geo<D>::kTileBytes;
    uint8_t q[2][kTileBytes];
    uint8_t k[kStages][kTileBytes];
    uint8_t v[kStages][kTileBytes];
    uint64_t q_full[2];
    uint64_t k_full[kStages], k_empty[kStages];
    uint64_t v_full[kStages], v_empty[kStages];
    uint64_t s_full[2], p_full[2], o_done[2];
    uint64_t s_read[2];   // separate-P scheme: S_t has been read into registers
    uint64_t pv_done[2];  // separate-P scheme: PV_t(j) has completed (P buffer free)
    uint64_t mma_drain, pv_drain;
    uint32_t tmem_base;
    int abort_flag;
    int never;  // stays 0: abort flag for waits that must ignore an abort
};

template <int D>
constexpr size_t smem_bytes() { return sizeof(AttnSmem<D>) + 1024; }  // + alignment slack

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

// Shared-memory descriptors are built once per buffer; a k-step or a ring
// stage only moves the start address, i.e. adds a constant (in 16-byte units)
// to the low field (addresses stay below 2^18, so the 14-bit field never
// carries).  This keeps the single MMA-issuing thread at a few instructions
// per tcgen05.mma -- computing descriptors per MMA made the issue thread,
// not the tensor core, the bottleneck.
//
// K-major 128 x D tile (D/32 swizzled 32-column chunks of 64-byte rows):
// k-step s covers columns [16s, 16s + 16).
__device__ __forceinline__ uint64_t kmajor_base(const uint8_t* tile) {
    return smem_desc(smem_u32(tile), 16, 512, kSwizzle64);
}
__host__ __device__ constexpr uint32_t kmajor_step(int s) {
    return static_cast<uint32_t>(((s >> 1) * kChunkBytes + (s & 1) * 32) >> 4);
}

// The same [128 kv rows x D] tile read as an MN-major operand (N = D along
// the contiguous dimension, K = kv rows): k-step s covers rows [16s, 16s + 16).
__device__ __forceinline__ uint64_t mnmajor_base(const uint8_t* tile) {
    return smem_desc(smem_u32(tile), kChunkBytes, 512, kSwizzle64);
}
__host__ __device__ constexpr uint32_t mnmajor_step(int s) { return static_cast<uint32_t>((s * 16 * 64) >> 4); }

template <int D>
constexpr uint32_t stage_step() { return Geo<D>::kTileBytes >> 4; }  // descriptor distance between ring stages

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

template <int D>
__device__ void producer(AttnSmem<D>& sm, const AttnArgs& a, const CUtensorMap* tq, const CUtensorMap* tk,
                         const CUtensorMap* tv, int b, int h, int qb0, bool has1, const int32_t* l0,
                         const int32_t* l1, volatile int* abort_flag) {
    prefetch_tensor_map(tq);
    prefetch_tensor_map(tk);
    prefetch_tensor_map(tv);
    const int ntiles = has1 ? 2 : 1;
    for (int t = 0; t < ntiles; ++t) {
        mbar_arrive_expect_tx(&sm.q_full[t], Geo<D>::kTileBytes);
        for (int c = 0; c < Geo<D>::kChunks; ++c)
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
            mbar_arrive_expect_tx(&sm.k_full[ks], Geo<D>::kTileBytes);
            for (int c = 0; c < Geo<D>::kChunks; ++c)
                tma_load_4d(sm.k[ks] + c * kChunkBytes, tk, &sm.k_full[ks], 32 * c, h, kv * 128, b);
            k_issued |= 1u << ks;
            k_par = (k_par & ~(1u << ks)) | (kph << ks);
            if (++ks == Geo<D>::kStages) {
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
            mbar_arrive_expect_tx(&sm.v_full[vs], Geo<D>::kTileBytes);
            for (int c = 0; c < Geo<D>::kChunks; ++c)
                tma_load_4d(sm.v[vs] + c * kChunkBytes, tv, &sm.v_full[vs], 32 * c, h, kv * 128, b);
            v_issued |= 1u << vs;
            v_par = (v_par & ~(1u << vs)) | (vph << vs);
            if (++vs == Geo<D>::kStages) {
                vs = 0;
                vph ^= 1u;
            }
        }
    }
    if (!ok) raise_timeout(a, abort_flag);
    // Drain: every load issued must have landed before the CTA may exit.
    volatile int* never = &sm.never;
    for (int t = 0; t < ntiles; ++t) mbar_wait(&sm.q_full[t], 0u, never, a.timeout_ns);
    for (int s = 0; s < Geo<D>::kStages; ++s) {
        if ((k_issued >> s) & 1u) mbar_wait(&sm.k_full[s], (k_par >> s) & 1u, never, a.timeout_ns);
        if ((v_issued >> s) & 1u) mbar_wait(&sm.v_full[s], (v_par >> s) & 1u, never, a.timeout_ns);
    }
}

struct MmaState {
    uint32_t ks = 0, kph = 0, vs = 0, vph = 0;
    uint32_t k_stage_t0 = 0, v_stage_t0 = 0;
    uint64_t dq[2], dk, dv;  // base descriptors: Q tiles, K stage 0, V stage 0
};

template <int D>
__device__ __forceinline__ bool issue_qk(AttnSmem<D>& sm, const AttnArgs& a, MmaState& st, uint32_t tmem, int t,
                                         const KvPlan& p, volatile int* abort_flag) {
    uint32_t stage;
    if (t == 0 || !p.shared) {
        if (!mbar_wait(&sm.k_full[st.ks], st.kph, abort_flag, a.timeout_ns)) return false;
        stage = st.ks;
        if (++st.ks == Geo<D>::kStages) {
            st.ks = 0;
            st.kph ^= 1u;
        }
    } else {
        stage = st.k_stage_t0;
    }
    if (t == 0) st.k_stage_t0 = stage;
    tc_fence_after_sync();
    constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
    const uint64_t dq = st.dq[t];
    const uint64_t dk = st.dk + stage * stage_step<D>();
    const uint32_t d = tmem + col_s(t);
#pragma unroll
    for (int s = 0; s < Geo<D>::kKSteps; ++s) mma_ss(d, dq + kmajor_step(s), dk + kmajor_step(s), idesc, s > 0 ? 1u : 0u);
    tc_commit(&sm.s_full[t]);
    if (t == 1 || !p.shared) tc_commit(&sm.k_empty[stage]);
    return true;
}

template <int D>
__device__ __forceinline__ bool issue_pv(AttnSmem<D>& sm, const AttnArgs& a, MmaState& st, uint32_t tmem, int t,
                                         const KvPlan& p, bool first, volatile int* abort_flag) {
    uint32_t stage;
    if (t == 0 || !p.shared) {
        if (!mbar_wait(&sm.v_full[st.vs], st.vph, abort_flag, a.timeout_ns)) return false;
        stage = st.vs;
        if (++st.vs == Geo<D>::kStages) {
            st.vs = 0;
            st.vph ^= 1u;
        }
    } else {
        stage = st.v_stage_t0;
    }
    if (t == 0) st.v_stage_t0 = stage;
    tc_fence_after_sync();
    constexpr uint32_t idesc = idesc_bf16_f32(128, D, 0, 1);
    const uint64_t dv = st.dv + stage * stage_step<D>();
    const uint32_t d = tmem + Geo<D>::col_o(t), pa = tmem + (Geo<D>::kSepP ? Geo<D>::kColP : col_s(t));
    // P_t: keys 2c and 2c+1 packed in column c of the P buffer (or of S_t)
    mma_ts(d, pa, dv, idesc, first ? 0u : 1u);
#pragma unroll
    for (int s = 1; s < 8; ++s) mma_ts(d, pa + 8 * s, dv + mnmajor_step(s), idesc, 1u);
    if (t == 1 || !p.shared) tc_commit(&sm.v_empty[stage]);
    return true;
}

// Separate-P scheme: two issuing threads.  QK^T and PV touch disjoint TMEM
// (S_t, versus the P buffer and O_t) and their hand-offs are separate
// barriers, so the QK issuer (warp 9) and the PV issuer (warp 10) run
// independently and neither's barrier latency holds up the other's MMAs.
// QK_t(j+1) may be issued as soon as the softmax has read S_t(j) (s_read);
// PV_t(j) as soon as P_t(j) is in the P buffer (p_full).
template <int D>
__device__ void qk_issuer(AttnSmem<D>& sm, const AttnArgs& a, uint32_t tmem, bool has1, const int32_t* l0,
                          const int32_t* l1, volatile int* abort_flag) {
    const int ntiles = has1 ? 2 : 1;
    MmaState st;
    st.dq[0] = kmajor_base(sm.q[0]);
    st.dq[1] = kmajor_base(sm.q[1]);
    st.dk = kmajor_base(sm.k[0]);
    bool ok = true;
    for (int t = 0; t < ntiles && ok; ++t) ok = mbar_wait(&sm.q_full[t], 0u, abort_flag, a.timeout_ns);
    KvPlan p = kv_plan(l0, l1, has1, 0);
    for (int t = 0; t < ntiles && ok; ++t) ok = issue_qk<D>(sm, a, st, tmem, t, p, abort_flag);
    for (int j = 0; j + 1 < a.n_iter && ok; ++j) {
        p = kv_plan(l0, l1, has1, j + 1);
        for (int t = 0; t < ntiles && ok; ++t) {
            if (!mbar_wait(&sm.s_read[t], static_cast<uint32_t>(j & 1), abort_flag, a.timeout_ns)) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            ok = issue_qk<D>(sm, a, st, tmem, t, p, abort_flag);
        }
    }
    if (!ok) raise_timeout(a, abort_flag);
    // Drain: every MMA this thread issued must have completed before TMEM is released.
    tc_commit(&sm.mma_drain);
    mbar_wait(&sm.mma_drain, 0u, &sm.never, a.timeout_ns);
}

template <int D>
__device__ void pv_issuer(AttnSmem<D>& sm, const AttnArgs& a, uint32_t tmem, bool has1, const int32_t* l0,
                          const int32_t* l1, volatile int* abort_flag) {
    const int ntiles = has1 ? 2 : 1;
    MmaState st;
    st.dv = mnmajor_base(sm.v[0]);
    bool ok = true;
    for (int j = 0; j < a.n_iter && ok; ++j) {
        const KvPlan p = kv_plan(l0, l1, has1, j);
        for (int t = 0; t < ntiles && ok; ++t) {
            if (!mbar_wait(&sm.p_full[t], static_cast<uint32_t>(j & 1), abort_flag, a.timeout_ns)) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            if (!issue_pv<D>(sm, a, st, tmem, t, p, j == 0, abort_flag)) {
                ok = false;
                break;
            }
            tc_commit(&sm.pv_done[t]);
            if (j + 1 == a.n_iter) tc_commit(&sm.o_done[t]);
        }
    }
    if (!ok) raise_timeout(a, abort_flag);
    tc_commit(&sm.pv_drain);
    mbar_wait(&sm.pv_drain, 0u, &sm.never, a.timeout_ns);
}

// P-over-S scheme: one issuing thread, PV_t(j) then QK_t(j+1) per tile (the
// QK overwrites the S/P columns the PV reads; MMAs from one thread complete
// in issue order).
template <int D>
__device__ void mma_issuer(AttnSmem<D>& sm, const AttnArgs& a, uint32_t tmem, bool has1, const int32_t* l0,
                           const int32_t* l1, volatile int* abort_flag) {
    const int ntiles = has1 ? 2 : 1;
    MmaState st;
    st.dq[0] = kmajor_base(sm.q[0]);
    st.dq[1] = kmajor_base(sm.q[1]);
    st.dk = kmajor_base(sm.k[0]);
    st.dv = mnmajor_base(sm.v[0]);
    bool ok = true;
    for (int t = 0; t < ntiles && ok; ++t) ok = mbar_wait(&sm.q_full[t], 0u, abort_flag, a.timeout_ns);
    // block lists are read one step ahead so their load latency stays off the issue path
    KvPlan p = kv_plan(l0, l1, has1, 0);
    KvPlan pn = a.n_iter > 1 ? kv_plan(l0, l1, has1, 1) : p;
    if (ok)
        for (int t = 0; t < ntiles && ok; ++t) ok = issue_qk<D>(sm, a, st, tmem, t, p, abort_flag);
    for (int j = 0; j < a.n_iter && ok; ++j) {
        const bool more = j + 1 < a.n_iter;
        const KvPlan pnn = (j + 2 < a.n_iter) ? kv_plan(l0, l1, has1, j + 2) : pn;
        for (int t = 0; t < ntiles && ok; ++t) {
            if (!mbar_wait(&sm.p_full[t], static_cast<uint32_t>(j & 1), abort_flag, a.timeout_ns)) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            if (!issue_pv<D>(sm, a, st, tmem, t, p, j == 0, abort_flag)) {
                ok = false;
                break;
            }
            if (more) {
                if (!issue_qk<D>(sm, a, st, tmem, t, pn, abort_flag)) ok = false;
            } else {
                tc_commit(&sm.o_done[t]);
            }
        }
        p = pn;
        pn = pnn;
    }
    if (!ok) raise_timeout(a, abort_flag);
    // Drain: every MMA issued must have completed before TMEM is released.
    tc_commit(&sm.mma_drain);
    volatile int* never = &sm.never;
    mbar_wait(&sm.mma_drain, 0u, never, a.timeout_ns);
}

// tcgen05.ld of 32 columns into / wait on a 32-register slice of a longer row.
__device__ __forceinline__ uint32_t (&slice32(uint32_t* x))[32] { return *reinterpret_cast<uint32_t(*)[32]>(x); }
__device__ __forceinline__ uint32_t (&slice16(uint32_t* x))[16] { return *reinterpret_cast<uint32_t(*)[16]>(x); }

// O row *= alpha (rare rescale).  Out of line: it runs only when a row max
// grows by more than 2^8, and its registers stay out of the steady-state loop.
template <int D>
__device__ __noinline__ void rescale_o(uint32_t tO, float alpha) {
#pragma unroll 1
    for (int cc = 0; cc < Geo<D>::kChunks; ++cc) {
        uint32_t o[32];
        tmem_ld_x32(tO + 32u * cc, o);
        tmem_wait_ld_x32(o);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
        tmem_st_x32(tO + 32u * cc, o);
    }
}

// Softmax of query tile t: thread r owns row r (TMEM lane r), all 128 keys.
template <int D>
__device__ void softmax_group(AttnSmem<D>& sm, const AttnArgs& a, uint32_t tmem, int t, bool has1, int b, int h,
                              int qb, const int32_t* list, volatile int* abort_flag) {
    constexpr bool kSep = Geo<D>::kSepP;
    const int lane = threadIdx.x & 31;
    const int quarter = (threadIdx.x >> 5) & 3;  // TMEM lanes [32*quarter, 32*quarter + 32)
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_addr + col_s(t);
    const uint32_t tO = tmem + lane_addr + Geo<D>::col_o(t);
    const uint32_t tP = tmem + lane_addr + Geo<D>::kColP;
    // Separate-P scheme: before this tile writes the shared P buffer at step j,
    // the PV that last read it must have completed -- the other tile's PV of
    // step j-1 (tile 0) or of step j (tile 1), or this tile's own PV of step
    // j-1 when the CTA has one tile.  That PV was issued after PV_t(j-1), so
    // its completion also leaves O_t stable for a rescale.  The wait names a
    // phase at most one ahead of the barrier's last completed one (the next
    // phase needs this tile's own P), so a parity wait is exact.
    auto wait_p_buffer = [&](int j) -> bool {
        const int u = has1 ? 1 - t : 0;
        const int ph = (has1 && t == 1) ? j : j - 1;
        if (ph < 0) return true;
        const bool r = __all_sync(0xffffffffu, mbar_wait(&sm.pv_done[u], static_cast<uint32_t>(ph & 1), abort_flag,
                                                         a.timeout_ns));
        if (r) tc_fence_after_sync();
        return r;
    };
    const float c = a.scale_log2;
    float m_used = -INFINITY;  // row reference max of scaled logits (log2 units)
    float l = 0.f;             // running row sum of P
    bool ok = true;
    for (int j = 0; j < a.n_iter; ++j) {
        // warp-uniform outcome: the tcgen05.ld/st below are warp-collective
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[t], static_cast<uint32_t>(j & 1), abort_flag, a.timeout_ns))) {
            ok = false;
            break;
        }
        tc_fence_after_sync();
        const int kv = list ? __ldg(list + j) : j;
        const int valid = (kv == a.nblk - 1) ? a.N - kv * 128 : 128;
        // the whole row of S in registers, the true block max before any
        // exponential, P packed in place over the same registers
        uint32_t x[128];
        float pm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int q = 0; q < 2; ++q) tmem_ld_x32(tS + 32u * q, slice32(x + 32 * q));
#pragma unroll
        for (int q = 0; q < 2; ++q) tmem_wait_ld_x32(slice32(x + 32 * q));
#pragma unroll
        for (int q = 2; q < 4; ++q) tmem_ld_x32(tS + 32u * q, slice32(x + 32 * q));
        // first half's max while the second half loads
        if (valid < 64) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
                if (i >= valid) x[i] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i)
            pm[i & 3] = max3(pm[i & 3], __uint_as_float(x[2 * i]), __uint_as_float(x[2 * i + 1]));
#pragma unroll
        for (int q = 2; q < 4; ++q) tmem_wait_ld_x32(slice32(x + 32 * q));
        if constexpr (kSep) {
            // S_t is in registers: release it for QK_t(j+1)
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.s_read[t]);
        }
        bool p_free = false;  // separate-P scheme: the P buffer wait is done
        if (valid < 128) {
#pragma unroll
            for (int i = 64; i < 128; ++i)
                if (i >= valid) x[i] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int i = 32; i < 64; ++i)
            pm[i & 3] = max3(pm[i & 3], __uint_as_float(x[2 * i]), __uint_as_float(x[2 * i + 1]));
        const float mx = c * fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3]));
        if (j == 0) {
            m_used = mx;  // the first block fixes the reference
        } else {
            const bool need = mx - m_used > 8.0f;
            if (__any_sync(0xffffffffu, need)) {
                // rare: O_t must be stable -- with P over S the commit behind
                // s_full covers PV_t(j-1); with a separate P buffer, its wait does
                if constexpr (kSep) {
                    if (!wait_p_buffer(j)) {
                        ok = false;
                        break;
                    }
                    p_free = true;
                }
                float alpha = 1.0f;
                if (need) {
                    alpha = ex2_approx(m_used - mx);
                    m_used = mx;
                }
                l *= alpha;
                rescale_o<D>(tO, alpha);
            }
        }
        const uint64_t c2 = f2(c, c), nm2 = f2(-m_used, -m_used);
        uint64_t acc[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            float a0, a1;
            f2_split(f2_fma(f2(__uint_as_float(x[2 * i]), __uint_as_float(x[2 * i + 1])), c2, nm2), a0, a1);
            const float p0 = ex2_approx(a0), p1 = ex2_approx(a1);
            acc[i & 1] = f2_add(acc[i & 1], f2(p0, p1));
            x[i] = pack_bf16x2(p0, p1);  // i < 2i: the S values read here are never needed again
            // P over S: each 16-column chunk is stored as soon as it is
            // complete (over S columns already read)
            if constexpr (!kSep)
                if ((i & 15) == 15) tmem_st_x16(tS + (i - 15), slice16(x + (i - 15)));
        }
        if constexpr (kSep) {
            if (!p_free && !wait_p_buffer(j)) {
                ok = false;
                break;
            }
            tmem_st_x32(tP, slice32(x));
            tmem_st_x32(tP + 32u, slice32(x + 32));
        }
        float s0, s1, s2, s3;
        f2_split(acc[0], s0, s1);
        f2_split(acc[1], s2, s3);
        l += (s0 + s1) + (s2 + s3);
        // one arrival per warp: every lane's TMEM stores are complete and
        // fenced before the warp converges and lane 0 releases the barrier
        tmem_wait_st();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full[t]);
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
    const float inv_l = 1.0f / l;
    const int n = qb * 128 + row;
    __nv_bfloat16* dst = a.o + static_cast<int64_t>(b) * a.sb + static_cast<int64_t>(n) * a.sn +
                         static_cast<int64_t>(h) * a.sh;
#pragma unroll
    for (int cc = 0; cc < Geo<D>::kChunks; ++cc) {
        uint32_t o[32];
        tmem_ld_x32(tO + 32u * cc, o);
        tmem_wait_ld_x32(o);
        if (n < a.N) {
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
            uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * cc);
#pragma unroll
            for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const AttnArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = smem_u32(smem_raw);
    AttnSmem<D>& sm = *reinterpret_cast<AttnSmem<D>*>(smem_raw + (((base + 1023u) & ~1023u) - base));

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
            mbar_init(&sm.s_full[t], 1);
            mbar_init(&sm.p_full[t], 4);  // one arrival per softmax warp of the tile
            mbar_init(&sm.o_done[t], 1);
            mbar_init(&sm.s_read[t], 4);  // one arrival per softmax warp of the tile
            mbar_init(&sm.pv_done[t], 1);
        }
        for (int s = 0; s < Geo<D>::kStages; ++s) {
            mbar_init(&sm.k_full[s], 1);
            mbar_init(&sm.k_empty[s], 1);
            mbar_init(&sm.v_full[s], 1);
            mbar_init(&sm.v_empty[s], 1);
        }
        mbar_init(&sm.mma_drain, 1);
        mbar_init(&sm.pv_drain, 1);
        sm.abort_flag = 0;
        sm.never = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = sm.tmem_base;
    volatile int* abort_flag = &sm.abort_flag;

    if (warp < kSoftmaxWarps) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
        const int t = warp >> 2;  // softmax warpgroup = query tile
        if (t == 0 || has1) softmax_group<D>(sm, a, tmem, t, has1, b, h, qb0 + t, t ? l1 : l0, abort_flag);
    } else {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
        if (warp == kProducerWarp) {
            if ((threadIdx.x & 31) == 0) producer<D>(sm, a, &tq, &tk, &tv, b, h, qb0, has1, l0, l1, abort_flag);
        } else if (warp == kMmaWarp) {
            if ((threadIdx.x & 31) == 0) {
                if constexpr (Geo<D>::kSepP)
                    qk_issuer<D>(sm, a, tmem, has1, l0, l1, abort_flag);
                else
                    mma_issuer<D>(sm, a, tmem, has1, l0, l1, abort_flag);
            }
        } else if (warp == kPvWarp) {
            if constexpr (Geo<D>::kSepP)
                if ((threadIdx.x & 31) == 0) pv_issuer<D>(sm, a, tmem, has1, l0, l1, abort_flag);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D>
cudaError_t run(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a, int64_t grid,
                cudaStream_t st) {
    constexpr size_t smem = smem_bytes<D>();
    static_assert(smem <= 232448, "shared memory per CTA");
    cudaError_t e = cudaFuncSetAttribute(attention_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attention_kernel<D><<<static_cast<unsigned>(grid), kThreads, smem, st>>>(tq, tk, tv, a);
    return cudaGetLastError();
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
    const int64_t grid = static_cast<int64_t>(s.B) * s.heads * a.npairs;
    if (s.d == 128) return run<128>(tq, tk, tv, a, grid, st);
    return run<96>(tq, tk, tv, a, grid, st);
}

}  // namespace h3a
