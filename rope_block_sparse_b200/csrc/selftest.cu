// Self-checks of the device building blocks (no counterpart on the pages):
//   wait_timeout_kernel  waits on a barrier nothing completes, with a short
//                        limit, and must report the timeout through the status
//                        word -- the same bounded wait every pipeline wait uses.
//   mma_selftest_kernel  one CTA runs the tensor-core steps of the attention
//                        kernel on a single tile: TMA loads of two 128 x 96 bf16
//                        tiles, S = A B^T into TMEM (K-major operands), bf16(S)
//                        written back to TMEM, R = bf16(S) B with B read as an
//                        MN-major operand and A taken from TMEM.
//   exp2_selftest_kernel evaluates the softmax's exponential (ex2.approx)
//                        element-wise, for checking it against 2^x.
#include "fastmath.cuh"
#include "h3a_internal.h"
#include "sm100.cuh"

namespace h3a {
namespace {

constexpr int kChunkBytes = 128 * 64;
constexpr int kTileBytes = 3 * kChunkBytes;

__global__ void wait_timeout_kernel(uint64_t limit_ns, int* status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // phase 0 of `bar` never completes: nobody arrives
        if (!mbar_wait(&bar, 0u, &abort_flag, limit_ns)) atomicOr(status, kDevTimeout);
    }
}

struct SelfSmem {
    uint8_t a[kTileBytes];
    uint8_t b[kTileBytes];
    uint64_t load_bar, mma_bar;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ uint64_t kdesc(const uint8_t* tile, int s) {
    return smem_desc(smem_u32(tile) + (s >> 1) * kChunkBytes + (s & 1) * 32, 16, 512, 4);
}

__device__ __forceinline__ uint64_t mndesc(const uint8_t* tile, int s) {
    return smem_desc(smem_u32(tile) + s * 16 * 64, kChunkBytes, 512, 4);
}

__global__ void __launch_bounds__(128, 1)
    mma_selftest_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb,
                        float* s_out, float* r_out, int* status, uint64_t timeout_ns) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = smem_u32(smem_raw);
    SelfSmem& sm = *reinterpret_cast<SelfSmem*>(smem_raw + (((base + 1023u) & ~1023u) - base));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(&sm.load_bar, 1);
        mbar_init(&sm.mma_bar, 1);
        sm.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = sm.tmem_base;
    volatile int* abort_flag = &sm.abort_flag;

    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&sm.load_bar, 2 * kTileBytes);
        for (int c = 0; c < 3; ++c) {
            tma_load_4d(sm.a + c * kChunkBytes, &ta, &sm.load_bar, 32 * c, 0, 0, 0);
            tma_load_4d(sm.b + c * kChunkBytes, &tb, &sm.load_bar, 32 * c, 0, 0, 0);
        }
        bool ok = mbar_wait(&sm.load_bar, 0u, abort_flag, timeout_ns);
        if (ok) {
            tc_fence_after_sync();
            constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
            for (int s = 0; s < 6; ++s) mma_ss(tmem, kdesc(sm.a, s), kdesc(sm.b, s), idesc, s > 0 ? 1u : 0u);
            tc_commit(&sm.mma_bar);
        } else {
            *abort_flag = 1;
            atomicOr(status, kDevTimeout);
        }
    }
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    const int row = warp * 32 + lane;
    bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.mma_bar, 0u, abort_flag, timeout_ns));
    if (ok) {
        tc_fence_after_sync();
        uint32_t p[2][32];
        for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t s[32];
            tmem_ld_x32(tmem + lane_addr + 32 * q4, s);
            tmem_wait_ld_x32(s);
            for (int i = 0; i < 32; ++i) s_out[row * 128 + 32 * q4 + i] = __uint_as_float(s[i]);
            for (int i = 0; i < 16; ++i)
                p[q4 >> 1][(q4 & 1) * 16 + i] = pack_bf16x2(__uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1]));
        }
        tmem_st_x32(tmem + lane_addr + 0, p[0]);
        tmem_st_x32(tmem + lane_addr + 32, p[1]);
        tmem_wait_st();
    }
    tc_fence_before_sync();
    __syncthreads();
    if (threadIdx.x == 0 && ok) {
        tc_fence_after_sync();
        constexpr uint32_t idesc = idesc_bf16_f32(128, 96, 0, 1);
        for (int s = 0; s < 8; ++s) mma_ts(tmem + 256, tmem + 8 * s, mndesc(sm.b, s), idesc, s > 0 ? 1u : 0u);
        tc_commit(&sm.mma_bar);
    }
    if (ok) {
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.mma_bar, 1u, abort_flag, timeout_ns));
        if (ok) {
            tc_fence_after_sync();
            for (int q3 = 0; q3 < 3; ++q3) {
                uint32_t r[32];
                tmem_ld_x32(tmem + lane_addr + 256 + 32 * q3, r);
                tmem_wait_ld_x32(r);
                for (int i = 0; i < 32; ++i) r_out[row * 96 + 32 * q3 + i] = __uint_as_float(r[i]);
            }
        } else if (lane == 0) {
            *abort_flag = 1;
            atomicOr(status, kDevTimeout);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

__global__ void exp2_selftest_kernel(const float* x, float* y, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) y[i] = ex2_approx(x[i]);
}

}  // namespace

cudaError_t launch_selftest_exp2(const float* x, float* y, int n, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    exp2_selftest_kernel<<<(n + 255) / 256, 256, 0, st>>>(x, y, n);
    return cudaGetLastError();
}

cudaError_t launch_selftest_wait(uint64_t limit_ns, int* status, cudaStream_t st) {
    wait_timeout_kernel<<<1, 32, 0, st>>>(limit_ns, status);
    return cudaGetLastError();
}

cudaError_t launch_selftest_mma(const CUtensorMap& ta, const CUtensorMap& tb, float* s_out, float* r_out,
                                int* status, uint64_t timeout_ns, cudaStream_t st) {
    const size_t smem = sizeof(SelfSmem) + 1024;
    cudaError_t e =
        cudaFuncSetAttribute(mma_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    mma_selftest_kernel<<<1, 128, smem, st>>>(ta, tb, s_out, r_out, status, timeout_ns);
    return cudaGetLastError();
}

}  // namespace h3a
