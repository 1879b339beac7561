// C-ABI front end of libh3a: argument validation, tensor-map encoding and
// launches on the caller's stream.  Nothing here allocates device memory; the
// only device state is the per-device status word below (and the copy of it
// that the last read took).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <string>

#include "h3a.h"
#include "h3a_internal.h"

// Sticky per-device status word: kernels OR error bits into it.
__device__ int g_h3a_status_word;
// What the last read of the status word took out of it.
__device__ int g_h3a_status_taken;

// Reads and clears the status word in one atomic step, so that an error a
// kernel on another stream ORs in at the same moment is either taken by this
// read or left for the next one -- never lost.
__global__ void status_take_kernel() { g_h3a_status_taken = atomicExch(&g_h3a_status_word, 0); }

namespace h3a {
namespace {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per pipeline wait
constexpr int kMaxDevices = 64;

thread_local std::string g_last_cuda_error;

h3a_status cuda_fail(cudaError_t e) {
    g_last_cuda_error = std::string(cudaGetErrorName(e)) + ": " + cudaGetErrorString(e);
    return H3A_ERR_CUDA;
}

// Device address of g_h3a_status_word, resolved once per device.
std::mutex g_status_mu;
// Serialises readers of g_h3a_status_taken (one per process at a time).
std::mutex g_take_mu;
int* g_status_ptr[kMaxDevices] = {};

h3a_status status_word(int** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return H3A_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_status_mu);
    if (g_status_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_h3a_status_word);
        if (e != cudaSuccess) return cuda_fail(e);
        g_status_ptr[dev] = static_cast<int*>(p);
    }
    *out = g_status_ptr[dev];
    return H3A_OK;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::once_flag g_encode_once;
EncodeTiledFn g_encode = nullptr;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validates a Q/K/V/O descriptor.  Fills `s` on success.  head_dim 96 for
// every call; the router and attention also take 128 (wide_ok).
h3a_status check_desc(const h3a_qkv_desc* d, Shape* s, bool wide_ok = false) {
    if (d == nullptr) return H3A_ERR_INVALID_ARG;
    if (d->head_dim != kHeadDim && !(wide_ok && d->head_dim == kHeadDimWide)) return H3A_ERR_UNSUPPORTED;
    if (d->B < 1 || d->N < 1 || d->heads < 1) return H3A_ERR_INVALID_ARG;
    if (d->stride_b < 0 || d->stride_n < 0 || d->stride_h < 0) return H3A_ERR_INVALID_ARG;
    if ((d->stride_b % 8) || (d->stride_n % 8) || (d->stride_h % 8)) return H3A_ERR_INVALID_ARG;
    if (d->heads > 1 && d->stride_h < d->head_dim) return H3A_ERR_INVALID_ARG;
    if (d->N > 1 && d->stride_n < d->head_dim) return H3A_ERR_INVALID_ARG;
    // byte strides must stay within the tensor-map limit (2^40)
    const int64_t lim = (int64_t(1) << 39);
    if (d->stride_b >= lim || d->stride_n >= lim || d->stride_h >= lim) return H3A_ERR_UNSUPPORTED;
    s->B = d->B;
    s->N = d->N;
    s->heads = d->heads;
    s->d = d->head_dim;
    s->sb = d->stride_b;
    s->sn = d->stride_n;
    s->sh = d->stride_h;
    return H3A_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Router workspace: the fp32 block means of Q, [B, heads, nblk, d], then those
// of K stored channel-major, [B, heads, d, pooled_k_stride(nblk)], each half
// starting on a 256-byte boundary.
size_t pooled_q_bytes(const Shape& s, int nblk) {
    return align256(static_cast<size_t>(s.B) * s.heads * nblk * s.d * sizeof(float));
}
size_t pooled_k_bytes(const Shape& s, int nblk) {
    return align256(static_cast<size_t>(s.B) * s.heads * s.d * pooled_k_stride(nblk) * sizeof(float));
}

}  // namespace

namespace {
// Tiled tensor map over a [B, N, heads, d] bf16 tensor (d contiguous) with the
// given box and swizzle; elements outside the tensor read as zero.
cudaError_t encode_qkv_map(CUtensorMap* map, const void* base, const Shape& s, const cuuint32_t (&box)[4],
                           CUtensorMapSwizzle swizzle) {
    std::call_once(g_encode_once, []() {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    });
    if (g_encode == nullptr) return cudaErrorNotSupported;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(s.d), static_cast<cuuint64_t>(s.heads),
                                static_cast<cuuint64_t>(s.N), static_cast<cuuint64_t>(s.B)};
    // byte strides of dims 1..3; a size-1 dim gets a nominal (unused) stride
    auto stride_or = [](int64_t st, int64_t fallback) { return static_cast<cuuint64_t>((st > 0 ? st : fallback) * 2); };
    const cuuint64_t strides[3] = {stride_or(s.sh, s.d), stride_or(s.sn, s.d), stride_or(s.sb, s.d)};
    const cuuint32_t elem_strides[4] = {1, 1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
                          elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}
}  // namespace

cudaError_t make_qkv_tensor_map(CUtensorMap* map, const void* base, const Shape& s) {
    const cuuint32_t box[4] = {32, 1, 128, 1};
    return encode_qkv_map(map, base, s, box, CU_TENSOR_MAP_SWIZZLE_64B);
}

cudaError_t make_head_slice_tensor_map(CUtensorMap* map, const void* base, const Shape& s) {
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(kHeadDim), static_cast<cuuint32_t>(kPrologueSliceHeads), 1, 1};
    return encode_qkv_map(map, base, s, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

}  // namespace h3a

using namespace h3a;

namespace {

// Shared checks of the router's shape, sparsity and workspace; on success
// fills nblk, k and the two pooled halves of the workspace.
h3a_status route_setup(const Shape& s, double sparsity, int32_t block, const void* workspace, size_t ws_bytes,
                       int* nblk, int64_t* kk, float** pq, float** pk) {
    if (block != kBlock) return H3A_ERR_UNSUPPORTED;
    if (!(sparsity >= 0.0 && sparsity < 1.0)) return H3A_ERR_INVALID_ARG;
    *nblk = (s.N + kBlock - 1) / kBlock;
    if (*nblk > route_max_blocks(s.d)) return H3A_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(s.B) * s.heads > 65535) return H3A_ERR_UNSUPPORTED;
    const size_t half = pooled_q_bytes(s, *nblk);
    if (workspace == nullptr || !aligned16(workspace) || ws_bytes < half + pooled_k_bytes(s, *nblk))
        return H3A_ERR_WORKSPACE;
    *kk = h3a_route_k(*nblk, sparsity);
    *pq = static_cast<float*>(const_cast<void*>(workspace));
    *pk = reinterpret_cast<float*>(static_cast<char*>(const_cast<void*>(workspace)) + half);
    return H3A_OK;
}

// Shared checks of the prologue's arguments.
h3a_status prologue_check(const void* q, const void* k, const h3a_qkv_desc* d, const float* gamma_q,
                          const float* gamma_k, h3a_grid grid, double theta, float eps, const void* q_out,
                          const void* k_out, Shape* s) {
    h3a_status rc = check_desc(d, s);
    if (rc != H3A_OK) return rc;
    if (!q || !k || !gamma_q || !gamma_k || !q_out || !k_out) return H3A_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(q_out) || !aligned16(k_out)) return H3A_ERR_INVALID_ARG;
    if (!(reinterpret_cast<uintptr_t>(gamma_q) % 4 == 0 && reinterpret_cast<uintptr_t>(gamma_k) % 4 == 0))
        return H3A_ERR_INVALID_ARG;
    if (grid.T < 1 || grid.H < 1 || grid.W < 1) return H3A_ERR_INVALID_ARG;
    if (static_cast<int64_t>(grid.T) * grid.H * grid.W != d->N) return H3A_ERR_INVALID_ARG;
    if (!(eps >= 0.0f) || !(theta > 0.0)) return H3A_ERR_INVALID_ARG;
    return H3A_OK;
}

}  // namespace

extern "C" {

const char* h3a_status_string(h3a_status s) {
    switch (s) {
        case H3A_OK: return "H3A_OK";
        case H3A_ERR_INVALID_ARG: return "H3A_ERR_INVALID_ARG";
        case H3A_ERR_UNSUPPORTED: return "H3A_ERR_UNSUPPORTED";
        case H3A_ERR_CUDA: return "H3A_ERR_CUDA";
        case H3A_ERR_TIMEOUT: return "H3A_ERR_TIMEOUT";
        case H3A_ERR_WORKSPACE: return "H3A_ERR_WORKSPACE";
    }
    return "H3A_ERR_UNKNOWN";
}

const char* h3a_last_cuda_error_string(void) { return g_last_cuda_error.c_str(); }

h3a_status h3a_qk_norm_rope(const void* q, const void* k, const h3a_qkv_desc* d, const float* gamma_q,
                            const float* gamma_k, h3a_grid grid, double theta, float eps, void* q_out, void* k_out,
                            h3a_stream_t stream) {
    Shape s;
    h3a_status rc = prologue_check(q, k, d, gamma_q, gamma_k, grid, theta, eps, q_out, k_out, &s);
    if (rc != H3A_OK) return rc;
    cudaError_t e = launch_qk_norm_rope(q, k, q_out, k_out, gamma_q, gamma_k, s, grid.T, grid.H, grid.W, theta, eps,
                                        reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? H3A_OK : cuda_fail(e);
}

double h3a_step_sparsity(int32_t step, int32_t first_sparse_step, double sparsity) {
    if (step < 1 || first_sparse_step < 1 || !(sparsity >= 0.0 && sparsity < 1.0)) return -1.0;
    return step >= first_sparse_step ? sparsity : 0.0;
}

h3a_status h3a_qk_fullnorm_rope(const void* q, const void* k, const h3a_qkv_desc* d, const float* gamma_q,
                                const float* gamma_k, h3a_grid grid, double theta, float eps, void* q_out,
                                void* k_out, h3a_stream_t stream) {
    Shape s;
    h3a_status rc = prologue_check(q, k, d, gamma_q, gamma_k, grid, theta, eps, q_out, k_out, &s);
    if (rc != H3A_OK) return rc;
    if (!aligned16(gamma_q) || !aligned16(gamma_k)) return H3A_ERR_INVALID_ARG;  // read as float4
    // one CTA per token, each holding its token's rows in registers
    if (s.heads > 74 || static_cast<int64_t>(s.B) * s.N >= (int64_t(1) << 31)) return H3A_ERR_UNSUPPORTED;
    cudaError_t e = launch_qk_fullnorm_rope(q, k, q_out, k_out, gamma_q, gamma_k, s, grid.H, grid.W, theta, eps,
                                            reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? H3A_OK : cuda_fail(e);
}

int64_t h3a_route_k(int64_t nkv, double sparsity) {
    if (nkv < 1 || !(sparsity >= 0.0 && sparsity < 1.0)) return -1;
    int64_t kk = static_cast<int64_t>(std::ceil((1.0 - sparsity) * static_cast<double>(nkv) - 1e-9));
    if (kk < 1) kk = 1;
    if (kk > nkv) kk = nkv;
    return kk;
}

h3a_status h3a_route_workspace_size(const h3a_qkv_desc* d, int32_t block, size_t* bytes) {
    Shape s;
    h3a_status rc = check_desc(d, &s, true);
    if (rc != H3A_OK) return rc;
    if (bytes == nullptr) return H3A_ERR_INVALID_ARG;
    if (block != kBlock) return H3A_ERR_UNSUPPORTED;
    const int nblk = (s.N + kBlock - 1) / kBlock;
    *bytes = pooled_q_bytes(s, nblk) + pooled_k_bytes(s, nblk);
    return H3A_OK;
}

h3a_status h3a_route(const void* q, const void* k, const h3a_qkv_desc* d, double sparsity, int32_t block,
                     int32_t* block_idx, int64_t* k_out, void* workspace, size_t ws_bytes, h3a_stream_t stream) {
    Shape s;
    h3a_status rc = check_desc(d, &s, true);
    if (rc != H3A_OK) return rc;
    if (block != kBlock) return H3A_ERR_UNSUPPORTED;
    if (!q || !k || !block_idx) return H3A_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || (reinterpret_cast<uintptr_t>(block_idx) & 3u)) return H3A_ERR_INVALID_ARG;
    int nblk;
    int64_t kk;
    float *pq, *pk;
    rc = route_setup(s, sparsity, block, workspace, ws_bytes, &nblk, &kk, &pq, &pk);
    if (rc != H3A_OK) return rc;
    if (k_out) *k_out = kk;
    cudaError_t e = launch_route(q, k, s, nblk, static_cast<int>(kk), pq, pk, block_idx,
                                 reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? H3A_OK : cuda_fail(e);
}

h3a_status h3a_qk_norm_rope_pool(const void* q, const void* k, const h3a_qkv_desc* d, const float* gamma_q,
                                 const float* gamma_k, h3a_grid grid, double theta, float eps, void* q_out,
                                 void* k_out, void* workspace, size_t ws_bytes, h3a_stream_t stream) {
    Shape s;
    h3a_status rc = prologue_check(q, k, d, gamma_q, gamma_k, grid, theta, eps, q_out, k_out, &s);
    if (rc != H3A_OK) return rc;
    const int nblk = (s.N + kBlock - 1) / kBlock;
    if (s.B > 65535 || (s.heads + kPrologueSliceHeads - 1) / kPrologueSliceHeads > 65535) return H3A_ERR_UNSUPPORTED;
    const size_t half = pooled_q_bytes(s, nblk);
    if (workspace == nullptr || !aligned16(workspace) || ws_bytes < half + pooled_k_bytes(s, nblk))
        return H3A_ERR_WORKSPACE;
    float* pq = static_cast<float*>(workspace);
    float* pk = reinterpret_cast<float*>(static_cast<char*>(workspace) + half);
    int* status = nullptr;
    rc = status_word(&status);
    if (rc != H3A_OK) return rc;
    CUtensorMap tq, tk;
    cudaError_t e = make_head_slice_tensor_map(&tq, q, s);
    if (e == cudaSuccess) e = make_head_slice_tensor_map(&tk, k, s);
    if (e != cudaSuccess) return cuda_fail(e);
    e = launch_qk_norm_rope_pool(tq, tk, q_out, k_out, gamma_q, gamma_k, s, grid.H, grid.W, theta, eps, pq, pk,
                                 status, kWaitLimitNs, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? H3A_OK : cuda_fail(e);
}

h3a_status h3a_route_pooled(const h3a_qkv_desc* d, double sparsity, int32_t block, int32_t* block_idx,
                            int64_t* k_out, const void* workspace, size_t ws_bytes, h3a_stream_t stream) {
    Shape s;
    h3a_status rc = check_desc(d, &s);
    if (rc != H3A_OK) return rc;
    if (!block_idx || (reinterpret_cast<uintptr_t>(block_idx) & 3u)) return H3A_ERR_INVALID_ARG;
    int nblk;
    int64_t kk;
    float *pq, *pk;
    rc = route_setup(s, sparsity, block, workspace, ws_bytes, &nblk, &kk, &pq, &pk);
    if (rc != H3A_OK) return rc;
    if (k_out) *k_out = kk;
    cudaError_t e = launch_route_scores(pq, pk, s, nblk, static_cast<int>(kk), block_idx,
                                        reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? H3A_OK : cuda_fail(e);
}

h3a_status h3a_attention(const void* q, const void* k, const void* v, const h3a_qkv_desc* d,
                         const int32_t* block_idx, int32_t k_blocks, int32_t block, float scale, void* o,
                         h3a_stream_t stream) {
    Shape s;
    h3a_status rc = check_desc(d, &s, true);
    if (rc != H3A_OK) return rc;
    if (block != kBlock) return H3A_ERR_UNSUPPORTED;
    if (!q || !k || !v || !o) return H3A_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return H3A_ERR_INVALID_ARG;
    if (!(scale >= 0.0f) || !std::isfinite(scale)) return H3A_ERR_INVALID_ARG;
    const int nblk = (s.N + kBlock - 1) / kBlock;
    if (block_idx != nullptr) {
        if ((reinterpret_cast<uintptr_t>(block_idx) & 3u) || k_blocks < 1 || k_blocks > nblk)
            return H3A_ERR_INVALID_ARG;
    }
    const int64_t grid = static_cast<int64_t>(s.B) * s.heads * ((nblk + 1) / 2);
    if (grid >= (int64_t(1) << 31)) return H3A_ERR_UNSUPPORTED;
    if (scale == 0.0f) scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(s.d)));
    int* status = nullptr;
    rc = status_word(&status);
    if (rc != H3A_OK) return rc;
    CUtensorMap tq, tk, tv;
    cudaError_t e = make_qkv_tensor_map(&tq, q, s);
    if (e == cudaSuccess) e = make_qkv_tensor_map(&tk, k, s);
    if (e == cudaSuccess) e = make_qkv_tensor_map(&tv, v, s);
    if (e != cudaSuccess) return cuda_fail(e);
    e = launch_attention(tq, tk, tv, o, s, block_idx, k_blocks, scale, status, kWaitLimitNs,
                         reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? H3A_OK : cuda_fail(e);
}

h3a_status h3a_residual_adaln(const void* x, const void* f, const float* gate, const float* shift,
                              const float* scale, int32_t B, int64_t rows, int32_t width, float eps, void* h_out,
                              void* y_out, h3a_stream_t stream) {
    if (B < 1 || rows < 0 || width < 8) return H3A_ERR_INVALID_ARG;
    if (width % 8) return H3A_ERR_INVALID_ARG;
    if (width > residual_adaln_max_width()) return H3A_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(B) * rows >= (int64_t(1) << 31)) return H3A_ERR_UNSUPPORTED;
    if (!x || !shift || !scale || !y_out) return H3A_ERR_INVALID_ARG;
    if (f && (!gate || !h_out)) return H3A_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(shift) || !aligned16(scale) || !aligned16(y_out)) return H3A_ERR_INVALID_ARG;
    if ((f && !aligned16(f)) || (gate && !aligned16(gate)) || (h_out && !aligned16(h_out)))
        return H3A_ERR_INVALID_ARG;
    if (!(eps >= 0.0f)) return H3A_ERR_INVALID_ARG;
    cudaError_t e = launch_residual_adaln(x, f, f ? gate : nullptr, shift, scale, B, rows, width, eps,
                                          f ? h_out : nullptr, y_out, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? H3A_OK : cuda_fail(e);
}

h3a_status h3a_swiglu(const void* in, int64_t rows, int32_t ffn_width, void* out, h3a_stream_t stream) {
    if (rows < 0 || ffn_width < 8 || (ffn_width % 8)) return H3A_ERR_INVALID_ARG;
    if (!in || !out || !aligned16(in) || !aligned16(out)) return H3A_ERR_INVALID_ARG;
    cudaError_t e = launch_swiglu(in, rows, ffn_width, out, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? H3A_OK : cuda_fail(e);
}

h3a_status h3a_residual_diff(const void* cur, const void* prev, int64_t n, double threshold, void* workspace,
                             size_t ws_bytes, double* rel_out, int32_t* reuse_out, h3a_stream_t stream) {
    if (n < 8 || (n % 8)) return H3A_ERR_INVALID_ARG;
    if (!cur || !prev || !rel_out || !aligned16(cur) || !aligned16(prev)) return H3A_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(rel_out) & 7u) || (reinterpret_cast<uintptr_t>(reuse_out) & 3u))
        return H3A_ERR_INVALID_ARG;
    if (!(threshold >= 0.0)) return H3A_ERR_INVALID_ARG;
    if (workspace == nullptr || !aligned16(workspace) || ws_bytes < residual_diff_workspace_bytes())
        return H3A_ERR_WORKSPACE;
    cudaError_t e = launch_residual_diff(cur, prev, n, threshold, workspace, rel_out, reuse_out,
                                         reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? H3A_OK : cuda_fail(e);
}

h3a_status h3a_last_device_error(h3a_stream_t stream) {
    int* status = nullptr;
    h3a_status rc = status_word(&status);
    if (rc != H3A_OK) return rc;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    std::lock_guard<std::mutex> lock(g_take_mu);
    // after everything already queued on `stream`: take the word, then copy it out
    status_take_kernel<<<1, 1, 0, st>>>();
    cudaError_t e = cudaGetLastError();
    int word = 0;
    if (e == cudaSuccess) e = cudaMemcpyFromSymbolAsync(&word, g_h3a_status_taken, sizeof(int), 0,
                                                        cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e);
    return (word & kDevTimeout) ? H3A_ERR_TIMEOUT : H3A_OK;
}

h3a_status h3a_selftest_wait_timeout(uint32_t limit_us, h3a_stream_t stream) {
    int* status = nullptr;
    h3a_status rc = status_word(&status);
    if (rc != H3A_OK) return rc;
    rc = h3a_last_device_error(stream);  // start from a clear word
    if (rc == H3A_ERR_CUDA) return rc;
    cudaError_t e = launch_selftest_wait(static_cast<uint64_t>(limit_us) * 1000ull, status,
                                         reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e);
    return h3a_last_device_error(stream);
}

h3a_status h3a_selftest_mma(const void* a, const void* b, float* s_out, float* r_out, h3a_stream_t stream) {
    if (!a || !b || !s_out || !r_out) return H3A_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(b) || !aligned16(s_out) || !aligned16(r_out)) return H3A_ERR_INVALID_ARG;
    int* status = nullptr;
    h3a_status rc = status_word(&status);
    if (rc != H3A_OK) return rc;
    Shape s{1, 128, 1, kHeadDim, 128 * kHeadDim, kHeadDim, kHeadDim};
    CUtensorMap ta, tb;
    cudaError_t e = make_qkv_tensor_map(&ta, a, s);
    if (e == cudaSuccess) e = make_qkv_tensor_map(&tb, b, s);
    if (e != cudaSuccess) return cuda_fail(e);
    e = launch_selftest_mma(ta, tb, s_out, r_out, status, kWaitLimitNs, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? H3A_OK : cuda_fail(e);
}

h3a_status h3a_selftest_exp2(const float* x, float* y, int32_t n, h3a_stream_t stream) {
    if (n < 0 || (n > 0 && (!x || !y))) return H3A_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x) & 3u) || (reinterpret_cast<uintptr_t>(y) & 3u)) return H3A_ERR_INVALID_ARG;
    cudaError_t e = launch_selftest_exp2(x, y, n, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? H3A_OK : cuda_fail(e);
}

}  // extern "C"
