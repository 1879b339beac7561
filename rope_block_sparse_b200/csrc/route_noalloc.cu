// h3a_route_noalloc: the blockwise router for callers that cannot allocate
// device memory.
//
// Some callers have no way to obtain device memory at the point where they
// route: an embedding runtime that hands out no allocator after start-up, a
// plugin running inside a host callback or a foreign allocator's critical
// section, or a serving loop with a fixed memory budget that must not grow.
// h3a_route needs a caller workspace for the pooled block means; this entry
// point takes none.  Its scratch is the file-scope array below, a fixed
// H3A_ROUTE_NOALLOC_MAX_BYTES (64 MiB) that every GPU loading the library holds
// until the process exits.
//
// In host code the array's name is only a host-side stand-in, not a device
// address, so the device address is resolved once per device with
// cudaGetSymbolAddress (that device current) and handed to the same router
// kernels h3a_route launches.  The pool kernel overwrites every pooled value
// the score kernel later reads, so nothing needs clearing between calls.  All
// calls share the one array: calls whose executions overlap on the GPU (other
// streams, other host threads) race on it.
#include <cuda_runtime.h>

#include <mutex>

#include "h3a.h"
#include "h3a_internal.h"

namespace h3a {
namespace {

constexpr size_t kNoallocScratchBytes = H3A_ROUTE_NOALLOC_MAX_BYTES;
constexpr int kMaxNoallocDevices = 64;

static __device__ __align__(256) unsigned char g_route_scratch[kNoallocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxNoallocDevices] = {};

// Device address of g_route_scratch on the current device, resolved on the
// first call made with that device current.
h3a_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return H3A_ERR_CUDA;
    if (dev < 0 || dev >= kMaxNoallocDevices) return H3A_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr) return H3A_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return H3A_OK;
}

}  // namespace
}  // namespace h3a

extern "C" h3a_status h3a_route_noalloc(const void* q, const void* k, const h3a_qkv_desc* d, double sparsity,
                                        int32_t block, int32_t* block_idx, int64_t* k_out, h3a_stream_t stream) {
    size_t need = 0;
    h3a_status rc = h3a_route_workspace_size(d, block, &need);
    if (rc != H3A_OK) return rc;
    if (need > h3a::kNoallocScratchBytes) return H3A_ERR_WORKSPACE;  // shape too large for the built-in scratch
    void* scratch = nullptr;
    rc = h3a::scratch_address(&scratch);
    if (rc != H3A_OK) return rc;
    return h3a_route(q, k, d, sparsity, block, block_idx, k_out, scratch, h3a::kNoallocScratchBytes, stream);
}
