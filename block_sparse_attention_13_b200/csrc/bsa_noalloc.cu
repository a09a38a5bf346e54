// bsa_plan_noalloc: block selection for callers that cannot allocate device
// memory themselves and therefore cannot hand bsa_plan a workspace.
//
// Who cannot allocate: code hosted by an engine that owns the whole device
// memory budget and hands a plug-in only its input and output tensors; and
// latency-critical callers for which cudaMalloc / cudaFree are off limits
// because they can synchronise the device and stall work on other streams.
// For them the plan's scratch (status word, pooled Q/K, pooled scores, CDF
// row buffers) lives in one fixed array in this library's device code.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/bsa.h"

namespace {

// Fixed scratch: 32 MiB on every GPU that loads this library's device code,
// held until the process exits. Enough for plans up to roughly the 480p-like
// grid (28,672 tokens x 32 heads needs about 14 MB); larger plans are
// rejected with BSA_ERR_WORKSPACE_TOO_SMALL.
constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(32) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array, looked up once per device. In host code the
// array's name is only a host-side stand-in, so kernels must be given this
// address instead.
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BSA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return BSA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return BSA_OK;
}

}  // namespace

extern "C" BSA_API int bsa_plan_noalloc(const bsa_params* p, const void* q, const void* k,
                                        int32_t* row_ptr, int32_t* col_idx,
                                        int64_t col_capacity, void* stream) {
    const size_t need = bsa_workspace_size(p);
    if (need == 0) {
        int64_t rows = 0, nnz = 0;
        const int rc = bsa_plan_sizes(p, &rows, &nnz);
        return rc != BSA_OK ? rc : BSA_ERR_INVALID_ARG;
    }
    if (need > kNoAllocScratchBytes) return BSA_ERR_WORKSPACE_TOO_SMALL;
    if (!q || !k || !row_ptr || !col_idx) return BSA_ERR_INVALID_ARG;
    void* scratch = nullptr;
    int rc = scratch_address(&scratch);
    if (rc != BSA_OK) return rc;
    // The array keeps the previous call's contents; only the status block must
    // start at zero (every other region is fully rewritten by the plan).
    if (cudaMemsetAsync(scratch, 0, 256, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return BSA_ERR_CUDA;
    return bsa_plan(p, q, k, scratch, kNoAllocScratchBytes, row_ptr, col_idx, col_capacity,
                    stream);
}
