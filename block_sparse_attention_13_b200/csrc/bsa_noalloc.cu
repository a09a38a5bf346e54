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

#include <cstdint>

#include "bsa_internal.cuh"

namespace {

// Fixed scratch: 32 MiB on every GPU that loads this library's device code,
// held until the process exits. Enough for plans up to roughly the 480p-like
// grid (28,672 tokens x 32 heads needs about 14 MB); larger plans are
// rejected with BSA_ERR_WORKSPACE_TOO_SMALL.
constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(32) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array in the CURRENT context. In host code the array's
// name is only a host-side stand-in, so kernels must be given this address
// instead. It is looked up on every call, not cached: an address belongs to the
// context it was looked up in, and a caller may make another context current on
// the same device (or reset the device) between calls. After the first lookup in
// a context the call is a cheap host-side table lookup; the first one loads the
// library's device code into that context.
int scratch_address(void** out) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
        (void)cudaGetLastError();  // do not leave the failure for the caller's next check
        return BSA_ERR_CUDA;
    }
    *out = p;
    return BSA_OK;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

}  // namespace

extern "C" BSA_API int bsa_plan_noalloc(const bsa_params* p, const void* q, const void* k,
                                        int32_t* row_ptr, int32_t* col_idx,
                                        int64_t col_capacity, void* stream) {
    // The host checks bsa_plan makes, in its order, before any CUDA call: an input
    // the library rejects queues no work and leaves no CUDA error behind.
    bsa::Dims g;
    int rc = bsa::make_dims(p, &g);
    if (rc != BSA_OK) return rc;
    if (!q || !k || !row_ptr || !col_idx) return BSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(row_ptr) || !aligned16(col_idx))
        return BSA_ERR_ALIGNMENT;
    if (bsa::ws_layout(g, *p).total > kNoAllocScratchBytes) return BSA_ERR_WORKSPACE_TOO_SMALL;
    if (col_capacity < bsa::max_nnz_of(g, *p)) return BSA_ERR_CAPACITY;
    if ((rc = bsa::device_ok()) != BSA_OK) return rc;
    void* scratch = nullptr;
    if ((rc = scratch_address(&scratch)) != BSA_OK) return rc;
    // The array keeps the previous call's contents; only the status block must
    // start at zero (every other region is fully rewritten by the plan).
    if (cudaMemsetAsync(scratch, 0, 256, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return BSA_ERR_CUDA;
    return bsa_plan(p, q, k, scratch, kNoAllocScratchBytes, row_ptr, col_idx, col_capacity,
                    stream);
}
