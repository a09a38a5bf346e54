// bsa_forward_host: selection and sparse attention for Q, K, V and O in HOST
// memory, with the host<->device copies overlapped with the kernels.
//
// Every (batch, head) pair is an independent problem for pooling, selection and
// attention ("LongCat-Video Technical Report", section "Block Sparse Attention
// (BSA)": blocks, pooled scores and the kept set are all per head), so the call
// splits the pairs into groups and runs group i on stream i % slots of the
// caller's streams: copy in the group's Q (computed frames only), K and V, run
// the plan's kernels and the forward kernel on device staging buffers, copy out
// the group's output (computed frames only). While one group computes, the next
// one's inputs and the previous one's output cross PCIe on the copy engines.
// The staging buffers live in the caller's workspace: the library allocates no
// device memory.
#include <cuda_runtime.h>

#include <cstdint>

#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr int kMaxHostSlots = 16;

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Parameters of one group of n (batch, head) pairs: the same grid and
// selection, as a problem of B = 1 and n heads.
bsa_params group_params(const bsa_params& p, int n) {
    bsa_params q = p;
    q.B = 1;
    q.heads = n;
    return q;
}

// Workspace of bsa_forward_host: a 256-byte status block shared by every group,
// then `slots` equal slots of staging (Q, K, V, O of one group; the plan's
// workspace; the CSR of one group).
struct HostLayout {
    size_t slot0, slot_bytes;
    size_t q, k, v, out, plan_ws, row_ptr, col_idx;  // offsets inside a slot
    size_t plan_ws_bytes;
    int64_t col_cap;  // col_idx entries of one slot
    size_t total;
};

int host_layout(const bsa_params& p, int group, int slots, HostLayout* L) {
    const bsa_params pg = group_params(p, group);
    Dims gd;
    const int rc = make_dims(&pg, &gd);
    if (rc != BSA_OK) return rc;
    const size_t tensor = round256(static_cast<size_t>(gd.BH) * gd.N * gd.d * 2);
    size_t off = 0;
    L->q = off;
    off += tensor;
    L->k = off;
    off += tensor;
    L->v = off;
    off += tensor;
    L->out = off;
    off += tensor;
    L->plan_ws = off;
    L->plan_ws_bytes = round256(ws_layout(gd, pg).total);
    off += L->plan_ws_bytes;
    L->row_ptr = off;
    off += round256(static_cast<size_t>(gd.rows + 1) * sizeof(int32_t));
    L->col_idx = off;
    L->col_cap = max_nnz_of(gd, pg);
    if (L->col_cap < 1) L->col_cap = 1;
    off += round256(static_cast<size_t>(L->col_cap) * sizeof(int32_t));
    L->slot_bytes = off;
    L->slot0 = 256;
    L->total = L->slot0 + static_cast<size_t>(slots) * L->slot_bytes;
    return BSA_OK;
}

// The launches bsa_plan makes, on device buffers of one group, with device
// errors recorded in `status`.
cudaError_t plan_group(const Dims& g, const bsa_params& p, const void* q, const void* k,
                       char* ws, int32_t* row_ptr, int32_t* col_idx, int64_t col_cap,
                       uint32_t* status, cudaStream_t st) {
    const WsLayout L = ws_layout(g, p);
    float* qp = reinterpret_cast<float*>(ws + L.qpool);
    float* kp = reinterpret_cast<float*>(ws + L.kpool);
    float* S = reinterpret_cast<float*>(ws + L.scores);
    int32_t* counts = reinterpret_cast<int32_t*>(ws + L.counts);
    int32_t* padded = reinterpret_cast<int32_t*>(ws + L.padded);
    cudaError_t e = launch_pool(g, q, k, qp, kp, st);
    if (e == cudaSuccess) e = launch_scores(g, qp, kp, S, st);
    if (e != cudaSuccess) return e;
    if (g.m == 1)
        return launch_select(g, p, S, row_ptr, col_idx, col_cap, counts, padded, L.pad_stride,
                             status, st);
    int32_t* kc_rp = reinterpret_cast<int32_t*>(ws + L.kc_row_ptr);
    int32_t* kc_ci = reinterpret_cast<int32_t*>(ws + L.kc_col_idx);
    e = launch_select(g, p, S, kc_rp, kc_ci, L.kc_cap, counts, padded, L.pad_stride, status, st);
    if (e != cudaSuccess) return e;
    return launch_expand_boxes(g, kc_rp, kc_ci, counts, row_ptr, col_idx, col_cap, status, st);
}

// Events that order the slot streams after the caller's stream and the
// caller's stream after them; destroyed on every return path (a destroyed
// event that is still pending is released once the device reaches it).
struct EventSet {
    cudaEvent_t ev[kMaxHostSlots + 1] = {};
    int n = 0;
    cudaError_t make(int count) {
        for (; n < count; ++n) {
            const cudaError_t e = cudaEventCreateWithFlags(&ev[n], cudaEventDisableTiming);
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    ~EventSet() {
        for (int i = 0; i < n; ++i) cudaEventDestroy(ev[i]);
    }
};

}  // namespace
}  // namespace bsa

using namespace bsa;

extern "C" {

size_t bsa_forward_host_workspace_size(const bsa_params* p, int32_t group, int32_t slots) {
    Dims g;
    if (make_dims(p, &g) != BSA_OK) return 0;
    if (group < 1 || group > g.BH || slots < 1 || slots > kMaxHostSlots) return 0;
    HostLayout L;
    if (host_layout(*p, group, slots, &L) != BSA_OK) return 0;
    return L.total;
}

int bsa_forward_host(const bsa_params* p, const void* q, const void* k, const void* v, void* out,
                     int32_t group, int32_t slots, void* const* streams, void* workspace,
                     size_t ws_bytes, void* stream) {
    TraceRange trace("bsa_forward_host");
    Dims g;
    int rc = make_dims(p, &g);
    if (rc != BSA_OK) return rc;
    if (!q || !k || !v || !out || !workspace || !streams) return BSA_ERR_INVALID_ARG;
    if (group < 1 || group > g.BH || slots < 1 || slots > kMaxHostSlots)
        return BSA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return BSA_ERR_ALIGNMENT;
    HostLayout L;
    if ((rc = host_layout(*p, group, slots, &L)) != BSA_OK) return rc;
    if (ws_bytes < L.total) return BSA_ERR_WORKSPACE_TOO_SMALL;
    if ((rc = device_ok()) != BSA_OK) return rc;

    cudaStream_t main_st = static_cast<cudaStream_t>(stream);
    EventSet events;
    if (events.make(slots + 1) != cudaSuccess) return BSA_ERR_CUDA;
    // every slot stream starts after the work already queued on the caller's stream
    if (cudaEventRecord(events.ev[slots], main_st) != cudaSuccess) return BSA_ERR_CUDA;
    for (int s = 0; s < slots; ++s)
        if (cudaStreamWaitEvent(static_cast<cudaStream_t>(streams[s]), events.ev[slots], 0) !=
            cudaSuccess)
            return BSA_ERR_CUDA;

    char* ws = static_cast<char*>(workspace);
    uint32_t* status = reinterpret_cast<uint32_t*>(ws);
    const size_t pair_bytes = static_cast<size_t>(g.N) * g.d * 2;     // one (batch, head)
    const size_t frame_bytes = static_cast<size_t>(g.H) * g.W * g.d * 2;
    const int q_end = p->q_end ? p->q_end : p->T;
    const size_t q_off = static_cast<size_t>(p->q_begin) * frame_bytes;   // computed frames
    const size_t q_len = static_cast<size_t>(q_end - p->q_begin) * frame_bytes;
    const char* qh = static_cast<const char*>(q);
    const char* kh = static_cast<const char*>(k);
    const char* vh = static_cast<const char*>(v);
    char* oh = static_cast<char*>(out);

    // A failure part way through stops queueing further groups, but the work
    // already queued on the slot streams still runs: the caller's stream is
    // made to wait for it on every return path after this point, so the host
    // buffers are not written after the caller has synchronised `stream`.
    int err = BSA_OK;
    int i = 0;
    for (int64_t g0 = 0; g0 < g.BH && err == BSA_OK; g0 += group, ++i) {
        const int n = static_cast<int>(g.BH - g0 < group ? g.BH - g0 : group);
        const int s = i % slots;
        cudaStream_t st = static_cast<cudaStream_t>(streams[s]);
        char* slot = ws + L.slot0 + static_cast<size_t>(s) * L.slot_bytes;
        const bsa_params pg = group_params(*p, n);
        Dims gd;
        if ((err = make_dims(&pg, &gd)) != BSA_OK) break;
        const size_t src = static_cast<size_t>(g0) * pair_bytes;
        // Q of the computed frames, K and V whole (the candidates span every frame)
        if (cudaMemcpy2DAsync(slot + L.q + q_off, pair_bytes, qh + src + q_off, pair_bytes, q_len,
                              n, cudaMemcpyHostToDevice, st) != cudaSuccess ||
            cudaMemcpyAsync(slot + L.k, kh + src, n * pair_bytes, cudaMemcpyHostToDevice, st) !=
                cudaSuccess ||
            cudaMemcpyAsync(slot + L.v, vh + src, n * pair_bytes, cudaMemcpyHostToDevice, st) !=
                cudaSuccess) {
            err = BSA_ERR_CUDA;
            break;
        }
        int32_t* rp = reinterpret_cast<int32_t*>(slot + L.row_ptr);
        int32_t* ci = reinterpret_cast<int32_t*>(slot + L.col_idx);
        if (plan_group(gd, pg, slot + L.q, slot + L.k, slot + L.plan_ws, rp, ci, L.col_cap, status,
                       st) != cudaSuccess ||
            launch_forward_any(gd, pg, slot + L.q, slot + L.k, slot + L.v, rp, ci, L.col_cap,
                               slot + L.plan_ws, status, slot + L.out, nullptr, kDefaultTimeoutNs,
                               0, st, nullptr) != cudaSuccess) {
            err = BSA_ERR_CUDA;
            break;
        }
        // the output of the computed frames; the others stay as the caller left them
        if (cudaMemcpy2DAsync(oh + src + q_off, pair_bytes, slot + L.out + q_off, pair_bytes, q_len,
                              n, cudaMemcpyDeviceToHost, st) != cudaSuccess) {
            err = BSA_ERR_CUDA;
            break;
        }
    }
    // the caller's stream continues once every slot's last operation is done
    for (int s = 0; s < slots; ++s) {
        if (cudaEventRecord(events.ev[s], static_cast<cudaStream_t>(streams[s])) != cudaSuccess ||
            cudaStreamWaitEvent(main_st, events.ev[s], 0) != cudaSuccess) {
            // cannot order the caller's stream after this slot: wait for it here
            (void)cudaStreamSynchronize(static_cast<cudaStream_t>(streams[s]));
            if (err == BSA_OK) err = BSA_ERR_CUDA;
        }
    }
    return err;
}

}  // extern "C"
