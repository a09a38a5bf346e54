// Internal declarations shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <cstdint>

#include "../../include/bsa.h"

namespace bsa {

// NVTX range over the host side of one call (argument checks and launches), so
// a profiler's timeline groups each entry point's kernels under its name. The
// calls cost a few nanoseconds when no profiler is attached.
struct TraceRange {
    explicit TraceRange(const char* name) { nvtxRangePushA(name); }
    ~TraceRange() { nvtxRangePop(); }
    TraceRange(const TraceRange&) = delete;
    TraceRange& operator=(const TraceRange&) = delete;
};

// Raises a kernel's dynamic shared-memory limit on the current device. The
// attribute belongs to that device's context, so `done` keeps one bit per device
// (a device numbered 64 or above sets it on every call). Two threads that race on
// the first launch both set it, which is harmless.
template <typename Kernel>
inline cudaError_t raise_smem_limit(Kernel kernel, int bytes, std::atomic<uint64_t>& done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t{1} << dev) : 0;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

constexpr int kChunkT = 4, kChunkH = 4, kChunkW = 8;
constexpr int kChunkTokens = kChunkT * kChunkH * kChunkW;  // 128

// Token-space origin (t, h, w) of chunk c.
__host__ __device__ __forceinline__ void chunk_origin(int c, int NH, int NW, int& t0, int& h0,
                                                      int& w0) {
    t0 = (c / (NH * NW)) * kChunkT;
    h0 = ((c / NW) % NH) * kChunkH;
    w0 = (c % NW) * kChunkW;
}

// Code of a wait site for the timeout record: role (1 TMA, 2 MMA, 3 softmax),
// barrier, tile and step.
__host__ __device__ __forceinline__ uint32_t site(int role, int bar, int tile, int step) {
    return static_cast<uint32_t>((role * 100 + bar * 10 + tile) * 10000 +
                                 (step < 9999 ? step : 9999));
}

// Derived sizes of one call.
struct Dims {
    int B, heads, T, H, W, d;
    int NT, NH, NW;      // (4,4,8) boxes per axis (the unit of the attention kernels' tiles)
    int Nc;              // query chunks per (batch, head) (= boxes, unless 64-token chunks)
    int qw, NWq;         // query chunk width along w (8, or 4 for 64-token chunks); chunks along w
    int NB;              // (4,4,8) boxes per (batch, head)
    int kw64;            // key chunks are (4,4,4) half-boxes (64-token query chunks only)
    int64_t N, BH, rows;
    int n_cond;      // condition query chunks per (batch, head); 0 without block-causal mask
    int q_skip;      // query chunks before q_begin (not computed)
    int Nq;          // query chunks computed per (batch, head): Nc - q_skip
    // key chunks: mT x mH x mW boxes each (1x1x1 unless the key chunk is larger)
    int mT, mH, mW, m;
    int NkT, NkH, NkW, Nk;
    int n_cond_k;    // condition key chunks per (batch, head)
    float scale;
};

// Workspace layout (byte offsets), identical for plan and forward.
struct WsLayout {
    size_t status;   // uint32 status word (+ padding to 256)
    size_t qpool;    // float [BH][Nq][d]
    size_t kpool;    // float [BH][Nk][d]
    size_t scores;   // float [BH][Nq][Nk]
    size_t counts;   // int32 [rows]            (CDF and box expansion)
    size_t padded;   // int32 [rows][pad_stride] (CDF only)
    int pad_stride;  // max chunks a CDF row may keep
    size_t kc_row_ptr;  // int32 [rows+1]   key-chunk CSR before box expansion (m > 1)
    size_t kc_col_idx;  // int32 [kc_cap]
    int64_t kc_cap;
    // 64-token query chunks: the forward's CSR over (4,4,8) boxes, one row per query
    // box (its two query chunks), with a quadrant pattern per entry
    size_t box_counts;  // int32 [BH*NB]
    size_t box_row_ptr; // int32 [BH*NB+1]
    size_t box_col_idx; // int32 [box_cap]
    size_t box_pat;     // uint8 [box_cap]
    int64_t box_cap;
    size_t total;
};

WsLayout ws_layout(const Dims& g, const bsa_params& p);

// Host-side checks shared by the entry points (no CUDA call except device_ok):
// parameter validation into derived sizes, the CSR capacity a plan needs, and
// whether the current device is an sm_100 part (BSA_OK, UNSUPPORTED or CUDA).
int make_dims(const bsa_params* p, Dims* g);
int64_t max_nnz_of(const Dims& g, const bsa_params& p);
int device_ok();

// 64-token query chunks: the dims of the attention kernels, whose rows are
// (4,4,8) boxes of two query chunks and whose key chunks are (4,4,8) boxes.
inline Dims box_dims(const Dims& g) {
    Dims gb = g;
    gb.Nc = gb.Nq = g.NB;
    gb.q_skip = 0;
    gb.rows = g.BH * g.NB;
    gb.qw = kChunkW;
    gb.NWq = g.NW;
    return gb;
}

// Backward workspace layout (byte offsets). With 64-token query chunks every
// size below is over boxes (box_dims), after the box CSR of the call.
struct BwdLayout {
    size_t status;   // uint32 status word (+ padding to 256)
    size_t aux;      // float [BH][Nq][2][128]: per half of 64 queries, LSE * log2(e) then <dO, O>
    size_t bitmap;   // uint32 [BH*Nc][words]: query rows per key chunk
    size_t rawcnt;   // int32 [BH*Nc]: entries per key chunk (duplicate check)
    size_t cnt;      // int32 [BH*Nc]: distinct rows per key chunk
    size_t col_ptr;  // int32 [BH*Nc + 1]
    size_t row_idx;  // int32 [idx_cap]
    int words;       // ceil(Nq / 32)
    int64_t idx_cap; // BH * Nq * Nc
    // 64-token query chunks only: the box CSR (launch_quad_union) and the quadrant
    // pattern of every CSC entry
    size_t box_counts;  // int32 [BH*NB]
    size_t box_row_ptr; // int32 [BH*NB+1]
    size_t box_col_idx; // int32 [box_cap]
    size_t box_pat;     // uint8 [box_cap]
    int64_t box_cap;
    size_t csc_pat;     // uint8 [idx_cap]
    size_t total;
};

BwdLayout bwd_layout(const Dims& g, const bsa_params& p);

// Launchers (return cudaError_t of the launch).
cudaError_t launch_pool(const Dims& g, const void* x0, const void* x1, float* p0, float* p1,
                        cudaStream_t st);
cudaError_t launch_rearrange(const Dims& g, const void* src, void* dst, int inverse,
                             cudaStream_t st);
// kshard > 0: kp is [shard][BH][kshard][d] (gathered pooled keys of a context-
// parallel group); 0: the plain [BH][Nk][d] layout.
cudaError_t launch_scores(const Dims& g, const float* qp, const float* kp, float* S,
                          cudaStream_t st, int kshard = 0);
cudaError_t launch_select(const Dims& g, const bsa_params& p, const float* S, int32_t* row_ptr,
                          int32_t* col_idx, int64_t col_cap, int32_t* counts, int32_t* padded,
                          int pad_stride, uint32_t* status, cudaStream_t st);
// out_f32 non-null: O is written there in fp32 (and `out` is not used). quad
// non-null: rows are query boxes of 64-token chunks, with a quadrant pattern per
// CSR entry (launch_quad_union); g then describes boxes (Nc = Nq = NB).
cudaError_t launch_forward(const Dims& g, const void* q, const void* k, const void* v,
                           const int32_t* row_ptr, const int32_t* col_idx, int64_t col_cap,
                           void* out, float* lse, uint32_t* status, uint64_t timeout_ns,
                           int debug_flags, cudaStream_t st, float* out_f32 = nullptr,
                           const uint8_t* quad = nullptr);
// 5-D TMA map over a [BH][T][H][W][d] bf16 tensor whose box is one (4,4,8)
// chunk x 64 channels (128-byte swizzle); box_t = 2 gives half a chunk (its
// first or last two frames: local tokens 0-63 or 64-127). False if the driver
// call failed.
bool make_chunk_map(CUtensorMap* tm, const void* base, const Dims& g, int box_t = kChunkT);
cudaError_t launch_scan_counts(const int32_t* counts, int64_t n, int32_t* ptr, cudaStream_t st);
// Key-chunk CSR -> CSR over the (4,4,8) boxes each selected key chunk covers.
cudaError_t launch_expand_boxes(const Dims& g, const int32_t* kc_row_ptr,
                                const int32_t* kc_col_idx, int32_t* counts, int32_t* row_ptr,
                                int32_t* col_idx, int64_t col_cap, uint32_t* status,
                                cudaStream_t st);
// 64-token query chunks: the chunk CSR (rows = query chunks) -> a CSR over
// (4,4,8) boxes with one row per query box and a 4-bit quadrant pattern per
// entry (bits 0-1: key halves the box's left query chunk attends to, bits 2-3:
// the right one's).
cudaError_t launch_quad_union(const Dims& g, const int32_t* row_ptr, const int32_t* col_idx,
                              int64_t col_cap, int32_t* counts, int32_t* box_row_ptr,
                              int32_t* box_col, uint8_t* box_pat, int64_t box_cap,
                              uint32_t* status, cudaStream_t st);
// The forward of one call on device buffers: for 64-token query chunks the box
// CSR is built first, in the regions ws_layout(g, p) gives inside `ws` (a
// workspace of at least that size; unused otherwise). Device errors go to status.
cudaError_t launch_forward_any(const Dims& g, const bsa_params& p, const void* q, const void* k,
                               const void* v, const int32_t* row_ptr, const int32_t* col_idx,
                               int64_t col_cap, char* ws, uint32_t* status, void* out, float* lse,
                               uint64_t timeout_ns, int debug_flags, cudaStream_t st,
                               float* out_f32);
cudaError_t launch_backward(const Dims& g, const bsa_params& p, const void* q, const void* k,
                            const void* v, const void* out, const float* lse, const void* dout,
                            const int32_t* row_ptr, const int32_t* col_idx, int64_t col_cap,
                            void* workspace, void* dq, void* dk, void* dv, uint64_t timeout_ns,
                            int debug_flags, cudaStream_t st);
// Context parallelism: CSR entries with lo <= column < hi, re-indexed to
// column - lo (order kept); and the log-sum-exp merge of a partial attention
// result into an accumulator.
cudaError_t launch_csr_slice(int64_t rows, const int32_t* row_ptr, const int32_t* col_idx,
                             int64_t col_cap, int lo, int hi, int32_t* counts, int32_t* out_row_ptr,
                             int32_t* out_col_idx, int64_t out_cap, uint32_t* status,
                             cudaStream_t st);
cudaError_t launch_lse_merge(const Dims& g, void* out, float* lse, const void* out_part,
                             const float* lse_part, cudaStream_t st);
// The same merge with fp32 accumulator and fp32 partial result.
cudaError_t launch_lse_merge_f32(const Dims& g, float* out, float* lse, const float* out_part,
                                 const float* lse_part, cudaStream_t st);
cudaError_t launch_grad_accumulate(int64_t n, const void* part, float* acc, int overwrite,
                                   cudaStream_t st);
cudaError_t launch_grad_finalize(int64_t n, const float* acc, void* out, cudaStream_t st);
cudaError_t launch_exp2_selftest(const float* x, float* y_poly, float* y_mufu, int64_t n,
                                 cudaStream_t st);
cudaError_t launch_selftest_timeout(uint32_t* status, uint64_t timeout_ns, cudaStream_t st);

// Default limit of every device-side wait (2 s of global time).
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;

}  // namespace bsa
