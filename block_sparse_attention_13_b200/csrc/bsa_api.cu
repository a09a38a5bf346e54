// C ABI of the block sparse attention library: argument checking, workspace
// layout and the launch sequence of each entry point. See include/bsa.h.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>

#include "bsa_internal.cuh"
#include "bsa_ptx.cuh"

namespace bsa {

static size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

static int64_t max_key_nnz_of(const Dims& g, const bsa_params& p);

WsLayout ws_layout(const Dims& g, const bsa_params& p) {
    WsLayout L{};
    size_t off = 0;
    L.status = off;
    off += 256;
    L.qpool = off;
    off += round_up((size_t)g.BH * g.Nq * g.d * sizeof(float), 256);
    L.kpool = off;
    off += round_up((size_t)g.BH * g.Nk * g.d * sizeof(float), 256);
    L.scores = off;
    off += round_up((size_t)g.BH * g.Nq * g.Nk * sizeof(float), 256);
    L.pad_stride = 0;
    L.counts = L.padded = L.kc_row_ptr = L.kc_col_idx = off;
    L.kc_cap = 0;
    if (p.mode != BSA_SEL_TOPK || g.m > 1) {
        L.counts = off;
        off += round_up((size_t)g.rows * sizeof(int32_t), 256);
    }
    if (p.mode != BSA_SEL_TOPK) {
        int cap = (int)std::floor((double)p.cdf_cap_frac * g.Nk);
        if (cap < 1) cap = 1;
        if (cap > g.Nk) cap = g.Nk;
        if (p.mode == BSA_SEL_TOPK_CDF && p.topk < cap) cap = p.topk;
        L.pad_stride = cap;
        L.padded = off;
        off += round_up((size_t)g.rows * cap * sizeof(int32_t), 256);
    }
    if (g.m > 1) {
        // selection in key chunks first, then the expansion to (4,4,8) boxes
        L.kc_cap = max_key_nnz_of(g, p);
        L.kc_row_ptr = off;
        off += round_up((size_t)(g.rows + 1) * sizeof(int32_t), 256);
        L.kc_col_idx = off;
        off += round_up((size_t)(L.kc_cap > 0 ? L.kc_cap : 1) * sizeof(int32_t), 256);
    }
    L.box_counts = L.box_row_ptr = L.box_col_idx = L.box_pat = off;
    L.box_cap = 0;
    if (g.qw != kChunkW) {
        // a query box's list is the union of its two chunks' lists: at most their sum
        L.box_cap = max_key_nnz_of(g, p);
        if (L.box_cap < 1) L.box_cap = 1;
        const size_t box_rows = (size_t)g.BH * g.NB;
        L.box_counts = off;
        off += round_up(box_rows * sizeof(int32_t), 256);
        L.box_row_ptr = off;
        off += round_up((box_rows + 1) * sizeof(int32_t), 256);
        L.box_col_idx = off;
        off += round_up((size_t)L.box_cap * sizeof(int32_t), 256);
        L.box_pat = off;
        off += round_up((size_t)L.box_cap, 256);
    }
    L.total = off;
    return L;
}

// Validates `p` and fills the derived sizes. Host only, no CUDA calls.
int make_dims(const bsa_params* p, Dims* g) {
    if (!p || !g) return BSA_ERR_INVALID_ARG;
    if (p->B <= 0 || p->heads <= 0 || p->T <= 0 || p->H <= 0 || p->W <= 0 || p->d <= 0)
        return BSA_ERR_SHAPE;
    // query chunks: (4,4,8), the [P3] default, or (4,4,4), the 64-token blocks of
    // [P1]'s block-size robustness study
    if (p->chunk_t != kChunkT || p->chunk_h != kChunkH ||
        (p->chunk_w != kChunkW && p->chunk_w != kChunkW / 2))
        return BSA_ERR_UNSUPPORTED;
    const bool q64 = p->chunk_w == kChunkW / 2;
    if (p->d != 64 && p->d != 128) return BSA_ERR_UNSUPPORTED;
    if (p->t_cond < 0 || p->t_cond % kChunkT || p->t_cond > p->T) return BSA_ERR_SHAPE;
    // key chunk shape: 0 = the query chunk's size on that axis; otherwise a
    // positive multiple of it, at most 8 boxes of (4,4,8) in all. With 64-token
    // query chunks the key chunk is (4,4,4) or (4,4,8).
    const int kt = p->kchunk_t ? p->kchunk_t : kChunkT, kh = p->kchunk_h ? p->kchunk_h : kChunkH,
              kw = p->kchunk_w ? p->kchunk_w : p->chunk_w;
    if (q64) {
        if (kt != kChunkT || kh != kChunkH || (kw != kChunkW && kw != kChunkW / 2))
            return BSA_ERR_UNSUPPORTED;
    } else {
        if (kt < 0 || kh < 0 || kw < 0 || kt % kChunkT || kh % kChunkH || kw % kChunkW)
            return BSA_ERR_UNSUPPORTED;
        if ((kt / kChunkT) * (kh / kChunkH) * (kw / kChunkW) > 8) return BSA_ERR_UNSUPPORTED;
    }
    if (p->t_cond % kt) return BSA_ERR_SHAPE;
    if (p->q_begin < 0 || p->q_begin % kChunkT || p->q_begin >= p->T) return BSA_ERR_SHAPE;
    // q_end: 0 = T; otherwise past q_begin, at most T, a multiple of 4 unless it is T
    const int q_end = p->q_end ? p->q_end : p->T;
    if (q_end <= p->q_begin || q_end > p->T || (q_end % kChunkT && q_end != p->T))
        return BSA_ERR_SHAPE;
    // 64-token query chunks: every query chunk is computed (no KV-cached step, no
    // context-parallel row range)
    if (q64 && (p->q_begin != 0 || q_end != p->T)) return BSA_ERR_UNSUPPORTED;
    if (!(std::isfinite(p->scale)) || p->scale < 0.f) return BSA_ERR_INVALID_ARG;
    if (p->mode == BSA_SEL_TOPK || p->mode == BSA_SEL_TOPK_CDF) {
        if (p->topk < 1) return BSA_ERR_INVALID_ARG;
    } else if (p->mode != BSA_SEL_CDF) {
        return BSA_ERR_INVALID_ARG;
    }
    if (p->mode != BSA_SEL_TOPK) {
        if (!(p->cdf_p > 0.f && p->cdf_p <= 1.f)) return BSA_ERR_INVALID_ARG;
        if (!(p->cdf_cap_frac > 0.f && p->cdf_cap_frac <= 1.f)) return BSA_ERR_INVALID_ARG;
    }
    g->B = p->B;
    g->heads = p->heads;
    g->T = p->T;
    g->H = p->H;
    g->W = p->W;
    g->d = p->d;
    // chunks per axis by ceiling division: edge chunks of a grid that is not a
    // multiple of the chunk shape are partial
    g->NT = (p->T + kChunkT - 1) / kChunkT;
    g->NH = (p->H + kChunkH - 1) / kChunkH;
    g->NW = (p->W + kChunkW - 1) / kChunkW;          // (4,4,8) boxes along w
    g->qw = p->chunk_w;
    g->NWq = (p->W + g->qw - 1) / g->qw;              // query chunks along w
    const int64_t nb = (int64_t)g->NT * g->NH * g->NW;
    const int64_t nc = (int64_t)g->NT * g->NH * g->NWq;
    g->N = (int64_t)p->T * p->H * p->W;
    g->BH = (int64_t)p->B * p->heads;
    // Limits of this implementation: selection keeps a row of scores in one
    // warp's registers (Nc, Nk <= 2048), grids index batch*heads in y (<= 65535),
    // and CSR offsets are int32.
    if (nc > 2048 || g->BH > 65535) return BSA_ERR_UNSUPPORTED;
    g->Nc = (int)nc;
    g->NB = (int)nb;
    if (q64) {
        // key chunks are (4,4,4) half-boxes or whole (4,4,8) boxes; no expansion
        g->kw64 = kw == kChunkW / 2;
        g->mT = g->mH = g->mW = g->m = 1;
        g->NkT = g->NT;
        g->NkH = g->NH;
        g->NkW = g->kw64 ? g->NWq : g->NW;
    } else {
        g->kw64 = 0;
        g->mT = kt / kChunkT;
        g->mH = kh / kChunkH;
        g->mW = kw / kChunkW;
        g->m = g->mT * g->mH * g->mW;
        g->NkT = (g->NT + g->mT - 1) / g->mT;
        g->NkH = (g->NH + g->mH - 1) / g->mH;
        g->NkW = (g->NW + g->mW - 1) / g->mW;
    }
    g->Nk = g->NkT * g->NkH * g->NkW;
    g->n_cond_k = (p->t_cond / kt) * g->NkH * g->NkW;
    g->q_skip = (p->q_begin / kChunkT) * g->NH * g->NWq;
    const int q_stop = q_end == p->T ? g->Nc : (q_end / kChunkT) * g->NH * g->NWq;
    g->Nq = q_stop - g->q_skip;
    g->rows = g->BH * g->Nq;
    const int nmax = g->Nc > g->Nk ? g->Nc : g->Nk;
    if (g->rows * (int64_t)nmax > INT32_MAX) return BSA_ERR_UNSUPPORTED;
    g->n_cond = (p->t_cond / kChunkT) * g->NH * g->NWq;
    g->scale = p->scale > 0.f ? p->scale : 1.0f / std::sqrt((float)p->d);
    return BSA_OK;
}

// Computed rows per (batch, head) that are condition rows (candidates: the
// n_cond condition chunks) and noisy rows (candidates: all chunks).
static int64_t cond_rows(const Dims& g) {
    const int c_end = g.n_cond < g.q_skip + g.Nq ? g.n_cond : g.q_skip + g.Nq;
    return c_end > g.q_skip ? c_end - g.q_skip : 0;
}
static int64_t noisy_rows(const Dims& g) { return g.Nq - cond_rows(g); }

// CSR entries in key chunks (exact for TOPK, an upper bound otherwise).
static int64_t max_key_nnz_of(const Dims& g, const bsa_params& p) {
    if (p.mode == BSA_SEL_TOPK) {
        const int64_t kc = p.topk < g.n_cond_k ? p.topk : g.n_cond_k;
        const int64_t kn = p.topk < g.Nk ? p.topk : g.Nk;
        return g.BH * (cond_rows(g) * kc + noisy_rows(g) * kn);
    }
    int64_t total = 0;
    for (int which = 0; which < 2; ++which) {
        const int na = which == 0 ? g.n_cond_k : g.Nk;
        const int64_t nrows = which == 0 ? cond_rows(g) : noisy_rows(g);
        if (nrows == 0) continue;
        int cap = (int)std::floor((double)p.cdf_cap_frac * na);
        if (cap < 1) cap = 1;
        if (p.mode == BSA_SEL_TOPK_CDF && p.topk < cap) cap = p.topk;
        total += nrows * cap;
    }
    return g.BH * total;
}

// CSR entries in (4,4,8) boxes: a key chunk covers at most m of them.
int64_t max_nnz_of(const Dims& g, const bsa_params& p) { return max_key_nnz_of(g, p) * g.m; }

static bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }
// int32 CSR arrays and fp32 vectors are read element by element: 4-byte alignment
static bool aligned4(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 3u) == 0; }

static int cuda_status(cudaError_t e) { return e == cudaSuccess ? BSA_OK : BSA_ERR_CUDA; }

cudaError_t launch_forward_any(const Dims& g, const bsa_params& p, const void* q, const void* k,
                               const void* v, const int32_t* row_ptr, const int32_t* col_idx,
                               int64_t col_cap, char* ws, uint32_t* status, void* out, float* lse,
                               uint64_t timeout_ns, int debug_flags, cudaStream_t st,
                               float* out_f32) {
    if (g.qw == kChunkW)
        return launch_forward(g, q, k, v, row_ptr, col_idx, col_cap, out, lse, status, timeout_ns,
                              debug_flags, st, out_f32);
    // 64-token query chunks: one tile per (4,4,8) box of queries, over the union of
    // its two chunks' key boxes with a quadrant pattern per entry
    const WsLayout L = ws_layout(g, p);
    int32_t* bcnt = reinterpret_cast<int32_t*>(ws + L.box_counts);
    int32_t* brp = reinterpret_cast<int32_t*>(ws + L.box_row_ptr);
    int32_t* bci = reinterpret_cast<int32_t*>(ws + L.box_col_idx);
    uint8_t* bpat = reinterpret_cast<uint8_t*>(ws + L.box_pat);
    cudaError_t e = launch_quad_union(g, row_ptr, col_idx, col_cap, bcnt, brp, bci, bpat,
                                      L.box_cap, status, st);
    if (e != cudaSuccess) return e;
    const Dims gb = box_dims(g);
    return launch_forward(gb, q, k, v, brp, bci, L.box_cap, out, lse, status, timeout_ns,
                          debug_flags, st, out_f32, bpat);
}

int device_ok() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return BSA_ERR_CUDA;
    return major == 10 ? BSA_OK : BSA_ERR_UNSUPPORTED;
}

// Workspace bsa_forward needs: the status block, plus the box CSR for 64-token
// query chunks (the plan's workspace, bsa_workspace_size, holds both).
static size_t forward_ws_bytes(const Dims& g, const bsa_params& p) {
    return g.qw == kChunkW ? 256 : ws_layout(g, p).total;
}

}  // namespace bsa

using namespace bsa;

extern "C" {

int bsa_version(void) { return 302; }

const char* bsa_status_string(int s) {
    switch (s) {
        case BSA_OK: return "ok";
        case BSA_ERR_INVALID_ARG: return "invalid argument";
        case BSA_ERR_SHAPE: return "invalid shape (sizes must be positive; t_cond, q_begin multiples of 4)";
        case BSA_ERR_UNSUPPORTED: return "unsupported configuration or device";
        case BSA_ERR_ALIGNMENT: return "tensor pointer not 16-byte aligned";
        case BSA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case BSA_ERR_CUDA: return "CUDA call or launch failed";
        case BSA_ERR_DEVICE_BAD_INDEX: return "device saw an out-of-range CSR index";
        case BSA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
        case BSA_ERR_CAPACITY: return "col_idx capacity too small";
        default: return "unknown status";
    }
}

size_t bsa_workspace_size(const bsa_params* p) {
    Dims g;
    if (make_dims(p, &g) != BSA_OK) return 0;
    return ws_layout(g, *p).total;
}

int bsa_plan_sizes(const bsa_params* p, int64_t* n_rows, int64_t* max_nnz) {
    Dims g;
    const int rc = make_dims(p, &g);
    if (rc != BSA_OK) return rc;
    if (!n_rows || !max_nnz) return BSA_ERR_INVALID_ARG;
    *n_rows = g.rows;
    *max_nnz = max_nnz_of(g, *p);
    return BSA_OK;
}

int bsa_shape_info(const bsa_params* p, bsa_shape* out) {
    Dims g;
    const int rc = make_dims(p, &g);
    if (rc != BSA_OK) return rc;
    if (!out) return BSA_ERR_INVALID_ARG;
    out->BH = g.BH;
    out->N = g.N;
    out->rows = g.rows;
    out->d = g.d;
    out->Nc = g.Nc;
    out->Nq = g.Nq;
    out->Nk = g.Nk;
    return BSA_OK;
}

int bsa_plan(const bsa_params* p, const void* q, const void* k, void* workspace, size_t ws_bytes,
             int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity, void* stream) {
    TraceRange trace("bsa_plan");
    Dims g;
    int rc = make_dims(p, &g);
    if (rc != BSA_OK) return rc;
    if (!q || !k || !workspace || !row_ptr || !col_idx) return BSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(workspace) || !aligned16(row_ptr) ||
        !aligned16(col_idx))
        return BSA_ERR_ALIGNMENT;
    const WsLayout L = ws_layout(g, *p);
    if (ws_bytes < L.total) return BSA_ERR_WORKSPACE_TOO_SMALL;
    if (col_capacity < max_nnz_of(g, *p)) return BSA_ERR_CAPACITY;
    if ((rc = device_ok()) != BSA_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    float* qp = reinterpret_cast<float*>(ws + L.qpool);
    float* kp = reinterpret_cast<float*>(ws + L.kpool);
    float* S = reinterpret_cast<float*>(ws + L.scores);
    uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
    {
        TraceRange stage("bsa_plan.pool");
        if ((rc = cuda_status(launch_pool(g, q, k, qp, kp, st))) != BSA_OK) return rc;
    }
    {
        TraceRange stage("bsa_plan.scores");
        if ((rc = cuda_status(launch_scores(g, qp, kp, S, st))) != BSA_OK) return rc;
    }
    TraceRange select_stage("bsa_plan.select");
    int32_t* counts = reinterpret_cast<int32_t*>(ws + L.counts);
    int32_t* padded = reinterpret_cast<int32_t*>(ws + L.padded);
    if (g.m == 1)
        return cuda_status(launch_select(g, *p, S, row_ptr, col_idx, col_capacity, counts, padded,
                                         L.pad_stride, status, st));
    // key chunks larger than the query chunk: select key chunks, then list their boxes
    int32_t* kc_rp = reinterpret_cast<int32_t*>(ws + L.kc_row_ptr);
    int32_t* kc_ci = reinterpret_cast<int32_t*>(ws + L.kc_col_idx);
    if ((rc = cuda_status(launch_select(g, *p, S, kc_rp, kc_ci, L.kc_cap, counts, padded,
                                        L.pad_stride, status, st))) != BSA_OK)
        return rc;
    return cuda_status(launch_expand_boxes(g, kc_rp, kc_ci, counts, row_ptr, col_idx, col_capacity,
                                           status, st));
}

// Internal: forward with a custom wait limit and debug flags (used by the
// binding's fault tests). Same contract as bsa_forward otherwise.
int bsa_forward_ex(const bsa_params* p, const void* q, const void* k, const void* v,
                   const int32_t* row_ptr, const int32_t* col_idx, int64_t col_capacity,
                   void* workspace, size_t ws_bytes, void* out, float* lse, uint64_t timeout_ns,
                   int debug_flags, void* stream) {
    TraceRange trace("bsa_forward");
    Dims g;
    int rc = make_dims(p, &g);
    if (rc != BSA_OK) return rc;
    if (!q || !k || !v || !row_ptr || !col_idx || !workspace || !out || col_capacity < 0)
        return BSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        !aligned16(workspace) || (lse && !aligned4(lse)) || !aligned4(row_ptr) ||
        !aligned4(col_idx))
        return BSA_ERR_ALIGNMENT;
    if (ws_bytes < forward_ws_bytes(g, *p)) return BSA_ERR_WORKSPACE_TOO_SMALL;
    if ((rc = device_ok()) != BSA_OK) return rc;
    char* ws = static_cast<char*>(workspace);
    return cuda_status(launch_forward_any(g, *p, q, k, v, row_ptr, col_idx, col_capacity, ws,
                                          reinterpret_cast<uint32_t*>(ws), out, lse,
                                          timeout_ns ? timeout_ns : kDefaultTimeoutNs, debug_flags,
                                          static_cast<cudaStream_t>(stream), nullptr));
}

int bsa_forward_partial(const bsa_params* p, const void* q, const void* k, const void* v,
                        const int32_t* row_ptr, const int32_t* col_idx, int64_t col_capacity,
                        void* workspace, size_t ws_bytes, float* out_f32, float* lse,
                        void* stream) {
    TraceRange trace("bsa_forward_partial");
    Dims g;
    int rc = make_dims(p, &g);
    if (rc != BSA_OK) return rc;
    if (!q || !k || !v || !row_ptr || !col_idx || !workspace || !out_f32 || !lse ||
        col_capacity < 0)
        return BSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out_f32) ||
        !aligned16(workspace) || !aligned4(lse) || !aligned4(row_ptr) || !aligned4(col_idx))
        return BSA_ERR_ALIGNMENT;
    if (ws_bytes < forward_ws_bytes(g, *p)) return BSA_ERR_WORKSPACE_TOO_SMALL;
    if ((rc = device_ok()) != BSA_OK) return rc;
    char* ws = static_cast<char*>(workspace);
    return cuda_status(launch_forward_any(g, *p, q, k, v, row_ptr, col_idx, col_capacity, ws,
                                          reinterpret_cast<uint32_t*>(ws), nullptr, lse,
                                          kDefaultTimeoutNs, 0, static_cast<cudaStream_t>(stream),
                                          out_f32));
}

int bsa_forward(const bsa_params* p, const void* q, const void* k, const void* v,
                const int32_t* row_ptr, const int32_t* col_idx, int64_t col_capacity,
                void* workspace, size_t ws_bytes, void* out, float* lse, void* stream) {
    return bsa_forward_ex(p, q, k, v, row_ptr, col_idx, col_capacity, workspace, ws_bytes, out,
                          lse, 0, 0, stream);
}

size_t bsa_backward_workspace_size(const bsa_params* p) {
    Dims g;
    if (make_dims(p, &g) != BSA_OK) return 0;
    return bwd_layout(g, *p).total;
}

int bsa_backward_ex(const bsa_params* p, const void* q, const void* k, const void* v,
                    const void* out, const float* lse, const void* dout, const int32_t* row_ptr,
                    const int32_t* col_idx, int64_t col_capacity, void* workspace, size_t ws_bytes,
                    void* dq, void* dk, void* dv, uint64_t timeout_ns, int debug_flags,
                    void* stream) {
    TraceRange trace("bsa_backward");
    Dims g;
    int rc = make_dims(p, &g);
    if (rc != BSA_OK) return rc;
    if (!q || !k || !v || !out || !lse || !dout || !row_ptr || !col_idx || !workspace || !dq ||
        !dk || !dv || col_capacity < 0)
        return BSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace) ||
        !aligned4(lse) || !aligned4(row_ptr) || !aligned4(col_idx))
        return BSA_ERR_ALIGNMENT;
    if (ws_bytes < bwd_layout(g, *p).total) return BSA_ERR_WORKSPACE_TOO_SMALL;
    if ((rc = device_ok()) != BSA_OK) return rc;
    return cuda_status(launch_backward(g, *p, q, k, v, out, lse, dout, row_ptr, col_idx, col_capacity,
                                       workspace, dq, dk, dv,
                                       timeout_ns ? timeout_ns : kDefaultTimeoutNs, debug_flags,
                                       static_cast<cudaStream_t>(stream)));
}

int bsa_backward(const bsa_params* p, const void* q, const void* k, const void* v,
                 const void* out, const float* lse, const void* dout, const int32_t* row_ptr,
                 const int32_t* col_idx, int64_t col_capacity, void* workspace, size_t ws_bytes,
                 void* dq, void* dk, void* dv, void* stream) {
    return bsa_backward_ex(p, q, k, v, out, lse, dout, row_ptr, col_idx, col_capacity, workspace,
                           ws_bytes, dq, dk, dv, 0, 0, stream);
}

int bsa_select_pooled(const bsa_params* p, const float* qpool, const float* kpool, int32_t kshard,
                      void* workspace, size_t ws_bytes, int32_t* row_ptr, int32_t* col_idx,
                      int64_t col_capacity, void* stream) {
    TraceRange trace("bsa_select_pooled");
    Dims g;
    int rc = make_dims(p, &g);
    if (rc != BSA_OK) return rc;
    if (g.qw != kChunkW) return BSA_ERR_UNSUPPORTED;  // the ring uses (4,4,8) chunks
    if (!qpool || !kpool || !workspace || !row_ptr || !col_idx) return BSA_ERR_INVALID_ARG;
    if (kshard < 0 || (kshard > 0 && g.Nk % kshard)) return BSA_ERR_INVALID_ARG;
    if (!aligned16(qpool) || !aligned16(kpool) || !aligned16(workspace) || !aligned16(row_ptr) ||
        !aligned16(col_idx))
        return BSA_ERR_ALIGNMENT;
    const WsLayout L = ws_layout(g, *p);
    if (ws_bytes < L.total) return BSA_ERR_WORKSPACE_TOO_SMALL;
    if (col_capacity < max_nnz_of(g, *p)) return BSA_ERR_CAPACITY;
    if ((rc = device_ok()) != BSA_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    float* S = reinterpret_cast<float*>(ws + L.scores);
    uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
    if ((rc = cuda_status(launch_scores(g, qpool, kpool, S, st, kshard))) != BSA_OK) return rc;
    int32_t* counts = reinterpret_cast<int32_t*>(ws + L.counts);
    int32_t* padded = reinterpret_cast<int32_t*>(ws + L.padded);
    if (g.m == 1)
        return cuda_status(launch_select(g, *p, S, row_ptr, col_idx, col_capacity, counts, padded,
                                         L.pad_stride, status, st));
    int32_t* kc_rp = reinterpret_cast<int32_t*>(ws + L.kc_row_ptr);
    int32_t* kc_ci = reinterpret_cast<int32_t*>(ws + L.kc_col_idx);
    if ((rc = cuda_status(launch_select(g, *p, S, kc_rp, kc_ci, L.kc_cap, counts, padded,
                                        L.pad_stride, status, st))) != BSA_OK)
        return rc;
    return cuda_status(launch_expand_boxes(g, kc_rp, kc_ci, counts, row_ptr, col_idx, col_capacity,
                                           status, st));
}

size_t bsa_csr_slice_workspace_size(int64_t n_rows) {
    if (n_rows < 0) return 0;
    return 256 + round_up((size_t)n_rows * sizeof(int32_t), 256);
}

int bsa_csr_slice(int64_t n_rows, const int32_t* row_ptr, const int32_t* col_idx,
                  int64_t col_capacity, int32_t lo, int32_t hi, void* workspace, size_t ws_bytes,
                  int32_t* out_row_ptr, int32_t* out_col_idx, int64_t out_capacity, void* stream) {
    TraceRange trace("bsa_csr_slice");
    if (n_rows < 0 || !row_ptr || !col_idx || !workspace || !out_row_ptr || !out_col_idx ||
        col_capacity < 0 || out_capacity < 0 || lo < 0 || hi < lo)
        return BSA_ERR_INVALID_ARG;
    if (!aligned16(workspace) || !aligned4(row_ptr) || !aligned4(col_idx) ||
        !aligned4(out_row_ptr) || !aligned4(out_col_idx))
        return BSA_ERR_ALIGNMENT;
    if (ws_bytes < bsa_csr_slice_workspace_size(n_rows)) return BSA_ERR_WORKSPACE_TOO_SMALL;
    int rc = device_ok();
    if (rc != BSA_OK) return rc;
    if (n_rows == 0) return BSA_OK;
    char* ws = static_cast<char*>(workspace);
    return cuda_status(launch_csr_slice(n_rows, row_ptr, col_idx, col_capacity, lo, hi,
                                        reinterpret_cast<int32_t*>(ws + 256), out_row_ptr,
                                        out_col_idx, out_capacity,
                                        reinterpret_cast<uint32_t*>(ws),
                                        static_cast<cudaStream_t>(stream)));
}

int bsa_lse_merge(const bsa_params* p, void* out, float* lse, const void* out_part,
                  const float* lse_part, void* stream) {
    TraceRange trace("bsa_lse_merge");
    Dims g;
    int rc = make_dims(p, &g);
    if (rc != BSA_OK) return rc;
    if (!out || !lse || !out_part || !lse_part) return BSA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(out_part) || !aligned4(lse) || !aligned4(lse_part))
        return BSA_ERR_ALIGNMENT;
    if ((rc = device_ok()) != BSA_OK) return rc;
    return cuda_status(launch_lse_merge(g, out, lse, out_part, lse_part,
                                        static_cast<cudaStream_t>(stream)));
}

int bsa_lse_merge_f32(const bsa_params* p, float* out, float* lse, const float* out_part,
                      const float* lse_part, void* stream) {
    TraceRange trace("bsa_lse_merge_f32");
    Dims g;
    int rc = make_dims(p, &g);
    if (rc != BSA_OK) return rc;
    if (!out || !lse || !out_part || !lse_part) return BSA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(out_part) || !aligned4(lse) || !aligned4(lse_part))
        return BSA_ERR_ALIGNMENT;
    if ((rc = device_ok()) != BSA_OK) return rc;
    return cuda_status(launch_lse_merge_f32(g, out, lse, out_part, lse_part,
                                            static_cast<cudaStream_t>(stream)));
}

int bsa_grad_accumulate(const bsa_params* p, const void* part, float* acc, int overwrite,
                        void* stream) {
    TraceRange trace("bsa_grad_accumulate");
    Dims g;
    int rc = make_dims(p, &g);
    if (rc != BSA_OK) return rc;
    if (!part || !acc || (overwrite != 0 && overwrite != 1)) return BSA_ERR_INVALID_ARG;
    if (!aligned16(part) || !aligned16(acc)) return BSA_ERR_ALIGNMENT;
    if ((rc = device_ok()) != BSA_OK) return rc;
    return cuda_status(launch_grad_accumulate(g.BH * g.N * g.d, part, acc, overwrite,
                                              static_cast<cudaStream_t>(stream)));
}

int bsa_grad_finalize(const bsa_params* p, const float* acc, void* out, void* stream) {
    TraceRange trace("bsa_grad_finalize");
    Dims g;
    int rc = make_dims(p, &g);
    if (rc != BSA_OK) return rc;
    if (!acc || !out) return BSA_ERR_INVALID_ARG;
    if (!aligned16(acc) || !aligned16(out)) return BSA_ERR_ALIGNMENT;
    if ((rc = device_ok()) != BSA_OK) return rc;
    return cuda_status(launch_grad_finalize(g.BH * g.N * g.d, acc, out,
                                            static_cast<cudaStream_t>(stream)));
}

int bsa_read_status(void* workspace, void* stream) {
    if (!workspace) return BSA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return BSA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return BSA_ERR_CUDA;
    // the status word and the record of the first expired wait (words 0 to 5)
    if (cudaMemsetAsync(workspace, 0, 6 * sizeof(uint32_t), st) != cudaSuccess) return BSA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return BSA_ERR_CUDA;
    if (word & kStatusTimeout) return BSA_ERR_DEVICE_TIMEOUT;
    if (word & kStatusBadIndex) return BSA_ERR_DEVICE_BAD_INDEX;
    if (word & kStatusCapacity) return BSA_ERR_CAPACITY;
    return BSA_OK;
}

int bsa_rearrange(const bsa_params* p, const void* x, void* out, int inverse, void* stream) {
    TraceRange trace("bsa_rearrange");
    Dims g;
    int rc = make_dims(p, &g);
    if (rc != BSA_OK) return rc;
    if (g.qw != kChunkW) return BSA_ERR_UNSUPPORTED;  // chunk-major copy of (4,4,8) chunks
    if (!x || !out || (inverse != 0 && inverse != 1)) return BSA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(out)) return BSA_ERR_ALIGNMENT;
    if ((rc = device_ok()) != BSA_OK) return rc;
    return cuda_status(launch_rearrange(g, x, out, inverse, static_cast<cudaStream_t>(stream)));
}

int bsa_pool(const bsa_params* p, const void* x, float* pooled, void* stream) {
    TraceRange trace("bsa_pool");
    Dims g;
    int rc = make_dims(p, &g);
    if (rc != BSA_OK) return rc;
    if (!x || !pooled) return BSA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(pooled)) return BSA_ERR_ALIGNMENT;
    if ((rc = device_ok()) != BSA_OK) return rc;
    return cuda_status(launch_pool(g, x, nullptr, pooled, nullptr, static_cast<cudaStream_t>(stream)));
}

int bsa_scores(const bsa_params* p, const float* qp, const float* kp, float* S, void* stream) {
    TraceRange trace("bsa_scores");
    Dims g;
    int rc = make_dims(p, &g);
    if (rc != BSA_OK) return rc;
    if (!qp || !kp || !S) return BSA_ERR_INVALID_ARG;
    if (!aligned16(qp) || !aligned16(kp) || !aligned16(S)) return BSA_ERR_ALIGNMENT;
    if ((rc = device_ok()) != BSA_OK) return rc;
    return cuda_status(launch_scores(g, qp, kp, S, static_cast<cudaStream_t>(stream)));
}

int bsa_selftest_exp2(const float* x, float* y_poly, float* y_mufu, int64_t n, void* stream) {
    if (!x || !y_poly || !y_mufu || n < 0 || (n & 1)) return BSA_ERR_INVALID_ARG;
    if (!aligned4(x) || !aligned4(y_poly) || !aligned4(y_mufu)) return BSA_ERR_ALIGNMENT;
    const int rc = device_ok();
    if (rc != BSA_OK) return rc;
    return cuda_status(launch_exp2_selftest(x, y_poly, y_mufu, n, static_cast<cudaStream_t>(stream)));
}

int bsa_selftest_timeout(void* workspace, uint64_t timeout_ns, void* stream) {
    if (!workspace || timeout_ns == 0) return BSA_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return BSA_ERR_ALIGNMENT;
    int rc = device_ok();
    if (rc != BSA_OK) return rc;
    return cuda_status(launch_selftest_timeout(static_cast<uint32_t*>(workspace), timeout_ns,
                                               static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
