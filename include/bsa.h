/*
 * bsa.h -- C ABI of the B200 (sm_100a) 3D Block Sparse Attention library.
 *
 * The operation is the 3D Block Sparse Attention (BSA) of a video diffusion
 * transformer, as described on the pages:
 *   [P1] "LongCat-Video Technical Report" (paper summary page), section
 *        "Block Sparse Attention (BSA)" -- 3D block partitioning, pooled block
 *        similarity, top-r key blocks per query block, masked softmax
 *        attention; section "Block Attention with KV-Cache for Efficient
 *        Multi-Task Inference" -- condition tokens attend only among themselves.
 *   [P3] "LongCat-Video Technical Report #" (detail page), section
 *        "3D Block Sparse Attention" -- default chunk shape [4,4,8], Top-K and
 *        CDF-threshold selection; section "开源实现" (open-source kernels) --
 *        gating-score, varlen forward and 3D rearrange kernels.
 *
 * Conventions for every entry point:
 *   - Tensors Q, K, V, O are bf16, contiguous [B, heads, T*H*W, d], tokens in
 *     [T,H,W] order (t slowest, w fastest). DEVICE pointers, 16-byte aligned.
 *   - Chunk c of a (batch, head) covers the (4,4,8) block (ct, ch, cw) with
 *     c = (ct*NH + ch)*NW + cw, NH = ceil(H/4), NW = ceil(W/8); its local token
 *     l = (lt*4 + lh)*8 + lw is token (4ct+lt, 4ch+lh, 8cw+lw) when that lies
 *     inside the grid (a partial edge chunk has fewer than 128 tokens).
 *   - CSR rows are ordered (batch, head, query chunk); row r's key chunks are
 *     col_idx[row_ptr[r] .. row_ptr[r+1]), ascending. int32, DEVICE memory,
 *     4-byte aligned (16 where bsa_plan or bsa_select_pooled writes them); an
 *     fp32 lse array is 4-byte aligned.
 *   - The caller allocates and owns every buffer. The library never allocates
 *     device memory. Its only process-wide state is the cached tensor-map entry
 *     point and, per device, whether each kernel's shared-memory limit has been
 *     raised; both are safe to reach from several host threads at once. The
 *     second is kept per device number: after making another context current
 *     on a device, or resetting it, the attention calls return BSA_ERR_CUDA.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Launches are
 *     asynchronous; errors found on the device are read with bsa_read_status.
 *   - Return value: BSA_OK (0) or a bsa_status code. No exception crosses the ABI.
 */
#ifndef BSA_H_
#define BSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BSA_API __attribute__((visibility("default")))
#else
#define BSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BSA_OK = 0,
    BSA_ERR_INVALID_ARG = 1,         /* null pointer, bad enum, k < 1, p outside (0,1] ...   */
    BSA_ERR_SHAPE = 2,               /* sizes <= 0, t_cond or q_begin not a multiple of 4 ... */
    BSA_ERR_UNSUPPORTED = 3,         /* d not in {64,128}, chunk shape != (4,4,8), no sm_100,
                                        or beyond the limits: Nc <= 2048 chunks per (batch,
                                        head), B*heads <= 65535, CSR rows*Nc < 2^31          */
    BSA_ERR_ALIGNMENT = 4,           /* a bf16 tensor or workspace pointer is not 16-byte
                                        aligned, or an int32 / fp32 array not 4-byte aligned */
    BSA_ERR_WORKSPACE_TOO_SMALL = 5, /* ws_bytes < bsa_workspace_size()                       */
    BSA_ERR_CUDA = 6,                /* a CUDA runtime/driver call or launch failed           */
    BSA_ERR_DEVICE_BAD_INDEX = 7,    /* device saw an out-of-range CSR row or column index    */
    BSA_ERR_DEVICE_TIMEOUT = 8,      /* a bounded device-side wait expired                    */
    BSA_ERR_CAPACITY = 9             /* col_idx capacity smaller than the selection needs     */
} bsa_status;

/* Selection modes ([P3] "3D Block Sparse Attention": Top-K, the CDF threshold
 * and a combination of the two). TOPK_CDF keeps a chunk when both rules keep it: the
 * first min(topk, CDF count) chunks of the common descending order (the pages
 * name the combination without defining it; this is the reading taken). */
typedef enum { BSA_SEL_TOPK = 0, BSA_SEL_CDF = 1, BSA_SEL_TOPK_CDF = 2 } bsa_select_mode;

typedef struct {
    int32_t B, heads, T, H, W, d; /* d in {64,128}; any T, H, W >= 1: chunks per axis are
                                   * ceil(T/4), ceil(H/4), ceil(W/8) ([P1] block counts by
                                   * ceiling division); an edge chunk of a grid that is not a
                                   * multiple of (4,4,8) is partial: pooling averages its
                                   * existing tokens, attention uses its existing keys, and
                                   * outputs exist for its existing queries only            */
    int32_t chunk_t, chunk_h, chunk_w; /* must be 4,4,8 ([P3] default chunk shape)          */
    float scale;        /* softmax scale; 0 means 1/sqrt(d) ([P1] scaled dot product)     */
    int32_t mode;       /* bsa_select_mode                                                */
    int32_t topk;       /* TOPK, TOPK_CDF: key chunks kept per query chunk (clamped to |A(i)|) */
    float cdf_p;        /* CDF, TOPK_CDF: cumulative pooled-softmax mass to reach, in (0,1] */
    float cdf_cap_frac; /* CDF, TOPK_CDF: at most max(1, floor(cap_frac*|A(i)|)) chunks, (0,1] */
    int32_t t_cond;     /* leading latent frames holding condition tokens; 0 = none; %4==0 */
    int32_t q_begin;    /* first latent frame whose queries are computed; 0 = all; %4==0, < T.
                         * Query chunks of earlier frames are neither read nor written and
                         * get no CSR row: with q_begin = t_cond this is the KV-cached
                         * video-continuation step of [P1] "Block Attention with KV-Cache":
                         * only the noisy queries are evaluated, against the cached
                         * condition K/V plus the noisy K/V, which stay in one
                         * [B,heads,T*H*W,d] buffer. Row r of the CSR is query chunk
                         * q_begin/4*NH*NW + r % Nq of (batch, head) r / Nq, where Nq is
                         * the number of chunks in frames [q_begin, q_end) (Nc -
                         * q_begin/4*NH*NW when q_end = T; bsa_shape_info reports it). */
    int32_t kchunk_t, kchunk_h, kchunk_w;
                        /* key chunk shape; 0 on an axis = the query chunk's size (4, 4, 8).
                         * Otherwise a multiple of it on that axis, at most 8 (4,4,8) boxes
                         * in all (key chunks of 128..1024 tokens: [P1]'s block-size
                         * robustness study; [P3]'s general kernel for key chunks above
                         * 128 tokens). K is pooled per key chunk, the scores are
                         * [Nq x Nk] and selection keeps topk KEY chunks per query chunk
                         * (t_cond must be a multiple of kchunk_t); the CSR that bsa_plan
                         * writes then lists the (4,4,8) boxes those key chunks cover, the
                         * unit bsa_forward / bsa_backward attend over. */
    int32_t q_end;      /* one past the last latent frame whose queries are computed; 0 = T;
                         * a multiple of 4 unless it is T. The computed query chunks are the
                         * frames [q_begin, q_end): a rank of a context-parallel group
                         * computes the rows of its own frame range (bsa_select_pooled). */
} bsa_params;

/* Library version: major*10000 + minor*100 + patch (0.2.0: bsa_shape_info and
 * bsa_forward_host added; 0.3.0: 64-token chunks, bsa_forward_partial and
 * bsa_lse_merge_f32; 0.3.1: bsa_backward for 64-token chunks; 0.3.2:
 * bsa_backward_ex). */
BSA_API int bsa_version(void);

/* Text for a status code (static storage; never NULL). */
BSA_API const char* bsa_status_string(int status);

/* Bytes of device workspace that bsa_plan / bsa_forward need for `p`
 * (status word, pooled Q/K in fp32, pooled scores, CDF scratch). 0 if `p` is
 * invalid. The same workspace serves both calls. */
BSA_API size_t bsa_workspace_size(const bsa_params* p);

/* CSR sizes for `p`: *n_rows = B*heads*Nq (Nq = query chunks of frames
 * [q_begin, q_end), Nc for the whole grid); *max_nnz = col_idx capacity that always suffices, in
 * (4,4,8) boxes (exact for TOPK with the default key chunk; an upper bound
 * otherwise). Host-only call. */
BSA_API int bsa_plan_sizes(const bsa_params* p, int64_t* n_rows, int64_t* max_nnz);

/* Element counts of the tensors a call for `p` reads and writes, so a binding
 * can check caller buffers before anything reaches the device:
 *   BH*N*d   q, k, v, out, dout, dq, dk, dv ([T,H,W] order, bf16);
 *   BH*N     lse (fp32);
 *   BH*Nc*128*d  the chunk-major side of bsa_rearrange (partial edge chunks
 *            padded to 128 slots);
 *   BH*Nc*d  bsa_pool's output; BH*Nq*d pooled queries and BH*Nk*d pooled
 *            keys of bsa_scores / bsa_select_pooled; BH*Nq*Nk their scores;
 *   rows+1   row_ptr.
 * Host-only call; SHAPE, UNSUPPORTED or INVALID_ARG as for bsa_plan_sizes. */
typedef struct {
    int64_t BH;    /* B*heads */
    int64_t N;     /* tokens per (batch, head): T*H*W */
    int64_t rows;  /* CSR rows: BH*Nq */
    int32_t d;     /* head dimension */
    int32_t Nc;    /* (4,4,8) chunks per (batch, head), partial edge chunks included */
    int32_t Nq;    /* query chunks computed per (batch, head): frames [q_begin, q_end) */
    int32_t Nk;    /* key chunks per (batch, head) (of the key chunk shape) */
} bsa_shape;
BSA_API int bsa_shape_info(const bsa_params* p, bsa_shape* out);

/*
 * Block selection ([P1] pooled block similarity + top-r; [P3] Top-K / CDF):
 *   1. mean-pool every (4,4,8) chunk of Q and K in fp32 ([P1] Q_pool, K_pool);
 *   2. pooled scores S[i,m] = <Q_pool[i], K_pool[m]> * scale in fp32;
 *   3. candidates A(i): all chunks, or -- when t_cond > 0 and chunk i lies
 *      entirely in frames < t_cond -- the condition chunks only ([P1] block
 *      attention for condition tokens);
 *   4. TOPK: the topk highest scores of A(i), ties to the lower chunk index;
 *      CDF: softmax of S over A(i), descending order (ties to the lower
 *      index), the shortest prefix with mass >= cdf_p, at most
 *      max(1, floor(cdf_cap_frac*|A(i)|)) chunks.
 * q, k: device bf16 [B,heads,N,d]. workspace: device, >= bsa_workspace_size.
 * row_ptr: device int32 [n_rows+1]; col_idx: device int32 [col_capacity],
 * written ascending per row. Errors: INVALID_ARG, SHAPE, UNSUPPORTED,
 * ALIGNMENT, WORKSPACE_TOO_SMALL, CAPACITY (host-detectable: col_capacity <
 * max_nnz), CUDA.
 */
BSA_API int bsa_plan(const bsa_params* p, const void* q, const void* k, void* workspace,
             size_t ws_bytes, int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
             void* stream);

/*
 * Sparse attention over the selected chunks ([P1] O = softmax(QK^T/sqrt(d)
 * with non-selected positions at -inf) V): for every query token of chunk i,
 * an exact softmax over the 128*|row i| keys of the chunks in CSR row i, with
 * bf16 tensor-core products, fp32 accumulation and fp32 online softmax.
 * q, k, v: device bf16 [B,heads,N,d]; out: device bf16, same shape, written in
 * [T,H,W] token order (the inverse 3D rearrangement is fused). lse: nullable
 * device fp32 [B,heads,N], natural-log log-sum-exp of the scaled logits per
 * query (-inf for an empty row). row_ptr/col_idx: CSR as written by bsa_plan,
 * or any caller CSR with col_capacity entries; rows or columns out of range
 * are skipped (their output is zero) and reported as DEVICE_BAD_INDEX by
 * bsa_read_status. Every device-side wait is bounded (2 s); one that expires
 * stops its CTA cleanly and is reported as DEVICE_TIMEOUT (bsa_forward_ex sets
 * the limit). Errors: INVALID_ARG, SHAPE, UNSUPPORTED, ALIGNMENT,
 * WORKSPACE_TOO_SMALL, CUDA.
 */
BSA_API int bsa_forward(const bsa_params* p, const void* q, const void* k, const void* v,
                const int32_t* row_ptr, const int32_t* col_idx, int64_t col_capacity,
                void* workspace, size_t ws_bytes, void* out, float* lse, void* stream);

/*
 * bsa_forward with the output kept in fp32: a partial result over one
 * partition of the keys, to be merged with the others by log-sum-exp
 * (bsa_lse_merge_f32) and rounded to bf16 only once at the end ([P1] ring
 * block sparse attention; [P3] "开源实现": LSE and output correction). Same
 * computation, arguments and errors as bsa_forward except: out_f32: device
 * fp32 [B,heads,N,d], 16-byte aligned, written in [T,H,W] token order
 * (normalised by the partition's own softmax sum; zeros for an empty row);
 * lse: required.
 */
BSA_API int bsa_forward_partial(const bsa_params* p, const void* q, const void* k, const void* v,
                                const int32_t* row_ptr, const int32_t* col_idx,
                                int64_t col_capacity, void* workspace, size_t ws_bytes,
                                float* out_f32, float* lse, void* stream);

/*
 * Bytes of device workspace that bsa_backward needs for `p` (0 if `p` is
 * invalid): a status block, LSE and <dO,O> per computed query token, and the
 * column-major (CSC) copy of a block mask of at most one entry per (row, key
 * chunk) pair; for 64-token query chunks these are over (4,4,8) boxes, after
 * the box CSR (as the forward builds it) and a quadrant pattern per CSC
 * entry. Host-only call.
 */
BSA_API size_t bsa_backward_workspace_size(const bsa_params* p);

/*
 * Gradients of bsa_forward for an upstream gradient dout ([P1] sparse
 * attention O = softmax(QK^T*scale, non-selected positions at -inf) V; [P3]
 * "开源实现": the trainable BSA's backward kernels and block-mask transpose).
 * With P = exp(QK^T*scale - lse) over the selected keys and D = <dout, out>
 * per query: dV = P^T dout, dS = P * (dout V^T - D), dQ = scale dS K,
 * dK = scale dS^T Q, each summed over the chunks of the CSR only. The block
 * selection itself has no gradient. 64-token query chunks ([P1] block-size
 * robustness) are supported as in bsa_forward: the kernels run over (4,4,8)
 * boxes of two query chunks and the union of their key boxes, each query
 * attending only to the key chunks its own chunk selected.
 * q, k, v, out, dout: device bf16 [B,heads,N,d] (out and lse exactly as
 * bsa_forward wrote them for the same CSR). lse: device fp32 [B,heads,N].
 * dq, dk, dv: device bf16 [B,heads,N,d], written in [T,H,W] token order:
 * every computed query chunk of dq (query chunks before q_begin are not
 * written; an empty CSR row gives zeros) and every key chunk of dk and dv
 * (zeros for a key chunk that no row selected). Results are deterministic
 * (no atomic accumulation). row_ptr/col_idx/col_capacity: the CSR given to
 * bsa_forward; rows or columns out of range, and a chunk listed twice in one
 * row, are reported as DEVICE_BAD_INDEX by bsa_read_status(workspace) (the
 * affected gradients are then not meaningful). Every device-side wait is
 * bounded (2 s); one that expires stops its CTA cleanly and is reported as
 * DEVICE_TIMEOUT (bsa_backward_ex sets the limit). workspace: device, >=
 * bsa_backward_workspace_size(p), 16-byte aligned, owned by the caller; its
 * first 256 bytes are the status block that bsa_read_status reads. Errors:
 * INVALID_ARG, SHAPE, UNSUPPORTED, ALIGNMENT, WORKSPACE_TOO_SMALL, CUDA.
 */
BSA_API int bsa_backward(const bsa_params* p, const void* q, const void* k, const void* v,
                         const void* out, const float* lse, const void* dout,
                         const int32_t* row_ptr, const int32_t* col_idx, int64_t col_capacity,
                         void* workspace, size_t ws_bytes, void* dq, void* dk, void* dv,
                         void* stream);

/* bsa_backward with an explicit limit for every device-side wait (timeout_ns;
 * 0 = the default of 2 s) and debug flags (bit 0: the dQ kernel's MMA thread,
 * bit 1: the dK/dV kernel's, withholds its first "scores ready" signal, so the
 * exponential warps' bounded wait expires, every role stops, the copies and
 * products in flight are waited for and TMEM is freed, and the call reports
 * DEVICE_TIMEOUT through bsa_read_status(workspace) without faulting or
 * hanging; the gradients are then not meaningful; used by the
 * failure-detection tests). Same contract as bsa_backward otherwise. */
BSA_API int bsa_backward_ex(const bsa_params* p, const void* q, const void* k, const void* v,
                            const void* out, const float* lse, const void* dout,
                            const int32_t* row_ptr, const int32_t* col_idx, int64_t col_capacity,
                            void* workspace, size_t ws_bytes, void* dq, void* dk, void* dv,
                            uint64_t timeout_ns, int debug_flags, void* stream);

/*
 * Context parallelism ([P1] ring block sparse attention: the sequence split
 * across ranks along the latent frames, pooled keys gathered from every rank,
 * each rank's queries selecting among all key chunks, partial attention over
 * every rank's K/V shard combined by an online softmax; [P3] "开源实现": LSE
 * and output correction).
 *
 * bsa_select_pooled: selection (scores + top-k / CDF, as bsa_plan) from pooled
 * inputs. `p` describes the whole group's grid, with [q_begin, q_end) the
 * frames of this rank's queries. qpool: device fp32 [B,heads,Nq,d] (this
 * rank's pooled query chunks, e.g. from bsa_pool on its shard). kpool: device
 * fp32 pooled key chunks of the whole grid, either [B,heads,Nk,d] (kshard = 0)
 * or, as an all-gather delivers them, [shard][B,heads,kshard,d] with kshard
 * key chunks per shard (Nk a multiple of kshard). The CSR has this rank's
 * rows and global chunk ids. Workspace, capacity and errors as bsa_plan.
 */
BSA_API int bsa_select_pooled(const bsa_params* p, const float* qpool, const float* kpool,
                              int32_t kshard, void* workspace, size_t ws_bytes, int32_t* row_ptr,
                              int32_t* col_idx, int64_t col_capacity, void* stream);

/* Bytes of device workspace bsa_csr_slice needs for n_rows rows (0 if n_rows < 0). */
BSA_API size_t bsa_csr_slice_workspace_size(int64_t n_rows);

/*
 * The part of a CSR that falls in one shard of key chunks: for every row, the
 * entries c with lo <= c < hi, written as c - lo in their original order.
 * row_ptr/col_idx: device int32 input (n_rows+1, col_capacity); out_row_ptr /
 * out_col_idx: device int32 output (n_rows+1, out_capacity). workspace: device,
 * >= bsa_csr_slice_workspace_size(n_rows), 16-byte aligned; its first bytes
 * are a status block (bsa_read_status: DEVICE_BAD_INDEX for an input row
 * outside col_capacity, CAPACITY if out_capacity is too small). Errors:
 * INVALID_ARG, ALIGNMENT, WORKSPACE_TOO_SMALL, CUDA.
 */
BSA_API int bsa_csr_slice(int64_t n_rows, const int32_t* row_ptr, const int32_t* col_idx,
                          int64_t col_capacity, int32_t lo, int32_t hi, void* workspace,
                          size_t ws_bytes, int32_t* out_row_ptr, int32_t* out_col_idx,
                          int64_t out_capacity, void* stream);

/*
 * Merge a partial attention result into an accumulator by log-sum-exp, for
 * every token of the grid `p` describes: with l1 = lse, l2 = lse_part,
 *   lse <- log(e^l1 + e^l2),  out <- e^(l1-lse) out + e^(l2-lse) out_part.
 * A token with lse_part = -inf (no key of that partition) keeps its value;
 * one with lse = -inf takes the part. out, out_part: device bf16
 * [B,heads,N,d]; lse, lse_part: device fp32 [B,heads,N] (natural log, as
 * bsa_forward writes them). Errors: INVALID_ARG, SHAPE, UNSUPPORTED,
 * ALIGNMENT, CUDA.
 */
BSA_API int bsa_lse_merge(const bsa_params* p, void* out, float* lse, const void* out_part,
                          const float* lse_part, void* stream);

/*
 * bsa_lse_merge with out and out_part in fp32 (device fp32 [B,heads,N,d],
 * 16-byte aligned), as bsa_forward_partial writes them: the merged result is
 * rounded once, by bsa_grad_finalize, after the last partition. Errors as for
 * bsa_lse_merge.
 */
BSA_API int bsa_lse_merge_f32(const bsa_params* p, float* out, float* lse, const float* out_part,
                              const float* lse_part, void* stream);

/*
 * Backward of the ring ([P1] ring block sparse attention; [P3] "开源实现":
 * the trainable BSA's backward kernels and the LSE correction for context
 * parallelism). bsa_backward over one K/V shard, given the merged output and
 * LSE of the whole ring, yields that shard's contributions to dQ, dK and dV;
 * each gradient is the sum of its contributions over the shards (dQ) or over
 * the ranks (dK, dV). These two calls keep that sum in fp32:
 *
 * acc <- part (overwrite = 1) or acc <- acc + part (overwrite = 0), for the
 * B*heads*N*d elements of the grid `p` describes. part: device bf16
 * [B,heads,N,d] (a gradient as bsa_backward writes it); acc: device fp32 of
 * the same shape. Both 16-byte aligned. Errors: INVALID_ARG, SHAPE,
 * UNSUPPORTED, ALIGNMENT, CUDA.
 */
BSA_API int bsa_grad_accumulate(const bsa_params* p, const void* part, float* acc, int overwrite,
                                void* stream);

/*
 * out <- acc rounded to bf16 (nearest even), for the grid `p` describes (the
 * last step of the ring's fp32 gradients, and of its fp32 merged output).
 * acc: device fp32 [B,heads,N,d]; out: device bf16 of the same shape. Both
 * 16-byte aligned. Errors: INVALID_ARG, SHAPE, UNSUPPORTED, ALIGNMENT, CUDA.
 */
BSA_API int bsa_grad_finalize(const bsa_params* p, const float* acc, void* out, void* stream);

/*
 * bsa_plan without a caller workspace: the same selection as bsa_plan, with
 * its scratch held in a fixed array inside this library, for callers that
 * cannot allocate device memory (a plug-in whose host engine owns the memory
 * budget and passes only input and output tensors, or a latency-critical
 * caller that must not call cudaMalloc/cudaFree because they can synchronise
 * the device). The paper has no counterpart; this is an interface convenience.
 *   - Limit: 32 MiB of scratch (bsa_workspace_size(p) must not exceed it,
 *     about the 480p-like grid with 32 heads); larger plans return
 *     BSA_ERR_WORKSPACE_TOO_SMALL. All of bsa_plan's host checks (shape,
 *     pointers, alignment, capacity, device) run before any CUDA call, with
 *     bsa_plan's error codes. The array occupies
 *     32 MiB on every GPU that loads this library's device code, until exit.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - Every call looks up the array's device address in the current context
 *     (an address belongs to the context it was looked up in, and a caller may
 *     switch contexts on one device). The first call in a context also loads
 *     this library's device code into it; make that first call on each device
 *     before any stream capture.
 *   - Every call reuses the same array, which keeps the previous call's
 *     contents; the call clears the part that must start at zero. Calls whose
 *     work overlaps on the GPU (e.g. on two streams without ordering) race on
 *     the array: serialise them.
 *   - Device-side errors are not kept for bsa_read_status (the status block
 *     lives in the shared array); the one the plan can raise (CAPACITY) is
 *     rejected on the host first.
 * Arguments and other errors as for bsa_plan.
 */
BSA_API int bsa_plan_noalloc(const bsa_params* p, const void* q, const void* k, int32_t* row_ptr,
                             int32_t* col_idx, int64_t col_capacity, void* stream);

/*
 * Selection and sparse attention (bsa_plan + bsa_forward) for q, k, v and out in
 * HOST memory, [B,heads,N,d] bf16 (pinned memory lets the copies run
 * asynchronously and overlap the kernels; pageable memory works but
 * serialises them). Each (batch, head) pair is an independent problem ([P1]
 * section "Block Sparse Attention (BSA)": blocks, pooled scores and the kept
 * set are per head), so the pairs are split into groups of `group`, and group
 * i runs on streams[i % slots]: its Q of the computed frames [q_begin, q_end),
 * its K and V are copied in, the plan's kernels and the forward kernel run on
 * staging buffers in the workspace, and its output of the computed frames is
 * copied out (out elsewhere is left as it was). Every slot stream first waits
 * for the work queued on `stream`, and `stream` waits for every slot at the
 * end: work queued on `stream` afterwards sees the finished output (read it on
 * the host after synchronising `stream`). Host buffers must not be touched until then.
 * group: 1..B*heads. slots: 1..16 streams (cudaStream_t; NULL entries are the
 * legacy default stream). workspace: device, 256-byte aligned,
 * >= bsa_forward_host_workspace_size(p, group, slots), owned by the caller;
 * its first 256 bytes are the status block that bsa_read_status reads (zero
 * it before the first call). Device errors of every group land there.
 * Errors: INVALID_ARG, SHAPE, UNSUPPORTED, ALIGNMENT, WORKSPACE_TOO_SMALL, CUDA.
 * A CUDA error part way through stops queueing further groups; `stream` still
 * waits for whatever was already queued on the slot streams (or the call waits
 * for it on the host), so after synchronising `stream` nothing writes the host
 * buffers any more, also when the call returned an error.
 */
BSA_API size_t bsa_forward_host_workspace_size(const bsa_params* p, int32_t group, int32_t slots);
BSA_API int bsa_forward_host(const bsa_params* p, const void* q, const void* k, const void* v,
                             void* out, int32_t group, int32_t slots, void* const* streams,
                             void* workspace, size_t ws_bytes, void* stream);

/* bsa_forward with an explicit limit for every device-side wait (timeout_ns;
 * 0 = the default of 2 s) and debug flags (bit 0: the MMA warp withholds its
 * first "scores ready" signal, so the softmax warps' bounded wait expires and
 * the kernel reports DEVICE_TIMEOUT without faulting or hanging; bit 1: every
 * CTA adds 1 to status word 8 as it returns; used by the failure-detection
 * tests). Same contract as bsa_forward otherwise. */
BSA_API int bsa_forward_ex(const bsa_params* p, const void* q, const void* k, const void* v,
                   const int32_t* row_ptr, const int32_t* col_idx, int64_t col_capacity,
                   void* workspace, size_t ws_bytes, void* out, float* lse, uint64_t timeout_ns,
                   int debug_flags, void* stream);

/* Synchronise `stream`, return the first device-side error recorded in the
 * workspace status word since the last call (BSA_OK if none) and clear it.
 * The status block (the first 256 bytes of every workspace) holds uint32
 * words: [0] error bits; [1] number of bounded waits that expired; [2] 1 once
 * [3..5] hold the first expired wait: its site code ((role*100 + barrier*10 +
 * tile)*10000 + step, role 1 = copy producer, 2 = MMA issuer, 3 = exponential
 * warps), the CTA index and the phase parity; [8] CTAs that finished, counted
 * only by bsa_forward_ex with debug bit 1. This call clears words 0 to 5.
 * workspace: device, the workspace (at least 256 bytes) of one of the calls
 * above. Errors: INVALID_ARG (NULL workspace), CUDA. */
BSA_API int bsa_read_status(void* workspace, void* stream);

/*
 * 3D rearrangement ([P1] "tokens ... rearranged in memory so that all tokens
 * within a block are contiguous"; [P3] rearrange_THW_to_3d_block and its
 * inverse). inverse = 0: x in [T,H,W] token order -> out chunk-major
 * [B,heads,Nc,128,d]; inverse = 1: chunk-major -> [T,H,W]. bf16, device,
 * 16-byte aligned, non-overlapping. A bit-exact permutation.
 */
BSA_API int bsa_rearrange(const bsa_params* p, const void* x, void* out, int inverse, void* stream);

/* Chunk mean-pool ([P1] Q_pool / K_pool) of one tensor: x bf16 [B,heads,N,d]
 * -> pooled fp32 [B,heads,Nc,d] (device). The same kernel bsa_plan runs. */
BSA_API int bsa_pool(const bsa_params* p, const void* x, float* pooled, void* stream);

/* Pooled scores ([P1] S_pool = Q_pool K_pool^T / sqrt(d); [P3] gating-score
 * kernel): qp fp32 [B,heads,Nq,d], kp fp32 [B,heads,Nc,d] -> S fp32
 * [B,heads,Nq,Nc] (device), S = <qp_i, kp_m> * scale (Nq = Nc when
 * q_begin = 0). The same kernel bsa_plan runs. */
BSA_API int bsa_scores(const bsa_params* p, const float* qp, const float* kp, float* S, void* stream);

/* Device self-test of the softmax exponentials: for n (even) floats x, writes
 * the FMA-pipe polynomial 2^x that the forward kernel uses for part of the
 * softmax numerators into y_poly, and the MUFU ex2.approx value into y_mufu.
 * Device pointers, 4-byte aligned. Used to check the polynomial against exact
 * 2^x. Errors: INVALID_ARG (n odd or negative), ALIGNMENT, UNSUPPORTED, CUDA. */
BSA_API int bsa_selftest_exp2(const float* x, float* y_poly, float* y_mufu, int64_t n,
                              void* stream);

/* Device self-test of the bounded-wait machinery: launches one CTA that waits
 * on a barrier nothing arrives at, for at most timeout_ns, then records
 * DEVICE_TIMEOUT in the workspace status word and returns. The context stays
 * usable. workspace: device, >= 256 bytes. */
BSA_API int bsa_selftest_timeout(void* workspace, uint64_t timeout_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H_ */
