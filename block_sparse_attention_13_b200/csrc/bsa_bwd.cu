// Block-sparse attention backward for sm_100a (tcgen05 + TMEM + TMA).
//
// Gradients of O = softmax(QK^T * scale, non-selected key chunks at -inf) V
// ("LongCat-Video Technical Report", section "Block Sparse Attention (BSA)",
// sparse attention computation; "LongCat-Video Technical Report #", section
// "开源实现": the trainable BSA ships backward kernels and a row-to-column
// transpose of the block mask). With P[q,j] = exp(s[q,j] - LSE[q]) recomputed
// from the forward's log-sum-exp and D[q] = <dO[q], O[q]>:
//   dV[j] = sum_q P[q,j] dO[q]          dP[q,j] = <dO[q], V[j]>
//   dS[q,j] = P[q,j] (dP[q,j] - D[q])    dQ[q] = scale sum_j dS[q,j] K[j]
//   dK[j] = scale sum_q dS[q,j] Q[q]
//
// Launch sequence (no atomics on gradients, so results are deterministic):
//   1. prep:  D = rowsum(dO * O) and LSE * log2(e), chunk-major per query chunk;
//   2. CSC:   the CSR block mask transposed (per key chunk, the query chunks
//             that selected it, ascending) through a per-column bitmap;
//   3. dQ:    one CTA per query chunk (CSR row): Q and dO copied to TMEM once,
//             then S = Q K^T and dP = dO V^T per selected key chunk, dS in
//             TMEM, dQ += dS K accumulated in TMEM;
//   4. dK/dV: one CTA per key chunk (CSC column): S^T = K Q^T and
//             dP^T = V dO^T per query chunk that selected it; P^T and dS^T
//             written back to TMEM in two phases so the exponentials overlap
//             the tensor core's work; dV += P^T dO and dK += dS^T Q in TMEM.
// Q, K, V, dO and the gradients stay in [T,H,W] token order; the same 5-D TMA
// box as the forward lands one chunk in shared memory in chunk-local order.
//
// 64-token query chunks ("LongCat-Video Technical Report", block-size
// robustness): as in the forward, the rows and key chunks of steps 1-4 are
// (4,4,8) boxes (two query chunks; the union of their key boxes), and every
// CSR and CSC entry carries a 4-bit quadrant pattern; the exponential warps set
// the weights of the quadrants a box's chunks did not select to zero, which
// leaves exactly the gradients of each chunk's own attention.
//
// Every mbarrier wait is bounded; on expiry the CTA records a timeout in the
// status word, drains its in-flight copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bsa_internal.cuh"
#include "bsa_ptx.cuh"

namespace bsa {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------------ prep
// Per computed query chunk r (chunk q_skip + r) of head bh, a 1 KB record in
// two halves of 64 local queries: aux[bh][r][h][0..63] = LSE * log2(e) and
// aux[bh][r][h][64..127] = <dO, O> of local queries 64h .. 64h+63. One CTA per
// (r, bh).
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ dout,
                                                       const float* __restrict__ lse,
                                                       float* __restrict__ aux, int q_skip, int Nq,
                                                       int T, int H, int W, int NH, int NW,
                                                       int64_t N) {
    constexpr int VPT = D / 8;               // 16-byte vectors per token row
    constexpr int ITERS = 128 * VPT / 256;   // vectors per thread
    const int r = blockIdx.x;
    const int64_t bh = blockIdx.y;
    int ct, ch, cw;
    chunk_origin(q_skip + r, NH, NW, ct, ch, cw);
    const int tid = threadIdx.x;
    float* dst = aux + (bh * Nq + r) * 256;
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
        const int vi = it * 256 + tid;
        const int l = vi / VPT, dv = vi % VPT;
        const int lt = l >> 5, lh = (l >> 3) & 3, lw = l & 7;
        // slots of a partial edge chunk past the grid: D = 0 (their dO rows load as zeros)
        const bool exists = ct + lt < T && ch + lh < H && cw + lw < W;
        const int64_t tok = (static_cast<int64_t>(ct + lt) * H + (ch + lh)) * W + cw + lw;
        const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
        const uint4 a = exists ? *reinterpret_cast<const uint4*>(o + (bh * N + tok) * D + dv * 8) : zero;
        const uint4 b = exists ? *reinterpret_cast<const uint4*>(dout + (bh * N + tok) * D + dv * 8) : zero;
        const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&av[e]));
            const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bv[e]));
            acc = fmaf(x.x, y.x, acc);
            acc = fmaf(x.y, y.y, acc);
        }
#pragma unroll
        for (int off = VPT / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (dv == 0) dst[(l >> 6) * 128 + 64 + (l & 63)] = acc;
    }
    if (tid < 128) {
        const int l = tid;
        const int lt = l >> 5, lh = (l >> 3) & 3, lw = l & 7;
        const bool exists = ct + lt < T && ch + lh < H && cw + lw < W;
        const int64_t tok = (static_cast<int64_t>(ct + lt) * H + (ch + lh)) * W + cw + lw;
        // a missing query gets LSE = +inf, so every P of it is exactly zero
        dst[(l >> 6) * 128 + (l & 63)] = exists ? lse[bh * N + tok] * kLog2e : INFINITY;
    }
}

// ------------------------------------------------------------------ CSR -> CSC
// One warp per CSR row: sets bit r (local row) in the bitmap of every listed
// key chunk and counts the entries per column (a duplicate entry shows up as
// count > popcount). Rows or columns out of range are dropped and reported.
__global__ void __launch_bounds__(256) csc_scatter_kernel(
    const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx, int64_t col_cap,
    int64_t rows, int Nq, int Nc, int words, uint32_t* __restrict__ bitmap,
    int32_t* __restrict__ rawcnt, uint32_t* status) {
    const int lane = threadIdx.x & 31;
    const int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (w >= rows) return;
    const int64_t bh = w / Nq;
    const int r = static_cast<int>(w % Nq);
    const int64_t beg = row_ptr[w], end = row_ptr[w + 1];
    if (!(beg >= 0 && end >= beg && end <= col_cap && end - beg <= Nc)) {
        if (lane == 0) atomicOr(status, kStatusBadIndex);
        return;
    }
    bool bad = false;
    for (int64_t e = beg + lane; e < end; e += 32) {
        const int c = col_idx[e];
        if (c < 0 || c >= Nc) {
            bad = true;
            continue;
        }
        const int64_t col = bh * Nc + c;
        atomicOr(bitmap + col * words + (r >> 5), 1u << (r & 31));
        atomicAdd(rawcnt + col, 1);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(status, kStatusBadIndex);
}

// Per column: number of distinct rows (popcount of its bitmap).
__global__ void __launch_bounds__(256) csc_count_kernel(const uint32_t* __restrict__ bitmap,
                                                        const int32_t* __restrict__ rawcnt,
                                                        int words, int64_t cols,
                                                        int32_t* __restrict__ cnt,
                                                        uint32_t* status) {
    const int64_t col = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (col >= cols) return;
    int n = 0;
    for (int i = 0; i < words; ++i) n += __popc(bitmap[col * words + i]);
    cnt[col] = n;
    if (n != rawcnt[col]) atomicOr(status, kStatusBadIndex);  // duplicate entry in a row
}

// One warp per column: writes its rows ascending at col_ptr[col].
__global__ void __launch_bounds__(256) csc_emit_kernel(const uint32_t* __restrict__ bitmap,
                                                       int words, int64_t cols,
                                                       const int32_t* __restrict__ col_ptr,
                                                       int32_t* __restrict__ row_idx,
                                                       int64_t idx_cap, uint32_t* status) {
    const int lane = threadIdx.x & 31;
    const int64_t col = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (col >= cols) return;
    const int64_t base = col_ptr[col];
    if (col_ptr[col + 1] > idx_cap) {
        if (lane == 0) atomicOr(status, kStatusCapacity);
        return;
    }
    int64_t run = 0;
    for (int w0 = 0; w0 < words; w0 += 32) {
        const int wi = w0 + lane;
        uint32_t bits = wi < words ? bitmap[col * words + wi] : 0u;
        const int n = __popc(bits);
        int incl = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int64_t pos = base + run + (incl - n);
        while (bits) {
            const int b = __ffs(bits) - 1;
            bits &= bits - 1;
            row_idx[pos++] = wi * 32 + b;
        }
        run += __shfl_sync(0xffffffffu, incl, 31);
    }
}

// ------------------------------------------------------------------ shared pieces
template <int D>
struct BwdCfg {
    static constexpr int kHalfBytes = 128 * 64 * 2;  // one TMA box: 128 tokens x 64 channels
    static constexpr int kHalves = D / 64;
    static constexpr int kTileBytes = kHalves * kHalfBytes;
    static constexpr int kMaxList = 2048;            // Nc limit of the library
    static constexpr int kThreads = 320;             // 8 softmax warps, TMA warp, MMA warp
    static constexpr int kTmaWarp = 8;
    static constexpr int kMmaWarp = 9;
    static constexpr uint32_t kTmemCols = 512;
    // six tiles, then (dK/dV kernel) three 1 KB per-query-chunk aux records, control, the
    // chunk list and (64-token query chunks) the quadrant pattern of each list entry
    static constexpr int kAux = 6 * kTileBytes;
    static constexpr int kCtl = kAux + 3 * 1024;
    static constexpr int kList = kCtl + 512;
    static constexpr int kPat = kList + kMaxList * 2;    // quadrant pattern per list entry
    static constexpr int kSmemBytes = kPat + kMaxList + 1024;  // + alignment slack
};

struct BwdArgs {
    const int32_t* row_ptr;   // CSR (dQ kernel)
    const int32_t* col_idx;
    int64_t col_cap;
    const int32_t* col_ptr;   // CSC (dK/dV kernel): local query rows per key chunk
    const int32_t* row_idx;
    int64_t idx_cap;
    const float* aux;         // [BH][Nq][half][LSE*log2(e) x64 | D x64]
    // 64-token query chunks (rows and key chunks are (4,4,8) boxes): the quadrant
    // pattern of every CSR entry and of every CSC entry (bit 2*hq + hk: the query
    // box's half hq attends to the key box's half hk; halves split w at 4)
    const uint8_t* row_pat;
    const uint8_t* col_pat;
    __nv_bfloat16* dq;        // for zero rows / columns written without TMA
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    uint32_t* status;
    int T, H, W, NH, NW, Nc;
    int q_skip, Nq;
    int64_t N;
    int64_t units;            // CTAs: CSR rows (dQ) or key chunks BH*Nc (dK/dV)
    float scale;
    float scale_log2;
    uint64_t timeout_ns;
    int debug_flags;          // bit 0: the dQ kernel, bit 1: the dK/dV kernel withholds
                              // its first S-ready signal (tests of the bounded waits)
};

// Rows of a 128 x D fp32 TMEM block (this thread's lane, columns from t_row)
// scaled by `mul`, rounded to bf16 and written as row m of a 128-byte-swizzled
// [128][64]-per-half staging tile (the layout of the 5-D TMA box).
template <int D>
__device__ __forceinline__ void stage_tmem_rows(uint32_t t_row, uint8_t* stage, int m, float mul,
                                                int g_begin = 0, int g_end = D / 32) {
    constexpr int kHalfBytes = 128 * 64 * 2;
#pragma unroll 1
    for (int g = g_begin; g < g_end; ++g) {
        uint32_t o[32];
        tmem_ld32(t_row + g * 32, o);
        tmem_wait_ld_tie(o);
        const int half = (g * 32) / 64;
        const int chunk0 = ((g * 32) % 64) / 8;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
            uint4 val;
            val.x = pack_bf16x2(__uint_as_float(o[c4 * 8 + 0]) * mul, __uint_as_float(o[c4 * 8 + 1]) * mul);
            val.y = pack_bf16x2(__uint_as_float(o[c4 * 8 + 2]) * mul, __uint_as_float(o[c4 * 8 + 3]) * mul);
            val.z = pack_bf16x2(__uint_as_float(o[c4 * 8 + 4]) * mul, __uint_as_float(o[c4 * 8 + 5]) * mul);
            val.w = pack_bf16x2(__uint_as_float(o[c4 * 8 + 6]) * mul, __uint_as_float(o[c4 * 8 + 7]) * mul);
            *reinterpret_cast<uint4*>(stage + half * kHalfBytes + m * 128 +
                                      (((chunk0 + c4) ^ (m & 7)) << 4)) = val;
        }
    }
}

// Zeros for local token m of the chunk at (t0, h0, w0) of head bh (nothing for
// a slot of a partial edge chunk past the grid).
template <int D>
__device__ __forceinline__ void zero_token(__nv_bfloat16* base, int64_t bh, int64_t N, int T,
                                           int H, int W, int t0, int h0, int w0, int m) {
    const int lt = m >> 5, lh = (m >> 3) & 3, lw = m & 7;
    if (t0 + lt >= T || h0 + lh >= H || w0 + lw >= W) return;
    const int64_t tok = (static_cast<int64_t>(t0 + lt) * H + (h0 + lh)) * W + w0 + lw;
    uint4* dst = reinterpret_cast<uint4*>(base + (bh * N + tok) * D);
#pragma unroll
    for (int j = 0; j < D / 8; ++j) dst[j] = make_uint4(0u, 0u, 0u, 0u);
}

// An mbarrier arrive that the 32 registers r depend on, and an empty statement
// that does the same for another 32: arithmetic on r cannot be scheduled above
// them, so an early release (S loaded, its TMEM columns free) is not delayed
// behind the work that follows it.
__device__ __forceinline__ void mbar_arrive_tied(uint64_t* bar, uint32_t (&r)[32]) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%32];"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 : "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void reg_tie(uint32_t (&r)[32]) {
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

// exp2 of a pair: every 4th pair on the FMA-pipe polynomial, the rest on MUFU.
__device__ __forceinline__ float2 exp2_pair(float2 x, int j) {
    return (j % 4 == 0) ? exp2_poly2(x) : make_float2(ex2_approx(x.x), ex2_approx(x.y));
}

// ------------------------------------------------------------------ dQ kernel
// One CTA per CSR row (query chunk). Q and dO are the A operands of every S and
// dP of the row, so after the TMA lands them the dS warps copy both into TMEM
// (bf16 pairs, one row per lane): S = Q K^T and dP = dO V^T then read only
// their B operand from shared memory. TMEM: Q at columns [0,64), dO at
// [64,128), S at [128,256), dP at [256,384), dQ at [384,512). Shared memory:
// Q's tile (a V slot once copied), dO's tile (dQ staging at the end), a
// three-slot K ring and a second V slot.
//
// The 8 dS warps split each row: warps w and w+4 share TMEM lanes 32(w%4)..
// and take key columns [0,64) and [64,128). A step has two phases. First they
// load S, release it (s_free: S of the next key chunk is computed in its place)
// and compute P = exp2(S * scale * log2(e) - LSE * log2(e)) into registers;
// then they load dP and write dS = P (dP - D) as packed bf16 over the first
// half of their dP columns, the TMEM A operand of dQ += dS K. MMA issue order
// per step j: S(j+1) once S(j) is loaded, dQ(j) once dS(j) is written, then
// dP(j+1) (the tensor core executes in issue order, so dP(j+1) overwrites dS(j)
// only after dQ(j) has read it). While the warps compute P(j+1), dQ(j) and
// dP(j+1) are queued. Two producer lanes keep the loads independent: lane 0
// refills K slots (K(j+3) after dQ(j)), lane 1 the V slots (V(j+2) after
// dP(j)).
struct __align__(8) DqCtl {
    uint64_t qd_full, qt_full, k_full[3], k_empty[3], v_full[2], v_empty[2];
    uint64_t s_full, s_free, dp_full, ds_full, dq_full, aux;
    int n_valid;
    uint32_t tmem_base;
    int abort_flag;
};

// Copy row m of a [128][64]-per-half 128-byte-swizzled bf16 tile (the layout of
// the 5-D TMA box), channels [64*half, 64*half + 64), into 32 TMEM columns as
// bf16 pairs (even channel in the low half), the layout of an A operand.
__device__ __forceinline__ void tile_row_to_tmem(const uint8_t* tile, int half, int m, uint32_t taddr) {
    constexpr int kHalfBytes = 128 * 64 * 2;
    const uint8_t* row = tile + half * kHalfBytes + m * 128;
    uint32_t r[32];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + ((c ^ (m & 7)) << 4));
        r[4 * c + 0] = v.x;
        r[4 * c + 1] = v.y;
        r[4 * c + 2] = v.z;
        r[4 * c + 3] = v.w;
    }
    tmem_st32(taddr, r);
}

template <int D, bool kQuad>
__global__ void __launch_bounds__(320, 1)
    bsa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                      const __grid_constant__ CUtensorMap tm_dq, const BwdArgs a) {
    using C = BwdCfg<D>;
    constexpr uint32_t kQt = 0, kDOt = 64, kS = 128, kDP = 256, kDQ = 384;  // TMEM columns
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sQ = smem;                    // then V slot 1
    uint8_t* sdO = smem + C::kTileBytes;   // then dQ staging
    auto sK = [&](int s) { return smem + (2 + s) * C::kTileBytes; };
    auto sV = [&](int s) { return s == 0 ? smem + 5 * C::kTileBytes : sQ; };
    DqCtl* ctl = reinterpret_cast<DqCtl*>(smem + C::kCtl);
    uint16_t* list = reinterpret_cast<uint16_t*>(smem + C::kList);
    uint8_t* plist = smem + C::kPat;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t row = blockIdx.x;

    if (threadIdx.x == 0) {
        mbar_init(&ctl->qd_full, 1);
        mbar_init(&ctl->qt_full, 256);
        for (int s = 0; s < 3; ++s) {
            mbar_init(&ctl->k_full[s], 1);
            mbar_init(&ctl->k_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&ctl->v_full[s], 1);
            mbar_init(&ctl->v_empty[s], 1);
        }
        mbar_init(&ctl->s_full, 1);
        mbar_init(&ctl->s_free, 256);
        mbar_init(&ctl->dp_full, 1);
        mbar_init(&ctl->ds_full, 256);
        mbar_init(&ctl->dq_full, 1);
        mbar_init(&ctl->aux, 1);
        ctl->abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == C::kTmaWarp) {
        // stage the row's chunk list (out-of-range entries dropped and reported)
        bool bad = false;
        int64_t beg = a.row_ptr[row], end = a.row_ptr[row + 1];
        if (!(beg >= 0 && end >= beg && end <= a.col_cap && end - beg <= a.Nc)) {
            bad = true;
            beg = end = 0;
        }
        int cnt = 0;
        for (int64_t e0 = beg; e0 < end; e0 += 32) {
            const int64_t e = e0 + lane;
            const int c = e < end ? a.col_idx[e] : 0;
            const bool valid = e < end && c >= 0 && c < a.Nc;
            if (e < end && !valid) bad = true;
            const uint32_t vb = __ballot_sync(0xffffffffu, valid);
            if (valid) {
                const int slot = cnt + __popc(vb & ((1u << lane) - 1u));
                list[slot] = static_cast<uint16_t>(c);
                if constexpr (kQuad) plist[slot] = a.row_pat[e];
            }
            cnt += __popc(vb);
        }
        if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(a.status, kStatusBadIndex);
        if (lane == 0) {
            ctl->n_valid = cnt;
            prefetch_tensormap(&tm_q);
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
            prefetch_tensormap(&tm_do);
            prefetch_tensormap(&tm_dq);
        }
    }
    if (warp == C::kMmaWarp) {
        tmem_alloc(&ctl->tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    const int n = ctl->n_valid;
    volatile int* abort_flag = &ctl->abort_flag;
    const uint64_t tmo = a.timeout_ns;
    const int bh = static_cast<int>(row / a.Nq);
    const int r_local = static_cast<int>(row % a.Nq);
    int q_t, q_h, q_w;
    chunk_origin(a.q_skip + r_local, a.NH, a.NW, q_t, q_h, q_w);
    // what this thread put in flight (K and V copies per slot; any product), for
    // the drain after an abort
    int nk[3] = {0, 0, 0}, nv[2] = {0, 0};
    bool issued = false;

    if (warp == C::kTmaWarp) {
        // ------------------------------------------------------------ TMA producers
        if (lane == 0 && n > 0) {
            // Q, dO, then the K ring
            mbar_arrive_expect_tx(&ctl->qd_full, 2 * C::kTileBytes);
#pragma unroll
            for (int c = 0; c < C::kHalves; ++c) {
                tma_load_5d(&tm_q, smem_u32(sQ) + c * C::kHalfBytes, &ctl->qd_full, c * 64, q_w,
                            q_h, q_t, bh);
                tma_load_5d(&tm_do, smem_u32(sdO) + c * C::kHalfBytes, &ctl->qd_full, c * 64, q_w,
                            q_h, q_t, bh);
            }
            bool ok = true;
            for (int j = 0; j < n && ok; ++j) {
                const int s = j % 3;
                if (j >= 3 && !mbar_wait(&ctl->k_empty[s], ((j - 3) / 3) & 1, abort_flag, a.status,
                                         tmo, site(1, 1, s, j))) {
                    ok = false;
                    break;
                }
                int kt, kh, kw;
                chunk_origin(list[j], a.NH, a.NW, kt, kh, kw);
                mbar_arrive_expect_tx(&ctl->k_full[s], C::kTileBytes);
#pragma unroll
                for (int c = 0; c < C::kHalves; ++c)
                    tma_load_5d(&tm_k, smem_u32(sK(s)) + c * C::kHalfBytes, &ctl->k_full[s], c * 64,
                                kw, kh, kt, bh);
                ++nk[s];
            }
        } else if (lane == 1 && n > 0) {
            // the V slots: V(0) in its own tile, V(1) in Q's once Q is in TMEM, then
            // V(j) once dP(j-2) has read V(j-2)
            bool ok = true;
            for (int j = 0; j < n && ok; ++j) {
                const int s = j & 1;
                if (j == 1 && !mbar_wait(&ctl->qt_full, 0, abort_flag, a.status, tmo, site(1, 3, 0, j))) {
                    ok = false;
                    break;
                }
                if (j >= 2 && !mbar_wait(&ctl->v_empty[s], ((j - 2) >> 1) & 1, abort_flag, a.status,
                                         tmo, site(1, 2, s, j))) {
                    ok = false;
                    break;
                }
                int vt, vh, vw;
                chunk_origin(list[j], a.NH, a.NW, vt, vh, vw);
                mbar_arrive_expect_tx(&ctl->v_full[s], C::kTileBytes);
#pragma unroll
                for (int c = 0; c < C::kHalves; ++c)
                    tma_load_5d(&tm_v, smem_u32(sV(s)) + c * C::kHalfBytes, &ctl->v_full[s], c * 64,
                                vw, vh, vt, bh);
                ++nv[s];
            }
        }
        __syncwarp();
    } else if (warp == C::kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n > 0) {
            constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, 0, 0);  // A from TMEM, B K-major
            constexpr uint32_t kIdQ = idesc_bf16_f32(128, D, 0, 1);    // dS from TMEM, K MN-major
            bool ok = mbar_wait(&ctl->qt_full, 0, abort_flag, a.status, tmo, site(2, 0, 0, 0));
            if (ok) tc_fence_after();
            // G = A B^T over the D channels: A (Q or dO) in TMEM at acol, B in shared memory
            auto issue_tk = [&](uint32_t dcol, uint32_t acol, uint32_t sb) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kHalfBytes + (kk & 3) * 32;
                    mma_ts(tmem + dcol, tmem + acol + 8u * kk, sdesc_sw128(sb + off, 16, 1024), kIdS,
                           kk > 0 ? 1u : 0u);
                }
            };
            // S(j) = Q K(j)^T. Past the first step the dS warps have seen K(j) land before
            // releasing S(j-1), so the wait on s_free covers it.
            auto issue_s = [&](int j) -> bool {
                const int s = j % 3;
                if (j == 0 && !mbar_wait(&ctl->k_full[s], 0, abort_flag, a.status, tmo, site(2, 1, s, j)))
                    return false;
                issue_tk(kS, kQt, smem_u32(sK(s)));
                issued = true;
                if (!((a.debug_flags & 1) && j == 0)) tc_commit(&ctl->s_full);
                return true;
            };
            // dP(j) = dO V(j)^T. Past the first step the dS warps have seen V(j) land before
            // arriving on ds_full for step j-1.
            auto issue_dp = [&](int j) -> bool {
                const int s = j & 1;
                if (j == 0 && !mbar_wait(&ctl->v_full[s], 0, abort_flag, a.status, tmo, site(2, 2, s, j)))
                    return false;
                issue_tk(kDP, kDOt, smem_u32(sV(s)));
                issued = true;
                tc_commit(&ctl->v_empty[s]);
                tc_commit(&ctl->dp_full);
                return true;
            };
            // dQ += dS(j) K(j): keys 16kk.. of dS sit at column 64*(kk/4) + 8*(kk%4) of dP's block
            auto issue_dq = [&](int j) {
                const int s = j % 3;
                const uint32_t sk = smem_u32(sK(s));
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tmem + kDQ, tmem + kDP + 64u * (kk >> 2) + 8u * (kk & 3),
                           sdesc_sw128(sk + kk * 2048, C::kHalfBytes, 1024), kIdQ,
                           (j > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&ctl->k_empty[s]);
            };
            ok = ok && issue_s(0) && issue_dp(0);
            for (int j = 0; j < n && ok; ++j) {
                if (j + 1 < n) {
                    // S(j) is in the dS warps' registers: compute S(j+1) in its place
                    if (!mbar_wait(&ctl->s_free, j & 1, abort_flag, a.status, tmo, site(2, 4, 0, j))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (!issue_s(j + 1)) { ok = false; break; }
                }
                if (!mbar_wait(&ctl->ds_full, j & 1, abort_flag, a.status, tmo, site(2, 3, 0, j))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                issue_dq(j);
                if (j + 1 < n && !issue_dp(j + 1)) { ok = false; break; }
            }
            if (ok) tc_commit(&ctl->dq_full);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ Q, dO to TMEM; dS; epilogue
        const int grp = warp >> 2;                    // key columns [64*grp, 64*grp + 64)
        const int m = (warp & 3) * 32 + lane;         // query row = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const float* aux_row = a.aux + (static_cast<int64_t>(bh) * a.Nq + r_local) * 256 +
                               (m >> 6) * 128 + (m & 63);
        const float lse2 = aux_row[0];
        const float Dm = aux_row[64];
        const float2 cc = make_float2(a.scale_log2, a.scale_log2);
        const float2 nl = make_float2(-lse2, -lse2);
        const float2 nd = make_float2(-Dm, -Dm);
        bool ok = true;
        if (n > 0) {
            // warp group g copies channel half g of Q and dO (D = 64: group 0 only)
            const bool got = mbar_wait(&ctl->qd_full, 0, abort_flag, a.status, tmo, site(3, 0, 0, 0));
            ok = __all_sync(0xffffffffu, got);
            if (ok && grp < C::kHalves) {
                tile_row_to_tmem(sQ, grp, m, tmem + lane_off + kQt + 32u * grp);
                tile_row_to_tmem(sdO, grp, m, tmem + lane_off + kDOt + 32u * grp);
                tmem_wait_st();
            }
            if (ok) {
                tc_fence_before();
                mbar_arrive(&ctl->qt_full);
            }
        }
        const uint32_t tS = tmem + lane_off + kS + 64u * grp;
        const uint32_t tP = tmem + lane_off + kDP + 64u * grp;
        for (int j = 0; j < n && ok; ++j) {
            // P phase
            bool got = mbar_wait(&ctl->s_full, j & 1, abort_flag, a.status, tmo, site(3, 4, 0, j));
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
            // 64-token query chunks: the key halves this query row attends to in this box
            // (its query half is bit 2 of its w index); masked weights are set to 0
            // after the exponential, so they never enter any arithmetic
            bool keep_a = true, keep_b = true;
            if constexpr (kQuad) {
                const uint32_t mine = (plist[j] >> ((m & 4) ? 2 : 0)) & 3u;
                keep_a = mine & 1u;
                keep_b = mine & 2u;
            }
            float p[64];
            {
                uint32_t sv0[32], sv1[32];
                tmem_ld32(tS, sv0);
                tmem_ld32(tS + 32, sv1);
                tmem_wait_ld_tie(sv0);
                tmem_wait_ld_tie(sv1);
                // S of this step is in registers: its columns may be overwritten. K(j+1) has
                // landed (seen here, so the MMA thread need not wait for it) before S(j+1).
                const bool k_in = j + 1 >= n || mbar_wait(&ctl->k_full[(j + 1) % 3], ((j + 1) / 3) & 1,
                                                          abort_flag, a.status, tmo, site(3, 1, (j + 1) % 3, j));
                if (!__all_sync(0xffffffffu, k_in)) { ok = false; break; }
                tc_fence_before();
                mbar_arrive_tied(&ctl->s_free, sv0);
                reg_tie(sv1);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const uint32_t* sv = e < 16 ? sv0 : sv1;
                    const int o = 2 * (e & 15);
                    const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[o]), __uint_as_float(sv[o + 1])),
                                                cc, nl);
                    float2 pe = exp2_pair(x, e);
                    // pair e holds key slots whose w index has bit 2 equal to bit 1 of e
                    if constexpr (kQuad)
                        if (!((e & 2) ? keep_b : keep_a)) pe = make_float2(0.0f, 0.0f);
                    p[2 * e] = pe.x;
                    p[2 * e + 1] = pe.y;
                }
            }
            // dS phase
            got = mbar_wait(&ctl->dp_full, j & 1, abort_flag, a.status, tmo, site(3, 5, 0, j));
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
            uint32_t pk[32];
            {
                uint32_t dv0[32], dv1[32];
                tmem_ld32(tP, dv0);
                tmem_ld32(tP + 32, dv1);
                tmem_wait_ld_tie(dv0);
                tmem_wait_ld_tie(dv1);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const uint32_t* dv = e < 16 ? dv0 : dv1;
                    const int o = 2 * (e & 15);
                    const float2 dp = __fadd2_rn(make_float2(__uint_as_float(dv[o]), __uint_as_float(dv[o + 1])),
                                                 nd);
                    const float2 ds = __fmul2_rn(make_float2(p[2 * e], p[2 * e + 1]), dp);
                    pk[e] = pack_bf16x2(ds.x, ds.y);
                }
            }
            // dS over the first 32 of this warp's dP columns: both halves are in registers
            tmem_st32(tP, pk);
            tmem_wait_st();
            // V(j+1) has landed (seen here for the MMA thread) before dP(j+1)
            const bool v_in = j + 1 >= n || mbar_wait(&ctl->v_full[(j + 1) & 1], ((j + 1) >> 1) & 1,
                                                      abort_flag, a.status, tmo, site(3, 2, (j + 1) & 1, j));
            if (!__all_sync(0xffffffffu, v_in)) { ok = false; break; }
            tc_fence_before();
            mbar_arrive(&ctl->ds_full);
        }
        if (ok && n > 0) {
            const bool got = mbar_wait(&ctl->dq_full, 0, abort_flag, a.status, tmo, site(3, 6, 0, 0));
            ok = __all_sync(0xffffffffu, got);
        }
        const bool all_ok = bar_red_and(1, 256, ok);
        if (all_ok && n > 0) {
            tc_fence_after();
            // dO's tile is dead once it is in TMEM; each warp group stages half the columns
            stage_tmem_rows<D>(tmem + lane_off + kDQ, sdO, m, a.scale, grp * D / 64, (grp + 1) * D / 64);
            fence_proxy_async_smem();
            named_bar_sync(1, 256);
            if (threadIdx.x == 0) {
#pragma unroll
                for (int c = 0; c < C::kHalves; ++c)
                    tma_store_5d(&tm_dq, smem_u32(sdO) + c * C::kHalfBytes, c * 64, q_w, q_h, q_t, bh);
                tma_store_commit_and_wait_all();
            }
        } else if (all_ok && grp == 0) {
            zero_token<D>(a.dq, bh, a.N, a.T, a.H, a.W, q_t, q_h, q_w, m);  // no selected chunk
        }
    }

    tc_fence_before();
    __syncthreads();
    // After an abort (the flag no longer changes here, whichever role gave up and
    // whenever), the copies and products still in flight land before the CTA's
    // shared memory and TMEM are released.
    if (*abort_flag) {
        if (warp == C::kTmaWarp) {
            if (lane == 0 && n > 0) drain_wait(&ctl->qd_full, 0, tmo);
            for (int s = 0; s < 3; ++s)
                if (nk[s] > 0) drain_wait(&ctl->k_full[s], (nk[s] - 1) & 1, tmo);
            for (int s = 0; s < 2; ++s)
                if (nv[s] > 0) drain_wait(&ctl->v_full[s], (nv[s] - 1) & 1, tmo);
        } else if (warp == C::kMmaWarp && issued) {
            tc_commit(&ctl->aux);
            drain_wait(&ctl->aux, 0, tmo);
        }
    }
    if (warp == C::kMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ------------------------------------------------------------------ dK/dV kernel
// One CTA per key chunk (CSC column). K and V stay resident; the query chunks
// that selected the key chunk come through two-slot Q and dO rings, each Q with
// its 1 KB aux record (LSE * log2(e) and D of its 128 queries: column q of S^T,
// half q / 64). The 8 exponential warps split each step: warps w and w+4 share
// TMEM lanes 32(w%4).. (key rows) and take query columns [0,64) and [64,128),
// the halves of the aux record. All four products are M = 128 keys x N = 128.
//
// TMEM: S^T = K Q^T at [0,128), dP^T = V dO^T at [128,256), dV at [256,384), dK
// at [384,512). A step has two phases on separate barriers. P phase: the warps
// load S^T, write P^T = exp2(S^T * scale * log2(e) - LSE * log2(e)) as packed
// bf16 over the first half of their S^T columns (the TMEM A operand of
// dV += P^T dO) and keep P in registers. dS phase: they load dP^T and write
// dS^T = P^T (dP^T - D) over the first half of their dP^T columns (the A operand
// of dK += dS^T Q). MMA issue order per step i: dV(i) and S^T(i+1) once P^T(i)
// is written, then dK(i) and dP^T(i+1) once dS^T(i) is written. The tensor
// core executes in issue order, so S^T(i+1) overwrites P^T(i) only after dV(i)
// has read it (and likewise dP^T(i+1) after dK(i)); while the warps run the dS
// phase of step i, dV(i) and S^T(i+1) are queued, and while they run the P
// phase of step i+1, dK(i) and dP^T(i+1). Before their dS-phase arrival the
// warps check that dO(i+1) has landed (requested a step earlier), so the MMA
// thread does not wait for it.
struct __align__(8) DkvCtl {
    uint64_t kv_full, q_full[2], q_empty[2], do_full[2], do_empty[2];
    uint64_t s_full, dp_full, p_full, ds_full, dkv_full, aux;
    int n_valid;
    uint32_t tmem_base;
    int abort_flag;
};

// Stage a CSC column's query rows (and, for 64-token query chunks, their
// quadrant patterns) in shared memory (out-of-range entries dropped and
// reported); returns the count on lane 0 (every lane of the calling warp takes
// part).
template <bool kQuad>
__device__ __forceinline__ int stage_column(const BwdArgs& a, int64_t col, uint16_t* list,
                                            uint8_t* plist, int lane) {
    bool bad = false;
    int64_t beg = a.col_ptr[col], end = a.col_ptr[col + 1];
    if (!(beg >= 0 && end >= beg && end <= a.idx_cap && end - beg <= a.Nq)) {
        bad = true;
        beg = end = 0;
    }
    int cnt = 0;
    for (int64_t e0 = beg; e0 < end; e0 += 32) {
        const int64_t e = e0 + lane;
        const int r = e < end ? a.row_idx[e] : 0;
        const bool valid = e < end && r >= 0 && r < a.Nq;
        if (e < end && !valid) bad = true;
        const uint32_t vb = __ballot_sync(0xffffffffu, valid);
        if (valid) {
            const int slot = cnt + __popc(vb & ((1u << lane) - 1u));
            list[slot] = static_cast<uint16_t>(r);
            if constexpr (kQuad) plist[slot] = a.col_pat[e];
        }
        cnt += __popc(vb);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(a.status, kStatusBadIndex);
    return cnt;
}

template <int D, bool kQuad>
__global__ void __launch_bounds__(320, 1)
    bsa_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                       const BwdArgs a) {
    using C = BwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sK = smem;
    uint8_t* sV = smem + C::kTileBytes;
    auto sQ = [&](int s) { return smem + (2 + s) * C::kTileBytes; };
    auto sdO = [&](int s) { return smem + (4 + s) * C::kTileBytes; };
    float* sAux = reinterpret_cast<float*>(smem + C::kAux);  // [slot][half][lse2 64 | D 64]
    DkvCtl* ctl = reinterpret_cast<DkvCtl*>(smem + C::kCtl);
    uint16_t* list = reinterpret_cast<uint16_t*>(smem + C::kList);
    uint8_t* plist = smem + C::kPat;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t col = blockIdx.x;
    const int bh = static_cast<int>(col / a.Nc);
    const int kc = static_cast<int>(col % a.Nc);

    if (threadIdx.x == 0) {
        mbar_init(&ctl->kv_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&ctl->q_full[s], 1);
            mbar_init(&ctl->q_empty[s], 1);
            mbar_init(&ctl->do_full[s], 1);
            mbar_init(&ctl->do_empty[s], 1);
        }
        mbar_init(&ctl->s_full, 1);
        mbar_init(&ctl->dp_full, 1);
        mbar_init(&ctl->p_full, 256);
        mbar_init(&ctl->ds_full, 256);
        mbar_init(&ctl->dkv_full, 1);
        mbar_init(&ctl->aux, 1);
        ctl->abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == C::kTmaWarp) {
        const int cnt = stage_column<kQuad>(a, col, list, plist, lane);
        if (lane == 0) {
            ctl->n_valid = cnt;
            prefetch_tensormap(&tm_q);
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
            prefetch_tensormap(&tm_do);
            prefetch_tensormap(&tm_dk);
            prefetch_tensormap(&tm_dv);
        }
    }
    if (warp == C::kMmaWarp) {
        tmem_alloc(&ctl->tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    const int n = ctl->n_valid;
    volatile int* abort_flag = &ctl->abort_flag;
    const uint64_t tmo = a.timeout_ns;
    int k_t, k_h, k_w;
    chunk_origin(kc, a.NH, a.NW, k_t, k_h, k_w);
    // what this thread put in flight (Q and dO copies per slot; any product), for
    // the drain after an abort
    int nq[2] = {0, 0}, nd[2] = {0, 0};
    bool issued = false;

    if (warp == C::kTmaWarp) {
        // ------------------------------------------------------------ TMA producers
        if (lane == 0 && n > 0) {
            // K and V, then the Q ring with each query chunk's aux record (Q(i+2) once
            // dK(i) has read Q(i); the warps have read the record by then)
            mbar_arrive_expect_tx(&ctl->kv_full, 2 * C::kTileBytes);
#pragma unroll
            for (int c = 0; c < C::kHalves; ++c) {
                tma_load_5d(&tm_k, smem_u32(sK) + c * C::kHalfBytes, &ctl->kv_full, c * 64, k_w, k_h,
                            k_t, bh);
                tma_load_5d(&tm_v, smem_u32(sV) + c * C::kHalfBytes, &ctl->kv_full, c * 64, k_w, k_h,
                            k_t, bh);
            }
            bool ok = true;
            for (int i = 0; i < n && ok; ++i) {
                const int s = i & 1;
                if (i >= 2 && !mbar_wait(&ctl->q_empty[s], ((i - 2) >> 1) & 1, abort_flag, a.status,
                                         tmo, site(1, 1, s, i))) {
                    ok = false;
                    break;
                }
                const int r = list[i];
                int qt, qh, qw;
                chunk_origin(a.q_skip + r, a.NH, a.NW, qt, qh, qw);
                mbar_arrive_expect_tx(&ctl->q_full[s], C::kTileBytes + 1024);
#pragma unroll
                for (int c = 0; c < C::kHalves; ++c)
                    tma_load_5d(&tm_q, smem_u32(sQ(s)) + c * C::kHalfBytes, &ctl->q_full[s], c * 64,
                                qw, qh, qt, bh);
                bulk_load(smem_u32(sAux + s * 256), a.aux + (static_cast<int64_t>(bh) * a.Nq + r) * 256,
                          1024, &ctl->q_full[s]);
                ++nq[s];
            }
        } else if (lane == 1 && n > 0) {
            // the dO ring: dO(i+2) once dV(i) has read dO(i)
            bool ok = true;
            for (int i = 0; i < n && ok; ++i) {
                const int s = i & 1;
                if (i >= 2 && !mbar_wait(&ctl->do_empty[s], ((i - 2) >> 1) & 1, abort_flag, a.status,
                                         tmo, site(1, 2, s, i))) {
                    ok = false;
                    break;
                }
                int qt, qh, qw;
                chunk_origin(a.q_skip + list[i], a.NH, a.NW, qt, qh, qw);
                mbar_arrive_expect_tx(&ctl->do_full[s], C::kTileBytes);
#pragma unroll
                for (int c = 0; c < C::kHalves; ++c)
                    tma_load_5d(&tm_do, smem_u32(sdO(s)) + c * C::kHalfBytes, &ctl->do_full[s], c * 64,
                                qw, qh, qt, bh);
                ++nd[s];
            }
        }
        __syncwarp();
    } else if (warp == C::kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n > 0) {
            constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, 0, 0);  // both operands K-major
            constexpr uint32_t kIdG = idesc_bf16_f32(128, D, 0, 1);    // A from TMEM, B MN-major
            bool ok = mbar_wait(&ctl->kv_full, 0, abort_flag, a.status, tmo, site(2, 0, 0, 0));
            if (ok) tc_fence_after();
            auto issue_ss = [&](uint32_t dcol, uint32_t sa, uint32_t sb) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kHalfBytes + (kk & 3) * 32;
                    mma_ss(tmem + dcol, sdesc_sw128(sa + off, 16, 1024), sdesc_sw128(sb + off, 16, 1024),
                           kIdS, kk > 0 ? 1u : 0u);
                }
            };
            // G += A B over 128 queries: queries 16kk.. of A sit at column 64*(kk/4) + 8*(kk%4)
            // of the TMEM block at acol; B is the query chunk's tile at sb
            auto issue_ts = [&](uint32_t dcol, uint32_t acol, uint32_t sb, bool first) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tmem + dcol, tmem + acol + 64u * (kk >> 2) + 8u * (kk & 3),
                           sdesc_sw128(sb + kk * 2048, C::kHalfBytes, 1024), kIdG,
                           (!first || kk > 0) ? 1u : 0u);
            };
            // S^T(i) = K Q(i)^T
            auto issue_st = [&](int i) -> bool {
                const int s = i & 1;
                if (!mbar_wait(&ctl->q_full[s], (i >> 1) & 1, abort_flag, a.status, tmo,
                               site(2, 1, s, i)))
                    return false;
                tc_fence_after();
                issue_ss(0u, smem_u32(sK), smem_u32(sQ(s)));
                issued = true;
                if (!((a.debug_flags & 2) && i == 0)) tc_commit(&ctl->s_full);
                return true;
            };
            // dP^T(i) = V dO(i)^T. Past the first step the warps have seen dO(i) land before
            // arriving on ds_full for step i-1.
            auto issue_dpt = [&](int i) -> bool {
                const int s = i & 1;
                if (i == 0 && !mbar_wait(&ctl->do_full[0], 0, abort_flag, a.status, tmo, site(2, 2, 0, 0)))
                    return false;
                issue_ss(128u, smem_u32(sV), smem_u32(sdO(s)));
                issued = true;
                tc_commit(&ctl->dp_full);
                return true;
            };
            ok = ok && issue_st(0) && issue_dpt(0);
            for (int i = 0; i < n && ok; ++i) {
                const int s = i & 1;
                if (!mbar_wait(&ctl->p_full, i & 1, abort_flag, a.status, tmo, site(2, 3, 0, i))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                issue_ts(256u, 0u, smem_u32(sdO(s)), i == 0);   // dV += P^T(i) dO(i)
                tc_commit(&ctl->do_empty[s]);
                if (i + 1 < n && !issue_st(i + 1)) { ok = false; break; }
                if (!mbar_wait(&ctl->ds_full, i & 1, abort_flag, a.status, tmo, site(2, 4, 0, i))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                issue_ts(384u, 128u, smem_u32(sQ(s)), i == 0);  // dK += dS^T(i) Q(i)
                tc_commit(&ctl->q_empty[s]);
                if (i + 1 < n && !issue_dpt(i + 1)) { ok = false; break; }
            }
            if (ok) tc_commit(&ctl->dkv_full);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ P^T, dS^T + epilogue
        const int grp = warp >> 2;                    // query columns [64*grp, 64*grp + 64)
        const int m = (warp & 3) * 32 + lane;         // key row = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + 64u * grp;
        const uint32_t tP = tS + 128u;
        const float2 cc = make_float2(a.scale_log2, a.scale_log2);
        bool ok = true;
        for (int i = 0; i < n; ++i) {
            const int s = i & 1;
            // P phase. The aux record arrived with Q(i), before S^T(i) could start: its 64
            // LSE * log2(e) values for this group's queries are loaded while S^T(i) runs.
            bool got = mbar_wait(&ctl->q_full[s], (i >> 1) & 1, abort_flag, a.status, tmo,
                                 site(3, 3, s, i));
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            const float* lse2 = sAux + s * 256 + grp * 128;  // this group's 64 queries
            const float* Dq = lse2 + 64;
            float4 l4v[16];
#pragma unroll
            for (int e4 = 0; e4 < 16; ++e4) l4v[e4] = *reinterpret_cast<const float4*>(lse2 + 4 * e4);
            got = mbar_wait(&ctl->s_full, i & 1, abort_flag, a.status, tmo, site(3, 4, 0, i));
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
            // 64-token query chunks: which query halves this key row (its half is bit 2
            // of its w index) is attended by in this box pair; masked weights are set
            // to 0 after the exponential
            bool keep_q0 = true, keep_q1 = true;
            if constexpr (kQuad) {
                const uint32_t pat = plist[i], hk = (m & 4) ? 1u : 0u;
                keep_q0 = (pat >> hk) & 1u;
                keep_q1 = (pat >> (2u + hk)) & 1u;
            }
            float p[64];
            uint32_t pk[32];
            {
                uint32_t sv0[32], sv1[32];
                tmem_ld32(tS, sv0);
                tmem_ld32(tS + 32, sv1);
                tmem_wait_ld_tie(sv0);
                tmem_wait_ld_tie(sv1);
#pragma unroll
                for (int e4 = 0; e4 < 16; ++e4) {
                    const float4 l4 = l4v[e4];
                    const uint32_t* sv = e4 < 8 ? sv0 : sv1;
                    const int o = (e4 & 7) * 4;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float2 x = __ffma2_rn(
                            make_float2(__uint_as_float(sv[o + 2 * h]), __uint_as_float(sv[o + 2 * h + 1])),
                            cc, h == 0 ? make_float2(-l4.x, -l4.y) : make_float2(-l4.z, -l4.w));
                        float2 pe = exp2_pair(x, 2 * e4 + h);
                        // columns 4*e4 + 2h, +1: query w index with bit 2 equal to bit 0 of e4
                        if constexpr (kQuad)
                            if (!((e4 & 1) ? keep_q1 : keep_q0)) pe = make_float2(0.0f, 0.0f);
                        p[4 * e4 + 2 * h] = pe.x;
                        p[4 * e4 + 2 * h + 1] = pe.y;
                        pk[2 * e4 + h] = pack_bf16x2(pe.x, pe.y);
                    }
                }
            }
            // P^T over the first 32 of this warp's S^T columns: both halves were read
            tmem_st32(tS, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&ctl->p_full);
            // dS phase
            got = mbar_wait(&ctl->dp_full, i & 1, abort_flag, a.status, tmo, site(3, 5, 0, i));
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
            {
                uint32_t dv0[32], dv1[32];
                tmem_ld32(tP, dv0);
                tmem_ld32(tP + 32, dv1);
                tmem_wait_ld_tie(dv0);
                tmem_wait_ld_tie(dv1);
#pragma unroll
                for (int e4 = 0; e4 < 16; ++e4) {
                    const float4 d4 = *reinterpret_cast<const float4*>(Dq + 4 * e4);
                    const uint32_t* dv = e4 < 8 ? dv0 : dv1;
                    const int o = (e4 & 7) * 4;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float2 dp = __fadd2_rn(
                            make_float2(__uint_as_float(dv[o + 2 * h]), __uint_as_float(dv[o + 2 * h + 1])),
                            h == 0 ? make_float2(-d4.x, -d4.y) : make_float2(-d4.z, -d4.w));
                        const float2 ds = __fmul2_rn(
                            make_float2(p[4 * e4 + 2 * h], p[4 * e4 + 2 * h + 1]), dp);
                        pk[2 * e4 + h] = pack_bf16x2(ds.x, ds.y);
                    }
                }
            }
            tmem_st32(tP, pk);
            tmem_wait_st();
            // dO(i+1) has landed (seen here for the MMA thread) before dP^T(i+1)
            got = i + 1 >= n || mbar_wait(&ctl->do_full[(i + 1) & 1], ((i + 1) >> 1) & 1, abort_flag,
                                          a.status, tmo, site(3, 2, (i + 1) & 1, i));
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_before();
            mbar_arrive(&ctl->ds_full);
        }
        if (ok && n > 0) {
            const bool got = mbar_wait(&ctl->dkv_full, 0, abort_flag, a.status, tmo, site(3, 6, 0, 0));
            ok = __all_sync(0xffffffffu, got);
        }
        const bool all_ok = bar_red_and(1, 256, ok);
        if (all_ok && n > 0) {
            tc_fence_after();
            // K and V are dead once every MMA has completed; each warp group stages half
            // the columns of dK (into K's tile) and dV (into V's)
            stage_tmem_rows<D>(tmem + lane_off + 384u, sK, m, a.scale, grp * D / 64, (grp + 1) * D / 64);
            stage_tmem_rows<D>(tmem + lane_off + 256u, sV, m, 1.0f, grp * D / 64, (grp + 1) * D / 64);
            fence_proxy_async_smem();
            named_bar_sync(1, 256);
            if (threadIdx.x == 0) {
#pragma unroll
                for (int c = 0; c < C::kHalves; ++c) {
                    tma_store_5d(&tm_dk, smem_u32(sK) + c * C::kHalfBytes, c * 64, k_w, k_h, k_t, bh);
                    tma_store_5d(&tm_dv, smem_u32(sV) + c * C::kHalfBytes, c * 64, k_w, k_h, k_t, bh);
                }
                tma_store_commit_and_wait_all();
            }
        } else if (all_ok && grp == 0) {
            zero_token<D>(a.dk, bh, a.N, a.T, a.H, a.W, k_t, k_h, k_w, m);  // never selected
        } else if (all_ok) {
            zero_token<D>(a.dv, bh, a.N, a.T, a.H, a.W, k_t, k_h, k_w, m);
        }
    }

    tc_fence_before();
    __syncthreads();
    // After an abort (final here), the copies and products still in flight land
    // before the CTA's shared memory and TMEM are released.
    if (*abort_flag) {
        if (warp == C::kTmaWarp) {
            if (lane == 0 && n > 0) drain_wait(&ctl->kv_full, 0, tmo);
            for (int s = 0; s < 2; ++s) {
                if (nq[s] > 0) drain_wait(&ctl->q_full[s], (nq[s] - 1) & 1, tmo);
                if (nd[s] > 0) drain_wait(&ctl->do_full[s], (nd[s] - 1) & 1, tmo);
            }
        } else if (warp == C::kMmaWarp && issued) {
            tc_commit(&ctl->aux);
            drain_wait(&ctl->aux, 0, tmo);
        }
    }
    if (warp == C::kMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// 64-token query chunks: the quadrant pattern of every CSC entry (column c, query
// box r) is the pattern of the box CSR entry (r, c), found by binary search in
// row r's ascending list. One warp per column.
__global__ void __launch_bounds__(256) csc_pattern_kernel(
    const int32_t* __restrict__ col_ptr, const int32_t* __restrict__ row_idx, int64_t idx_cap,
    const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx, int64_t col_cap,
    const uint8_t* __restrict__ row_pat, int64_t cols, int Nq, int Nc, uint8_t* __restrict__ col_pat,
    uint32_t* status) {
    const int64_t c = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (c >= cols) return;
    const int64_t bh = c / Nc;
    const int kc = static_cast<int>(c % Nc);
    int64_t beg = col_ptr[c], end = col_ptr[c + 1];
    if (!(beg >= 0 && end >= beg && end <= idx_cap)) {
        if (lane == 0) atomicOr(status, kStatusBadIndex);
        return;
    }
    for (int64_t e = beg + lane; e < end; e += 32) {
        const int r = row_idx[e];
        uint8_t pat = 0;
        if (r >= 0 && r < Nq) {
            const int64_t row = bh * Nq + r;
            int64_t lo = row_ptr[row], hi = row_ptr[row + 1];
            if (lo >= 0 && hi >= lo && hi <= col_cap) {
                while (lo < hi) {  // first entry >= kc
                    const int64_t mid = (lo + hi) >> 1;
                    if (col_idx[mid] < kc) lo = mid + 1; else hi = mid;
                }
                if (lo < row_ptr[row + 1] && col_idx[lo] == kc) pat = row_pat[lo];
                else atomicOr(status, kStatusBadIndex);
            } else {
                atomicOr(status, kStatusBadIndex);
            }
        }
        col_pat[e] = pat;
    }
}

template <int D, bool kQuad>
cudaError_t launch_bwd_dq(const CUtensorMap* m, const BwdArgs& dq_args, const BwdArgs& dkv_args,
                          cudaStream_t st) {
    using C = BwdCfg<D>;
    static std::atomic<uint64_t> dq_attr{0}, dkv_attr{0};
    {
        cudaError_t e = raise_smem_limit(bsa_bwd_dq_kernel<D, kQuad>, C::kSmemBytes, dq_attr);
        if (e == cudaSuccess)
            e = raise_smem_limit(bsa_bwd_dkv_kernel<D, kQuad>, C::kSmemBytes, dkv_attr);
        if (e != cudaSuccess) return e;
    }
    // m: q, k, v, dout, dq, dk, dv (whole chunks)
    bsa_bwd_dq_kernel<D, kQuad>
        <<<static_cast<unsigned>(dq_args.units), C::kThreads, C::kSmemBytes, st>>>(
            m[0], m[1], m[2], m[3], m[4], dq_args);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bsa_bwd_dkv_kernel<D, kQuad>
        <<<static_cast<unsigned>(dkv_args.units), C::kThreads, C::kSmemBytes, st>>>(
            m[0], m[1], m[2], m[3], m[5], m[6], dkv_args);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_bwd_d(const CUtensorMap* m, const BwdArgs& dq_args, const BwdArgs& dkv_args,
                         bool quad, cudaStream_t st) {
    return quad ? launch_bwd_dq<D, true>(m, dq_args, dkv_args, st)
                : launch_bwd_dq<D, false>(m, dq_args, dkv_args, st);
}

}  // namespace

BwdLayout bwd_layout(const Dims& g0, const bsa_params& p) {
    auto round_up = [](size_t x) { return (x + 255) / 256 * 256; };
    const bool quad = g0.qw != kChunkW;
    const Dims g = quad ? box_dims(g0) : g0;
    BwdLayout L{};
    L.words = (g.Nq + 31) / 32;
    L.idx_cap = g.rows * static_cast<int64_t>(g.Nc);  // every (row, chunk) pair
    const size_t cols = static_cast<size_t>(g.BH) * g.Nc;
    size_t off = 0;
    L.status = off;
    off += 256;
    L.aux = off;
    off += round_up(static_cast<size_t>(g.rows) * 256 * sizeof(float));
    L.bitmap = off;
    off += round_up(cols * L.words * sizeof(uint32_t));
    L.rawcnt = off;
    off += round_up(cols * sizeof(int32_t));
    L.cnt = off;
    off += round_up(cols * sizeof(int32_t));
    L.col_ptr = off;
    off += round_up((cols + 1) * sizeof(int32_t));
    L.row_idx = off;
    off += round_up(static_cast<size_t>(L.idx_cap) * sizeof(int32_t));
    L.box_counts = L.box_row_ptr = L.box_col_idx = L.box_pat = L.csc_pat = off;
    L.box_cap = 0;
    if (quad) {
        L.box_cap = ws_layout(g0, p).box_cap;  // the forward's bound on a box row's union
        const size_t box_rows = static_cast<size_t>(g0.BH) * g0.NB;
        L.box_counts = off;
        off += round_up(box_rows * sizeof(int32_t));
        L.box_row_ptr = off;
        off += round_up((box_rows + 1) * sizeof(int32_t));
        L.box_col_idx = off;
        off += round_up(static_cast<size_t>(L.box_cap) * sizeof(int32_t));
        L.box_pat = off;
        off += round_up(static_cast<size_t>(L.box_cap));
        L.csc_pat = off;
        off += round_up(static_cast<size_t>(L.idx_cap));
    }
    L.total = off;
    return L;
}

cudaError_t launch_backward(const Dims& g0, const bsa_params& p, const void* q, const void* k,
                            const void* v, const void* out, const float* lse, const void* dout,
                            const int32_t* row_ptr, const int32_t* col_idx, int64_t col_cap,
                            void* workspace, void* dq, void* dk, void* dv, uint64_t timeout_ns,
                            int debug_flags, cudaStream_t st) {
    const BwdLayout L = bwd_layout(g0, p);
    // 64-token query chunks: the attention kernels work on (4,4,8) boxes, over the
    // box CSR with a quadrant pattern per entry (the forward's own construction)
    const bool quad = g0.qw != kChunkW;
    const Dims g = quad ? box_dims(g0) : g0;
    char* ws = static_cast<char*>(workspace);
    uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
    float* aux = reinterpret_cast<float*>(ws + L.aux);
    uint32_t* bitmap = reinterpret_cast<uint32_t*>(ws + L.bitmap);
    int32_t* rawcnt = reinterpret_cast<int32_t*>(ws + L.rawcnt);
    int32_t* cnt = reinterpret_cast<int32_t*>(ws + L.cnt);
    int32_t* col_ptr = reinterpret_cast<int32_t*>(ws + L.col_ptr);
    int32_t* row_idx = reinterpret_cast<int32_t*>(ws + L.row_idx);
    const int64_t cols = g.BH * g.Nc;

    // whole-chunk maps q, k, v, dout, dq, dk, dv
    CUtensorMap m[7];
    const void* bases[7] = {q, k, v, dout, dq, dk, dv};
    for (int i = 0; i < 7; ++i)
        if (!make_chunk_map(&m[i], bases[i], g)) return cudaErrorInvalidValue;

    cudaError_t e = cudaMemsetAsync(ws + L.bitmap, 0, L.cnt - L.bitmap, st);  // bitmap + rawcnt
    if (e != cudaSuccess) return e;
    const int32_t* rp = row_ptr;
    const int32_t* ci = col_idx;
    int64_t cap = col_cap;
    const uint8_t* rpat = nullptr;
    uint8_t* cpat = nullptr;
    if (quad) {
        int32_t* bcnt = reinterpret_cast<int32_t*>(ws + L.box_counts);
        int32_t* brp = reinterpret_cast<int32_t*>(ws + L.box_row_ptr);
        int32_t* bci = reinterpret_cast<int32_t*>(ws + L.box_col_idx);
        uint8_t* bpat = reinterpret_cast<uint8_t*>(ws + L.box_pat);
        if ((e = launch_quad_union(g0, row_ptr, col_idx, col_cap, bcnt, brp, bci, bpat, L.box_cap,
                                   status, st)) != cudaSuccess)
            return e;
        rp = brp;
        ci = bci;
        cap = L.box_cap;
        rpat = bpat;
        cpat = reinterpret_cast<uint8_t*>(ws + L.csc_pat);
    }
    dim3 pgrid(static_cast<unsigned>(g.Nq), static_cast<unsigned>(g.BH));
    const auto* o16 = static_cast<const __nv_bfloat16*>(out);
    const auto* g16 = static_cast<const __nv_bfloat16*>(dout);
    if (g.d == 128)
        bwd_prep_kernel<128><<<pgrid, 256, 0, st>>>(o16, g16, lse, aux, g.q_skip, g.Nq, g.T, g.H,
                                                   g.W, g.NH, g.NW, g.N);
    else
        bwd_prep_kernel<64><<<pgrid, 256, 0, st>>>(o16, g16, lse, aux, g.q_skip, g.Nq, g.T, g.H,
                                                  g.W, g.NH, g.NW, g.N);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    csc_scatter_kernel<<<static_cast<unsigned>((g.rows + 7) / 8), 256, 0, st>>>(
        rp, ci, cap, g.rows, g.Nq, g.Nc, L.words, bitmap, rawcnt, status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    csc_count_kernel<<<static_cast<unsigned>((cols + 255) / 256), 256, 0, st>>>(bitmap, rawcnt,
                                                                               L.words, cols, cnt,
                                                                               status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = launch_scan_counts(cnt, cols, col_ptr, st)) != cudaSuccess) return e;
    csc_emit_kernel<<<static_cast<unsigned>((cols + 7) / 8), 256, 0, st>>>(
        bitmap, L.words, cols, col_ptr, row_idx, L.idx_cap, status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (quad) {
        csc_pattern_kernel<<<static_cast<unsigned>((cols + 7) / 8), 256, 0, st>>>(
            col_ptr, row_idx, L.idx_cap, rp, ci, cap, rpat, cols, g.Nq, g.Nc, cpat, status);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }

    BwdArgs args{};
    args.row_ptr = rp;
    args.col_idx = ci;
    args.col_cap = cap;
    args.col_ptr = col_ptr;
    args.row_idx = row_idx;
    args.idx_cap = L.idx_cap;
    args.aux = aux;
    args.row_pat = rpat;
    args.col_pat = cpat;
    args.dq = static_cast<__nv_bfloat16*>(dq);
    args.dk = static_cast<__nv_bfloat16*>(dk);
    args.dv = static_cast<__nv_bfloat16*>(dv);
    args.status = status;
    args.T = g.T;
    args.H = g.H;
    args.W = g.W;
    args.NH = g.NH;
    args.NW = g.NW;
    args.Nc = g.Nc;
    args.q_skip = g.q_skip;
    args.Nq = g.Nq;
    args.N = g.N;
    args.scale = g.scale;
    args.scale_log2 = g.scale * kLog2e;
    args.timeout_ns = timeout_ns;
    args.debug_flags = debug_flags;
    BwdArgs dq_args = args, dkv_args = args;
    dq_args.units = g.rows;
    dkv_args.units = cols;
    return g.d == 128 ? launch_bwd_d<128>(m, dq_args, dkv_args, quad, st)
                      : launch_bwd_d<64>(m, dq_args, dkv_args, quad, st);
}

}  // namespace bsa
