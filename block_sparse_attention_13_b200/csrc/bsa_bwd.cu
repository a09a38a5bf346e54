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
//   3. dQ:    one CTA per query chunk (CSR row): S = Q K^T and dP = dO V^T per
//             selected key chunk, dS in TMEM, dQ += dS K accumulated in TMEM;
//   4. dK/dV: one CTA per key chunk (CSC column): S^T = K Q^T and
//             dP^T = V dO^T per query chunk that selected it, in two halves of
//             64 queries so the exponentials of one half overlap the tensor
//             core's work on the other; dV += P^T dO and dK += dS^T Q in TMEM.
// Q, K, V, dO and the gradients stay in [T,H,W] token order; the same 5-D TMA
// box as the forward lands one chunk in shared memory in chunk-local order.
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
    // both kernels: six tiles, then 2 KB of per-query-chunk aux, control, list
    static constexpr int kAux = 6 * kTileBytes;
    static constexpr int kCtl = kAux + 2048;
    static constexpr int kList = kCtl + 512;
    static constexpr int kSmemBytes = kList + kMaxList * 2 + 1024;  // + alignment slack
};

struct BwdArgs {
    const int32_t* row_ptr;   // CSR (dQ kernel)
    const int32_t* col_idx;
    int64_t col_cap;
    const int32_t* col_ptr;   // CSC (dK/dV kernel): local query rows per key chunk
    const int32_t* row_idx;
    int64_t idx_cap;
    const float* aux;         // [BH][Nq][half][LSE*log2(e) x64 | D x64]
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

// exp2 of a pair: every 4th pair on the FMA-pipe polynomial, the rest on MUFU.
__device__ __forceinline__ float2 exp2_pair(float2 x, int j) {
    return (j % 4 == 0) ? exp2_poly2(x) : make_float2(ex2_approx(x.x), ex2_approx(x.y));
}

// ------------------------------------------------------------------ dQ kernel
// One CTA per CSR row (query chunk). Shared memory tiles: Q, dO, K[3], V.
// TMEM: S slots at columns 0 and 128, dP at 256, dQ at 384. The 8 dS warps
// split each row: warps w and w+4 share TMEM lanes 32(w%4).. and take key
// columns [0,64) and [64,128); each writes its 32 columns of packed bf16 dS
// over the first half of the S columns it has just read ([0,32) and [64,96)),
// the TMEM A operand of dQ += dS K. MMA issue order per step j, once dS(j) is
// written: dP(j+1), dQ(j), S(j+2); S(j+1) was issued a step earlier. Two
// producer lanes keep the loads independent: lane 0 refills K slots (K(j+3)
// after dQ(j)), lane 1 the V tile (V(j+1) after dP(j)).
struct __align__(8) DqCtl {
    uint64_t qd_full, k_full[3], k_empty[3], v_full, v_empty, s_full[2];
    uint64_t dp_full, ds_full, dq_full, aux;
    int n_valid;
    uint32_t tmem_base;
    int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(320, 1)
    bsa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                      const __grid_constant__ CUtensorMap tm_dq, const BwdArgs a) {
    using C = BwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sQ = smem;
    uint8_t* sdO = smem + C::kTileBytes;
    auto sK = [&](int s) { return smem + (2 + s) * C::kTileBytes; };
    uint8_t* sV = smem + 5 * C::kTileBytes;
    DqCtl* ctl = reinterpret_cast<DqCtl*>(smem + C::kCtl);
    uint16_t* list = reinterpret_cast<uint16_t*>(smem + C::kList);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t row = blockIdx.x;

    if (threadIdx.x == 0) {
        mbar_init(&ctl->qd_full, 1);
        for (int s = 0; s < 3; ++s) {
            mbar_init(&ctl->k_full[s], 1);
            mbar_init(&ctl->k_empty[s], 1);
        }
        mbar_init(&ctl->v_full, 1);
        mbar_init(&ctl->v_empty, 1);
        mbar_init(&ctl->s_full[0], 1);
        mbar_init(&ctl->s_full[1], 1);
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
            if (valid) list[cnt + __popc(vb & ((1u << lane) - 1u))] = static_cast<uint16_t>(c);
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
            int nk[3] = {0, 0, 0};
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
            if (!ok || *abort_flag) {
                drain_wait(&ctl->qd_full, 0, tmo);
                for (int s = 0; s < 3; ++s)
                    if (nk[s] > 0) drain_wait(&ctl->k_full[s], (nk[s] - 1) & 1, tmo);
            }
        } else if (lane == 1 && n > 0) {
            // the V tile: V(j) once dP(j-1) has read V(j-1)
            int nv = 0;
            bool ok = true;
            for (int j = 0; j < n && ok; ++j) {
                if (j >= 1 && !mbar_wait(&ctl->v_empty, (j - 1) & 1, abort_flag, a.status, tmo,
                                         site(1, 2, 0, j))) {
                    ok = false;
                    break;
                }
                int vt, vh, vw;
                chunk_origin(list[j], a.NH, a.NW, vt, vh, vw);
                mbar_arrive_expect_tx(&ctl->v_full, C::kTileBytes);
#pragma unroll
                for (int c = 0; c < C::kHalves; ++c)
                    tma_load_5d(&tm_v, smem_u32(sV) + c * C::kHalfBytes, &ctl->v_full, c * 64, vw, vh,
                                vt, bh);
                ++nv;
            }
            if ((!ok || *abort_flag) && nv > 0) drain_wait(&ctl->v_full, (nv - 1) & 1, tmo);
        }
        __syncwarp();
    } else if (warp == C::kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n > 0) {
            constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, 0, 0);  // both operands K-major
            constexpr uint32_t kIdQ = idesc_bf16_f32(128, D, 0, 1);    // dS from TMEM, K MN-major
            bool issued = false;
            bool ok = mbar_wait(&ctl->qd_full, 0, abort_flag, a.status, tmo, site(2, 0, 0, 0));
            if (ok) tc_fence_after();
            auto issue_ss = [&](uint32_t dcol, uint32_t sa, uint32_t sb) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kHalfBytes + (kk & 3) * 32;
                    mma_ss(tmem + dcol, sdesc_sw128(sa + off, 16, 1024), sdesc_sw128(sb + off, 16, 1024),
                           kIdS, kk > 0 ? 1u : 0u);
                }
            };
            auto issue_s = [&](int j) -> bool {
                const int s = j % 3, t = j & 1;
                if (!mbar_wait(&ctl->k_full[s], (j / 3) & 1, abort_flag, a.status, tmo, site(2, 1, s, j)))
                    return false;
                tc_fence_after();
                issue_ss(128u * t, smem_u32(sQ), smem_u32(sK(s)));
                issued = true;
                tc_commit(&ctl->s_full[t]);
                return true;
            };
            auto issue_dp = [&](int j) -> bool {
                if (!mbar_wait(&ctl->v_full, j & 1, abort_flag, a.status, tmo, site(2, 2, 0, j)))
                    return false;
                tc_fence_after();
                issue_ss(256u, smem_u32(sdO), smem_u32(sV));
                issued = true;
                tc_commit(&ctl->v_empty);
                tc_commit(&ctl->dp_full);
                return true;
            };
            // dQ += dS(j) K(j): keys 16kk.. of dS sit at column 64*(kk/4) + 8*(kk%4) of the S slot
            auto issue_dq = [&](int j) {
                const int s = j % 3, t = j & 1;
                const uint32_t sk = smem_u32(sK(s));
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tmem + 384u, tmem + 128u * t + 64u * (kk >> 2) + 8u * (kk & 3),
                           sdesc_sw128(sk + kk * 2048, C::kHalfBytes, 1024), kIdQ,
                           (j > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&ctl->k_empty[s]);
            };
            ok = ok && issue_s(0) && issue_dp(0) && (n < 2 || issue_s(1));
            for (int j = 0; j < n && ok; ++j) {
                if (!mbar_wait(&ctl->ds_full, j & 1, abort_flag, a.status, tmo, site(2, 3, 0, j))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (j + 1 < n && !issue_dp(j + 1)) { ok = false; break; }
                issue_dq(j);
                if (j + 2 < n && !issue_s(j + 2)) { ok = false; break; }
            }
            if (ok) {
                tc_commit(&ctl->dq_full);
            } else if (issued) {
                tc_commit(&ctl->aux);
                drain_wait(&ctl->aux, 0, tmo);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ dS + epilogue
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
        for (int j = 0; j < n; ++j) {
            const int t = j & 1;
            bool got = mbar_wait(&ctl->s_full[t], (j >> 1) & 1, abort_flag, a.status, tmo, site(3, 4, t, j));
            got = got && mbar_wait(&ctl->dp_full, j & 1, abort_flag, a.status, tmo, site(3, 5, 0, j));
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
            const uint32_t tS = tmem + lane_off + 128u * t + 64u * grp;
            const uint32_t tP = tmem + lane_off + 256u + 64u * grp;
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                uint32_t sv[32], pv[32];
                tmem_ld32(tS + g * 32, sv);
                tmem_ld32(tP + g * 32, pv);
                tmem_wait_ld_tie(sv);
                tmem_wait_ld_tie(pv);
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float2 x = __ffma2_rn(
                        make_float2(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])), cc, nl);
                    const float2 p = exp2_pair(x, e);
                    const float2 dp = __fadd2_rn(
                        make_float2(__uint_as_float(pv[2 * e]), __uint_as_float(pv[2 * e + 1])), nd);
                    const float2 ds = __fmul2_rn(p, dp);
                    pk[e] = pack_bf16x2(ds.x, ds.y);
                }
                // dS over this warp's S columns [16g, 16g+16): already read
                tmem_st16(tS + g * 16, pk);
            }
            tmem_wait_st();
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
            // Q is dead once every MMA has completed; each warp group stages half the columns
            stage_tmem_rows<D>(tmem + lane_off + 384u, sQ, m, a.scale, grp * D / 64, (grp + 1) * D / 64);
            fence_proxy_async_smem();
            named_bar_sync(1, 256);
            if (threadIdx.x == 0) {
#pragma unroll
                for (int c = 0; c < C::kHalves; ++c)
                    tma_store_5d(&tm_dq, smem_u32(sQ) + c * C::kHalfBytes, c * 64, q_w, q_h, q_t, bh);
                tma_store_commit_and_wait_all();
            }
        } else if (all_ok && grp == 0) {
            zero_token<D>(a.dq, bh, a.N, a.T, a.H, a.W, q_t, q_h, q_w, m);  // no selected chunk
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == C::kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ------------------------------------------------------------------ dK/dV kernel
// One CTA per key chunk (CSC column). Shared memory tiles: K, V (this key
// chunk) and Q[2], dO[2] (query chunks of the column, double-buffered), each
// query chunk loaded in two halves of 64 queries (its frames 0-1 and 2-3)
// together with the matching half of its aux record; a half is released as
// soon as its last MMA has run. TMEM: S^T = K Q^T and dP^T = V dO^T per half
// (S^T half h at column 64h, dP^T half h at 128 + 64h), dV accumulates at 256,
// dK at 384. The 8 softmax warps split each half: warps w and w+4 share TMEM
// lanes 32(w%4).. (key rows) and take its query columns [0,32) and [32,64),
// writing packed bf16 P^T / dS^T over the first 16 of the columns they read
// (the TMEM A operands of dV += P^T dO and dK += dS^T Q).
// MMA issue order per step i:
//   dV,dK(i,h0)  S^T,dP^T(i+1,h0)  dV,dK(i,h1)  S^T,dP^T(i+1,h1)
// so the exponentials of one half run while the tensor core works on the other.
struct __align__(8) DkvCtl {
    uint64_t kv_full, qd_full[2][2], qd_empty[2][2], sd_full[2], p_full[2], dkv_full, aux;
    int n_valid;
    uint32_t tmem_base;
    int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(320, 1)
    bsa_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tm_qh, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_doh,
                       const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                       const BwdArgs a) {
    using C = BwdCfg<D>;
    constexpr int kHalfTile = C::kTileBytes / 2;  // 64 tokens x D
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
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t col = blockIdx.x;
    const int bh = static_cast<int>(col / a.Nc);
    const int kc = static_cast<int>(col % a.Nc);

    if (threadIdx.x == 0) {
        mbar_init(&ctl->kv_full, 1);
        for (int s = 0; s < 2; ++s) {
            for (int h = 0; h < 2; ++h) {
                mbar_init(&ctl->qd_full[s][h], 1);
                mbar_init(&ctl->qd_empty[s][h], 1);
            }
            mbar_init(&ctl->sd_full[s], 1);
            mbar_init(&ctl->p_full[s], 256);
        }
        mbar_init(&ctl->dkv_full, 1);
        mbar_init(&ctl->aux, 1);
        ctl->abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == C::kTmaWarp) {
        // stage the column's query rows (out-of-range entries dropped and reported)
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
            if (valid) list[cnt + __popc(vb & ((1u << lane) - 1u))] = static_cast<uint16_t>(r);
            cnt += __popc(vb);
        }
        if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(a.status, kStatusBadIndex);
        if (lane == 0) {
            ctl->n_valid = cnt;
            prefetch_tensormap(&tm_qh);
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
            prefetch_tensormap(&tm_doh);
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

    if (warp == C::kTmaWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && n > 0) {
            mbar_arrive_expect_tx(&ctl->kv_full, 2 * C::kTileBytes);
#pragma unroll
            for (int c = 0; c < C::kHalves; ++c) {
                tma_load_5d(&tm_k, smem_u32(sK) + c * C::kHalfBytes, &ctl->kv_full, c * 64, k_w, k_h,
                            k_t, bh);
                tma_load_5d(&tm_v, smem_u32(sV) + c * C::kHalfBytes, &ctl->kv_full, c * 64, k_w, k_h,
                            k_t, bh);
            }
            int nq[2][2] = {{0, 0}, {0, 0}};
            bool ok = true;
            for (int i = 0; i < n && ok; ++i) {
                const int s = i & 1;
                const int r = list[i];
                int qt, qh, qw;
                chunk_origin(a.q_skip + r, a.NH, a.NW, qt, qh, qw);
                for (int h = 0; h < 2; ++h) {
                    if (i >= 2 && !mbar_wait(&ctl->qd_empty[s][h], ((i - 2) >> 1) & 1, abort_flag,
                                             a.status, tmo, site(1, 1 + h, s, i))) {
                        ok = false;
                        break;
                    }
                    uint64_t* bar = &ctl->qd_full[s][h];
                    mbar_arrive_expect_tx(bar, 2 * kHalfTile + 512);
#pragma unroll
                    for (int c = 0; c < C::kHalves; ++c) {
                        tma_load_5d(&tm_qh, smem_u32(sQ(s)) + c * C::kHalfBytes + h * 8192, bar, c * 64,
                                    qw, qh, qt + 2 * h, bh);
                        tma_load_5d(&tm_doh, smem_u32(sdO(s)) + c * C::kHalfBytes + h * 8192, bar,
                                    c * 64, qw, qh, qt + 2 * h, bh);
                    }
                    bulk_load(smem_u32(sAux + s * 256 + h * 128),
                              a.aux + (static_cast<int64_t>(bh) * a.Nq + r) * 256 + h * 128, 512, bar);
                    ++nq[s][h];
                }
            }
            if (!ok || *abort_flag) {
                drain_wait(&ctl->kv_full, 0, tmo);
                for (int s = 0; s < 2; ++s)
                    for (int h = 0; h < 2; ++h)
                        if (nq[s][h] > 0) drain_wait(&ctl->qd_full[s][h], (nq[s][h] - 1) & 1, tmo);
            }
        }
        __syncwarp();
    } else if (warp == C::kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n > 0) {
            constexpr uint32_t kIdS = idesc_bf16_f32(128, 64, 0, 0);  // keys x 64 queries, K-major
            constexpr uint32_t kIdG = idesc_bf16_f32(128, D, 0, 1);   // P^T/dS^T from TMEM, MN-major
            bool issued = false;
            bool ok = mbar_wait(&ctl->kv_full, 0, abort_flag, a.status, tmo, site(2, 0, 0, 0));
            if (ok) tc_fence_after();
            // S^T and dP^T for queries [64h, 64h+64) of step i
            auto issue_sd = [&](int i, int h) -> bool {
                const int s = i & 1;
                if (!mbar_wait(&ctl->qd_full[s][h], (i >> 1) & 1, abort_flag, a.status, tmo,
                               site(2, 1, s * 2 + h, i)))
                    return false;
                tc_fence_after();
                const uint32_t sk = smem_u32(sK), sv = smem_u32(sV);
                const uint32_t sq = smem_u32(sQ(s)) + h * 8192, sd = smem_u32(sdO(s)) + h * 8192;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kHalfBytes + (kk & 3) * 32;
                    mma_ss(tmem + 64u * h, sdesc_sw128(sk + off, 16, 1024),
                           sdesc_sw128(sq + off, 16, 1024), kIdS, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kHalfBytes + (kk & 3) * 32;
                    mma_ss(tmem + 128u + 64u * h, sdesc_sw128(sv + off, 16, 1024),
                           sdesc_sw128(sd + off, 16, 1024), kIdS, kk > 0 ? 1u : 0u);
                }
                issued = true;
                tc_commit(&ctl->sd_full[h]);
                return true;
            };
            // dV += P^T dO and dK += dS^T Q over queries [64h, 64h+64) of step i
            auto issue_pg = [&](int i, int h) -> bool {
                const int s = i & 1;
                if (!mbar_wait(&ctl->p_full[h], i & 1, abort_flag, a.status, tmo, site(2, 2, h, i)))
                    return false;
                tc_fence_after();
                const uint32_t sq = smem_u32(sQ(s)), sd = smem_u32(sdO(s));
                // queries 16kk.. of half h: column 64h + 32*(kk/2) + 8*(kk%2) of S^T / dP^T
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts(tmem + 256u, tmem + 64u * h + 32u * (kk >> 1) + 8u * (kk & 1),
                           sdesc_sw128(sd + (4 * h + kk) * 2048, C::kHalfBytes, 1024), kIdG,
                           (i > 0 || h > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts(tmem + 384u, tmem + 128u + 64u * h + 32u * (kk >> 1) + 8u * (kk & 1),
                           sdesc_sw128(sq + (4 * h + kk) * 2048, C::kHalfBytes, 1024), kIdG,
                           (i > 0 || h > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&ctl->qd_empty[s][h]);
                return true;
            };
            ok = ok && issue_sd(0, 0) && issue_sd(0, 1);
            for (int i = 0; i < n && ok; ++i) {
                ok = issue_pg(i, 0) && (i + 1 >= n || issue_sd(i + 1, 0)) && issue_pg(i, 1) &&
                     (i + 1 >= n || issue_sd(i + 1, 1));
            }
            if (ok) {
                tc_commit(&ctl->dkv_full);
            } else if (issued) {
                tc_commit(&ctl->aux);
                drain_wait(&ctl->aux, 0, tmo);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ P^T, dS^T + epilogue
        const int grp = warp >> 2;                    // query columns [32*grp, 32*grp + 32) of a half
        const int m = (warp & 3) * 32 + lane;         // key row = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const float2 cc = make_float2(a.scale_log2, a.scale_log2);
        bool ok = true;
        for (int i = 0; i < n && ok; ++i) {
            const int s = i & 1;
            for (int h = 0; h < 2; ++h) {
                // this half's aux record arrived with its Q/dO copies
                bool got = mbar_wait(&ctl->qd_full[s][h], (i >> 1) & 1, abort_flag, a.status, tmo,
                                     site(3, 3, s * 2 + h, i));
                got = got && mbar_wait(&ctl->sd_full[h], i & 1, abort_flag, a.status, tmo, site(3, 4, h, i));
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                tc_fence_after();
                const float* lse2 = sAux + s * 256 + h * 128;
                const float* Dq = lse2 + 64;
                const uint32_t tS = tmem + lane_off + 64u * h + 32u * grp;
                const uint32_t tP = tmem + lane_off + 128u + 64u * h + 32u * grp;
                {
                    uint32_t sv[32], pv[32];
                    tmem_ld32(tS, sv);
                    tmem_ld32(tP, pv);
                    tmem_wait_ld_tie(sv);
                    tmem_wait_ld_tie(pv);
                    uint32_t pk[16], dk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int qi = 32 * grp + 2 * e;  // query of this pair within the half
                        const float2 l2 = *reinterpret_cast<const float2*>(lse2 + qi);
                        const float2 dd = *reinterpret_cast<const float2*>(Dq + qi);
                        const float2 x = __ffma2_rn(
                            make_float2(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])), cc,
                            make_float2(-l2.x, -l2.y));
                        const float2 p = exp2_pair(x, e);
                        const float2 dp = make_float2(__uint_as_float(pv[2 * e]) - dd.x,
                                                      __uint_as_float(pv[2 * e + 1]) - dd.y);
                        const float2 ds = __fmul2_rn(p, dp);
                        pk[e] = pack_bf16x2(p.x, p.y);
                        dk[e] = pack_bf16x2(ds.x, ds.y);
                    }
                    tmem_st16(tS, pk);
                    tmem_st16(tP, dk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&ctl->p_full[h]);
            }
        }
        if (ok && n > 0) {
            const bool got = mbar_wait(&ctl->dkv_full, 0, abort_flag, a.status, tmo, site(3, 6, 0, 0));
            ok = __all_sync(0xffffffffu, got);
        }
        const bool all_ok = bar_red_and(1, 256, ok);
        if (all_ok && n > 0) {
            tc_fence_after();
            // K and V tiles are dead once every MMA has completed: group 0 stages
            // dV, group 1 dK (scaled)
            if (grp == 0)
                stage_tmem_rows<D>(tmem + lane_off + 256u, sV, m, 1.0f);
            else
                stage_tmem_rows<D>(tmem + lane_off + 384u, sK, m, a.scale);
            fence_proxy_async_smem();
            named_bar_sync(1, 256);
            if (threadIdx.x == 0) {
#pragma unroll
                for (int c = 0; c < C::kHalves; ++c) {
                    tma_store_5d(&tm_dv, smem_u32(sV) + c * C::kHalfBytes, c * 64, k_w, k_h, k_t, bh);
                    tma_store_5d(&tm_dk, smem_u32(sK) + c * C::kHalfBytes, c * 64, k_w, k_h, k_t, bh);
                }
                tma_store_commit_and_wait_all();
            }
        } else if (all_ok) {
            // no query chunk selected this key chunk: zero gradients
            zero_token<D>(grp ? a.dk : a.dv, bh, a.N, a.T, a.H, a.W, k_t, k_h, k_w, m);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == C::kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int D>
cudaError_t launch_bwd_d(const Dims& g, const CUtensorMap* m, const BwdArgs& dq_args,
                         const BwdArgs& dkv_args, cudaStream_t st) {
    using C = BwdCfg<D>;
    static std::atomic<uint64_t> dq_attr{0}, dkv_attr{0};
    {
        cudaError_t e = raise_smem_limit(bsa_bwd_dq_kernel<D>, C::kSmemBytes, dq_attr);
        if (e == cudaSuccess) e = raise_smem_limit(bsa_bwd_dkv_kernel<D>, C::kSmemBytes, dkv_attr);
        if (e != cudaSuccess) return e;
    }
    // m: q, k, v, dout, dq, dk, dv (whole chunks), then q and dout (half chunks)
    bsa_bwd_dq_kernel<D><<<static_cast<unsigned>(dq_args.units), C::kThreads, C::kSmemBytes, st>>>(
        m[0], m[1], m[2], m[3], m[4], dq_args);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bsa_bwd_dkv_kernel<D><<<static_cast<unsigned>(dkv_args.units), C::kThreads, C::kSmemBytes, st>>>(
        m[7], m[1], m[2], m[8], m[5], m[6], dkv_args);
    return cudaGetLastError();
}

}  // namespace

BwdLayout bwd_layout(const Dims& g) {
    auto round_up = [](size_t x) { return (x + 255) / 256 * 256; };
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
    L.total = off;
    return L;
}

cudaError_t launch_backward(const Dims& g, const void* q, const void* k, const void* v,
                            const void* out, const float* lse, const void* dout,
                            const int32_t* row_ptr, const int32_t* col_idx, int64_t col_cap,
                            void* workspace, void* dq, void* dk, void* dv, uint64_t timeout_ns,
                            cudaStream_t st) {
    const BwdLayout L = bwd_layout(g);
    char* ws = static_cast<char*>(workspace);
    uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
    float* aux = reinterpret_cast<float*>(ws + L.aux);
    uint32_t* bitmap = reinterpret_cast<uint32_t*>(ws + L.bitmap);
    int32_t* rawcnt = reinterpret_cast<int32_t*>(ws + L.rawcnt);
    int32_t* cnt = reinterpret_cast<int32_t*>(ws + L.cnt);
    int32_t* col_ptr = reinterpret_cast<int32_t*>(ws + L.col_ptr);
    int32_t* row_idx = reinterpret_cast<int32_t*>(ws + L.row_idx);
    const int64_t cols = g.BH * g.Nc;

    // whole-chunk maps q, k, v, dout, dq, dk, dv, then half-chunk maps of q and dout
    CUtensorMap m[9];
    const void* bases[9] = {q, k, v, dout, dq, dk, dv, q, dout};
    for (int i = 0; i < 9; ++i)
        if (!make_chunk_map(&m[i], bases[i], g, i < 7 ? kChunkT : kChunkT / 2))
            return cudaErrorInvalidValue;

    cudaError_t e = cudaMemsetAsync(ws + L.bitmap, 0, L.cnt - L.bitmap, st);  // bitmap + rawcnt
    if (e != cudaSuccess) return e;
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
        row_ptr, col_idx, col_cap, g.rows, g.Nq, g.Nc, L.words, bitmap, rawcnt, status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    csc_count_kernel<<<static_cast<unsigned>((cols + 255) / 256), 256, 0, st>>>(bitmap, rawcnt,
                                                                               L.words, cols, cnt,
                                                                               status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = launch_scan_counts(cnt, cols, col_ptr, st)) != cudaSuccess) return e;
    csc_emit_kernel<<<static_cast<unsigned>((cols + 7) / 8), 256, 0, st>>>(
        bitmap, L.words, cols, col_ptr, row_idx, L.idx_cap, status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    BwdArgs args{};
    args.row_ptr = row_ptr;
    args.col_idx = col_idx;
    args.col_cap = col_cap;
    args.col_ptr = col_ptr;
    args.row_idx = row_idx;
    args.idx_cap = L.idx_cap;
    args.aux = aux;
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
    BwdArgs dq_args = args, dkv_args = args;
    dq_args.units = g.rows;
    dkv_args.units = cols;
    return g.d == 128 ? launch_bwd_d<128>(g, m, dq_args, dkv_args, st)
                      : launch_bwd_d<64>(g, m, dq_args, dkv_args, st);
}

}  // namespace bsa
