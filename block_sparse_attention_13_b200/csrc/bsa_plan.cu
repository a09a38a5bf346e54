// Block selection kernels: 3D gather + chunk mean-pool, pooled scores,
// warp-level top-k / CDF selection into CSR, and the 3D rearrangement.
//
// Method ("LongCat-Video Technical Report", section "Block Sparse Attention
// (BSA)"): Q_pool / K_pool are block means over the n tokens of each 3D block,
// S_pool = Q_pool K_pool^T / sqrt(d), and each query block keeps the r key
// blocks with the highest scores. "LongCat-Video Technical Report #", section
// "3D Block Sparse Attention": chunk shape [4,4,8]; Top-K and CDF-threshold
// selection. Block-causal candidates: "LongCat-Video Technical Report",
// section "Block Attention with KV-Cache for Efficient Multi-Task Inference".
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bsa_internal.cuh"
#include "bsa_ptx.cuh"

namespace bsa {

namespace {

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void add_bf16x2(float& a, float& b, uint32_t u) {
    a += __uint_as_float(u << 16);
    b += __uint_as_float(u & 0xFFFF0000u);
}

// ------------------------------------------------------------------------
// Gather + mean-pool. One CTA per (chunk, batch*head, tensor). A chunk is 16
// contiguous segments (lt, lh) of 8 tokens (lw = 0..7); consecutive threads
// read consecutive 16-byte vectors, so every warp load is one contiguous
// 512-byte run. Each thread always covers the same 8 channels and sums them
// over its tokens in fp32; a shared-memory pass finishes the 128-token sum.
// Tensor z (blockIdx.z) pools chunks [c_begin, c_begin + n_out) of its own
// chunk grid into rows 0 .. n_out-1 of its output. A chunk is mt x mh x mw
// boxes of (4,4,bw) tokens, bw = 8 or 4 (a key chunk can be larger than the
// query chunk; 64-token chunks are single (4,4,4) boxes); a partial edge chunk
// averages the tokens it has.
struct PoolSide {
    int c_begin, n_out;
    int mt, mh, mw;  // boxes per chunk along t, h, w
    int NHc, NWc;    // chunks of this grid along h, w
    int bw;          // box width along w: 8, or 4 for 64-token chunks
};

template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ x0,
                                                   const __nv_bfloat16* __restrict__ x1,
                                                   float* __restrict__ p0, float* __restrict__ p1,
                                                   PoolSide s0, PoolSide s1, int T, int H, int W,
                                                   int64_t N) {
    constexpr int VPT = D / 8;               // 16-byte vectors per token row
    constexpr int ITERS = 128 * VPT / 256;   // vectors per thread
    constexpr int GROUPS = 256 / VPT;        // threads that share one channel group
    __shared__ float red[GROUPS][D + 1];

    const __nv_bfloat16* x = blockIdx.z ? x1 : x0;
    float* pooled = blockIdx.z ? p1 : p0;
    const PoolSide sd = blockIdx.z ? s1 : s0;
    if (static_cast<int>(blockIdx.x) >= sd.n_out) return;
    const int c = sd.c_begin + blockIdx.x;
    const int64_t bh = blockIdx.y;
    const int ct = c / (sd.NHc * sd.NWc), ch = (c / sd.NWc) % sd.NHc, cw = c % sd.NWc;
    const int tid = threadIdx.x;
    const int dvec = tid % VPT;

    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    const __nv_bfloat16* base = x + bh * N * D;
    // sums the existing tokens of the box at (t0, h0, w0); returns their count
    auto add_box = [&](int t0, int h0, int w0) -> int {
        const int nt = min(kChunkT, T - t0), nh = min(kChunkH, H - h0), nw = min(sd.bw, W - w0);
        if (nt <= 0 || nh <= 0 || nw <= 0) return 0;  // box past the grid
        if (nt == kChunkT && nh == kChunkH && nw == kChunkW) {
            // a whole box: every load unconditional, all in flight together
            uint4 u[ITERS];
#pragma unroll
            for (int it = 0; it < ITERS; ++it) {
                const int l = (it * 256 + tid) / VPT;  // local token (lt*4 + lh)*8 + lw
                const int lt = l >> 5, lh = (l >> 3) & 3, lw = l & 7;
                const int64_t tok = ((int64_t)(t0 + lt) * H + (h0 + lh)) * W + w0 + lw;
                u[it] = ld_nc_v4(base + tok * D + dvec * 8);
            }
#pragma unroll
            for (int it = 0; it < ITERS; ++it) {
                add_bf16x2(acc[0], acc[1], u[it].x);
                add_bf16x2(acc[2], acc[3], u[it].y);
                add_bf16x2(acc[4], acc[5], u[it].z);
                add_bf16x2(acc[6], acc[7], u[it].w);
            }
        } else {
            // a partial box, or a (4,4,4) box of 64 tokens: local token l is
            // (lt*4 + lh)*bw + lw
            const int lb = sd.bw == kChunkW ? 3 : 2;  // log2(bw)
#pragma unroll
            for (int it = 0; it < ITERS; ++it) {
                const int l = (it * 256 + tid) / VPT;
                if (l >= (16 << lb)) continue;
                const int lt = l >> (lb + 2), lh = (l >> lb) & 3, lw = l & ((1 << lb) - 1);
                if (lt >= nt || lh >= nh || lw >= nw) continue;
                const int64_t tok = ((int64_t)(t0 + lt) * H + (h0 + lh)) * W + w0 + lw;
                const uint4 u = ld_nc_v4(base + tok * D + dvec * 8);
                add_bf16x2(acc[0], acc[1], u.x);
                add_bf16x2(acc[2], acc[3], u.y);
                add_bf16x2(acc[4], acc[5], u.z);
                add_bf16x2(acc[6], acc[7], u.w);
            }
        }
        return nt * nh * nw;
    };
    int n_tok = 0;
    if (sd.mt * sd.mh * sd.mw == 1) {
        n_tok = add_box(ct * kChunkT, ch * kChunkH, cw * sd.bw);
    } else {
        for (int bt = 0; bt < sd.mt; ++bt)
            for (int bhh = 0; bhh < sd.mh; ++bhh)
                for (int bw = 0; bw < sd.mw; ++bw)
                    n_tok += add_box((ct * sd.mt + bt) * kChunkT, (ch * sd.mh + bhh) * kChunkH,
                                     (cw * sd.mw + bw) * sd.bw);
    }
    const int grp = tid / VPT;
#pragma unroll
    for (int e = 0; e < 8; ++e) red[grp][dvec * 8 + e] = acc[e];
    __syncthreads();
    if (tid < D) {
        float s = 0.f;
#pragma unroll
        for (int g2 = 0; g2 < GROUPS; ++g2) s += red[g2][tid];
        pooled[(bh * sd.n_out + blockIdx.x) * D + tid] = s * (1.0f / static_cast<float>(n_tok));
    }
}

// ------------------------------------------------------------------------
// 3D rearrangement: a (lt, lh) segment of 8 tokens is contiguous both in the
// [T,H,W] layout and in the chunk-major layout, so the copy is two streams of
// contiguous 16-byte vectors. Slots of a partial edge chunk past the grid are
// zero in the chunk-major layout and are not written back by the inverse.
template <int D>
__global__ void __launch_bounds__(256) rearrange_kernel(const __nv_bfloat16* __restrict__ src,
                                                        __nv_bfloat16* __restrict__ dst, int T,
                                                        int H, int W, int NH, int NW, int Nc,
                                                        int64_t N, int inverse) {
    constexpr int VPT = D / 8;
    constexpr int ITERS = 128 * VPT / 256;
    const int c = blockIdx.x;
    const int64_t bh = blockIdx.y;
    const int ct = c / (NH * NW), ch = (c / NW) % NH, cw = c % NW;
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
        const int v = it * 256 + threadIdx.x;
        const int l = v / VPT, dv = v % VPT;
        const int lt = l >> 5, lh = (l >> 3) & 3, lw = l & 7;
        const int t = ct * kChunkT + lt, h = ch * kChunkH + lh, w = cw * kChunkW + lw;
        const int64_t blk = ((bh * Nc + c) * kChunkTokens + l) * D + dv * 8;
        if (t >= T || h >= H || w >= W) {
            if (!inverse) *reinterpret_cast<uint4*>(dst + blk) = make_uint4(0u, 0u, 0u, 0u);
            continue;
        }
        const int64_t tok = ((int64_t)t * H + h) * W + w;
        const int64_t thw = (bh * N + tok) * D + dv * 8;
        const int64_t s_off = inverse ? blk : thw;
        const int64_t d_off = inverse ? thw : blk;
        *reinterpret_cast<uint4*>(dst + d_off) = ld_nc_v4(src + s_off);
    }
}

// ------------------------------------------------------------------------
// Pooled scores S[bh][i][m] = <qp[i], kp[m]> * scale in fp32 FMA. 128x128
// output tile per CTA, 8x8 register micro-tile per thread (64 FMAs per 16
// values read from shared memory), operands staged transposed in shared
// memory 16 channels at a time, two stages deep.
// kp holds the key chunks in shards of `kshard` chunks, [shard][BH][kshard][D]
// (kshard = Nk: one shard, the plain [BH][Nk][D] layout); the gathered pooled
// keys of a context-parallel group arrive that way.
__global__ void __launch_bounds__(256, 2) scores_kernel(const float* __restrict__ qp,
                                                     const float* __restrict__ kp,
                                                     float* __restrict__ S, int Nq, int Nk,
                                                     int kshard, int D, float scale) {
    constexpr int BT = 128, BK = 16, LD = BT + 4;
    // two stages: the next 16 channels are fetched into registers while the
    // current ones are multiplied, then stored into the other stage
    __shared__ __align__(16) float As[2][BK][LD];
    __shared__ __align__(16) float Bs[2][BK][LD];
    const int64_t bh = blockIdx.z;
    const int i0 = blockIdx.y * BT, m0 = blockIdx.x * BT;
    const float* A = qp + bh * (int64_t)Nq * D;
    const int64_t BH = gridDim.z;
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    // the two rows (of A and of B) this thread stages, and their channel quad
    const float* arow[2];
    const float* brow[2];
    int rr[2], kq[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int idx = tid + 256 * j;  // 512 float4 per 128x16 tile
        rr[j] = idx / (BK / 4);
        kq[j] = idx % (BK / 4);
        arow[j] = i0 + rr[j] < Nq ? A + (int64_t)(i0 + rr[j]) * D : nullptr;
        const int m = m0 + rr[j];
        if (m < Nk) {
            const int sh = m / kshard, ml = m - sh * kshard;
            brow[j] = kp + ((sh * BH + bh) * kshard + ml) * D;
        } else {
            brow[j] = nullptr;
        }
    }
    float4 ra[2], rb[2];
    auto fetch = [&](int k0) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            ra[j] = arow[j] ? *reinterpret_cast<const float4*>(arow[j] + k0 + kq[j] * 4)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
            rb[j] = brow[j] ? *reinterpret_cast<const float4*>(brow[j] + k0 + kq[j] * 4)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    auto stage = [&](int st) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int r = rr[j], c = kq[j] * 4;
            As[st][c + 0][r] = ra[j].x; As[st][c + 1][r] = ra[j].y;
            As[st][c + 2][r] = ra[j].z; As[st][c + 3][r] = ra[j].w;
            Bs[st][c + 0][r] = rb[j].x; Bs[st][c + 1][r] = rb[j].y;
            Bs[st][c + 2][r] = rb[j].z; Bs[st][c + 3][r] = rb[j].w;
        }
    };
    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;

    fetch(0);
    stage(0);
    __syncthreads();
    const int nk = D / BK;
    for (int c = 0; c < nk; ++c) {
        const int st = c & 1;
        if (c + 1 < nk) fetch((c + 1) * BK);
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4*>(&As[st][kk][ty * 8]);
            const float4 a1 = *reinterpret_cast<const float4*>(&As[st][kk][ty * 8 + 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&Bs[st][kk][tx * 8]);
            const float4 b1 = *reinterpret_cast<const float4*>(&Bs[st][kk][tx * 8 + 4]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int p = 0; p < 8; ++p)
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[p][q] = fmaf(av[p], bv[q], acc[p][q]);
        }
        if (c + 1 < nk) stage(st ^ 1);  // the other stage was last read before the previous sync
        __syncthreads();
    }
    float* out = S + bh * (int64_t)Nq * Nk;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        const int i = i0 + ty * 8 + p;
        if (i >= Nq) continue;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int m = m0 + tx * 8 + h * 4;
            float* o = out + (int64_t)i * Nk + m;
            if ((Nk & 3) == 0 && m + 3 < Nk) {
                *reinterpret_cast<float4*>(o) =
                    make_float4(acc[p][h * 4 + 0] * scale, acc[p][h * 4 + 1] * scale,
                                acc[p][h * 4 + 2] * scale, acc[p][h * 4 + 3] * scale);
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (m + q < Nk) o[q] = acc[p][h * 4 + q] * scale;
            }
        }
    }
}

// ------------------------------------------------------------------------
// Selection: one warp per CSR row. Scores become order-preserving 32-bit keys
// (larger score -> larger key; invalid slots are 0, below every real key).
// The k-th largest key is found by a 32-step bitwise search with warp
// reductions; rows are then emitted in ascending chunk order with ballots,
// keeping the lowest indices among keys equal to the threshold.

__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

template <int MAXJ>
__device__ __forceinline__ uint32_t kth_largest_key(const uint32_t (&key)[MAXJ], int k) {
    uint32_t v = 0;
    for (int bit = 31; bit >= 0; --bit) {
        const uint32_t t = v | (1u << bit);
        int c = 0;
#pragma unroll
        for (int j = 0; j < MAXJ; ++j) c += key[j] >= t;
        c = __reduce_add_sync(0xffffffffu, c);
        if (c >= k) v = t;
    }
    return v;
}

// One warp per CSR row. Query chunks are numbered on the (4,4,8) grid (Ncq per
// (batch, head), the first n_cond_q of them condition chunks); candidates are
// the Nk key chunks (the first n_cond_k of them condition chunks), which are
// the query chunks themselves unless the key chunk shape is larger.
template <int MAXJ>
__global__ void __launch_bounds__(256) select_kernel(
    const float* __restrict__ S, int Ncq, int Nk, int n_cond_q, int n_cond_k, int q_skip,
    int Nq, int64_t rows, int mode, int topk, float cdf_p, float cap_frac,
    int32_t* __restrict__ row_ptr, int32_t* __restrict__ col_idx, int64_t col_cap,
    int32_t* __restrict__ counts, int32_t* __restrict__ padded, int pad_stride, uint32_t* status) {
    const int lane = threadIdx.x & 31;
    const int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (w >= rows) return;
    (void)Ncq;
    // computed query chunks per (batch, head): q_skip .. q_skip + Nq - 1
    const int64_t bh = w / Nq;
    const int i = q_skip + (int)(w % Nq);       // query chunk of this row
    const int na = (n_cond_q > 0 && i < n_cond_q) ? n_cond_k : Nk;  // candidates are [0, na)
    const float* srow = S + w * (int64_t)Nk;

    uint32_t key[MAXJ];
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int m = j * 32 + lane;
        key[j] = (m < na) ? order_key(srow[m]) : 0u;
    }

    int count;
    if (mode == BSA_SEL_TOPK) {
        count = topk < na ? topk : na;
    } else {
        // softmax over A(i) in fp32; shortest descending prefix with mass >= p
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < MAXJ; ++j)
            if (key[j]) mx = fmaxf(mx, key_value(key[j]));
        mx = warp_max(mx);
        float e[MAXJ];
        float z = 0.f;
#pragma unroll
        for (int j = 0; j < MAXJ; ++j) {
            e[j] = key[j] ? expf(key_value(key[j]) - mx) : 0.f;
            z += e[j];
        }
        z = warp_sum(z);
        const float target = cdf_p * z;
        uint32_t v = 0;
        for (int bit = 31; bit >= 0; --bit) {
            const uint32_t t = v | (1u << bit);
            float msum = 0.f;
#pragma unroll
            for (int j = 0; j < MAXJ; ++j) msum += (key[j] >= t) ? e[j] : 0.f;
            msum = warp_sum(msum);
            if (msum >= target) v = t;
        }
        int mstar = na;
        if (v != 0) {
            int cgt = 0, ceq = 0;
            float mgt = 0.f;
#pragma unroll
            for (int j = 0; j < MAXJ; ++j) {
                cgt += key[j] > v;
                ceq += key[j] == v;
                mgt += (key[j] > v) ? e[j] : 0.f;
            }
            cgt = __reduce_add_sync(0xffffffffu, cgt);
            ceq = __reduce_add_sync(0xffffffffu, ceq);
            mgt = warp_sum(mgt);
            const float ev = expf(key_value(v) - mx);
            int needed = 0;
            float cum = mgt;
            while (needed < ceq) {  // equal scores, taken in index order
                cum += ev;
                ++needed;
                if (cum >= target) break;
            }
            mstar = cgt + needed;
        }
        // same double-precision formula as the host's workspace sizing
        int cap = (int)floor((double)cap_frac * (double)na);
        if (cap < 1) cap = 1;
        if (cap > pad_stride) cap = pad_stride;
        count = mstar < cap ? mstar : cap;
        // combination: kept by both rules, i.e. the first min(k, CDF count) chunks
        if (mode == BSA_SEL_TOPK_CDF && topk < count) count = topk;
    }

    // emit the top-`count` chunks by (score desc, index asc), ascending
    const uint32_t v = kth_largest_key(key, count);
    int cgt = 0;
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) cgt += key[j] > v;
    cgt = __reduce_add_sync(0xffffffffu, cgt);
    const int need_eq = count - cgt;

    int32_t* dst;
    int64_t off;
    if (mode == BSA_SEL_TOPK) {
        const int kc = topk < n_cond_k ? topk : n_cond_k;
        const int kn = topk < Nk ? topk : Nk;
        // rows of a (batch, head): condition rows q_skip .. min(n_cond_q, q_skip+Nq)-1,
        // then noisy rows
        const int q_stop = q_skip + Nq;
        const int c_end = n_cond_q < q_stop ? n_cond_q : q_stop;
        const int c_rows = c_end > q_skip ? c_end - q_skip : 0;
        const int first_noisy = n_cond_q > q_skip ? n_cond_q : q_skip;
        const int64_t per_bh = (int64_t)c_rows * kc + (int64_t)(Nq - c_rows) * kn;
        off = bh * per_bh + (i < n_cond_q ? (int64_t)(i - q_skip) * kc
                                          : (int64_t)c_rows * kc + (int64_t)(i - first_noisy) * kn);
        if (off + count > col_cap) {
            if (lane == 0) atomicOr(status, kStatusCapacity);
            return;
        }
        dst = col_idx + off;
        if (lane == 0) {
            row_ptr[w + 1] = (int32_t)(off + count);
            if (w == 0) row_ptr[0] = 0;
        }
    } else {
        dst = padded + w * (int64_t)pad_stride;
        if (lane == 0) counts[w] = count;
    }
    const uint32_t lt_mask = (1u << lane) - 1u;
    int run_sel = 0, run_eq = 0;
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        if (j * 32 >= na) break;
        const bool gt = key[j] > v;
        const bool eq = key[j] == v;
        const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
        const int eq_before = run_eq + __popc(eqb & lt_mask);
        const bool sel = gt || (eq && eq_before < need_eq);
        const uint32_t sb = __ballot_sync(0xffffffffu, sel);
        if (sel) dst[run_sel + __popc(sb & lt_mask)] = j * 32 + lane;
        run_sel += __popc(sb);
        run_eq += __popc(eqb);
    }
}

// Exclusive scan of CDF row counts into row_ptr (one CTA).
__global__ void __launch_bounds__(1024) scan_counts_kernel(const int32_t* __restrict__ counts,
                                                          int64_t rows, int32_t* __restrict__ row_ptr) {
    __shared__ int64_t warp_tot[32];
    const int tid = threadIdx.x;
    const int64_t per = (rows + 1023) / 1024;
    const int64_t beg = tid * per;
    const int64_t end = beg + per < rows ? beg + per : rows;
    int64_t local = 0;
    for (int64_t r = beg; r < end; ++r) local += counts[r];
    // inclusive scan of `local` over the block
    int64_t x = local;
    const int lane = tid & 31, wid = tid >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[wid] = x;
    __syncthreads();
    if (wid == 0) {
        int64_t t = warp_tot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        warp_tot[lane] = t;
    }
    __syncthreads();
    int64_t run = x - local + (wid > 0 ? warp_tot[wid - 1] : 0);
    for (int64_t r = beg; r < end; ++r) {
        run += counts[r];
        row_ptr[r + 1] = (int32_t)run;
    }
    if (tid == 0) row_ptr[0] = 0;
}

// Copy each padded CDF row to its CSR position (one warp per row).
__global__ void __launch_bounds__(256) compact_kernel(const int32_t* __restrict__ counts,
                                                      const int32_t* __restrict__ padded,
                                                      int pad_stride, int64_t rows,
                                                      const int32_t* __restrict__ row_ptr,
                                                      int32_t* __restrict__ col_idx,
                                                      int64_t col_cap, uint32_t* status) {
    const int lane = threadIdx.x & 31;
    const int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (w >= rows) return;
    const int64_t off = row_ptr[w];
    const int n = counts[w];
    if (off + n > col_cap) {
        if (lane == 0) atomicOr(status, kStatusCapacity);
        return;
    }
    for (int e = lane; e < n; e += 32) col_idx[off + e] = padded[w * (int64_t)pad_stride + e];
}

// ------------------------------------------------------------------------
// Key chunks larger than the query chunk: each selected key chunk is replaced
// by the (4,4,8) boxes it covers inside the grid (box ids on the query-chunk
// grid), so the attention kernels see a CSR over 128-token boxes.
struct BoxGrid {
    int NT, NH, NW;     // boxes per axis
    int mT, mH, mW;     // boxes per key chunk per axis
    int NkH, NkW, Nk;   // key chunks along h, w and in total
};

__device__ __forceinline__ void key_chunk_boxes(const BoxGrid& g, int kc, int& t0, int& h0, int& w0,
                                                int& nt, int& nh, int& nw) {
    const int kct = kc / (g.NkH * g.NkW), kch = (kc / g.NkW) % g.NkH, kcw = kc % g.NkW;
    t0 = kct * g.mT;
    h0 = kch * g.mH;
    w0 = kcw * g.mW;
    nt = min(g.mT, g.NT - t0);
    nh = min(g.mH, g.NH - h0);
    nw = min(g.mW, g.NW - w0);
}

// One warp per row: boxes of the row's key chunks.
__global__ void __launch_bounds__(256) expand_count_kernel(const int32_t* __restrict__ kc_row_ptr,
                                                           const int32_t* __restrict__ kc_col_idx,
                                                           int64_t rows, BoxGrid g,
                                                           int32_t* __restrict__ counts) {
    const int lane = threadIdx.x & 31;
    const int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (w >= rows) return;
    int n = 0;
    for (int64_t e = kc_row_ptr[w] + lane; e < kc_row_ptr[w + 1]; e += 32) {
        int t0, h0, w0, nt, nh, nw;
        key_chunk_boxes(g, kc_col_idx[e], t0, h0, w0, nt, nh, nw);
        n += nt * nh * nw;
    }
    n = __reduce_add_sync(0xffffffffu, n);
    if (lane == 0) counts[w] = n;
}

// One warp per row: each lane writes the boxes of one key chunk, key chunks in
// row order, boxes in (t, h, w) order inside a key chunk.
__global__ void __launch_bounds__(256) expand_emit_kernel(const int32_t* __restrict__ kc_row_ptr,
                                                          const int32_t* __restrict__ kc_col_idx,
                                                          int64_t rows, BoxGrid g,
                                                          const int32_t* __restrict__ row_ptr,
                                                          int32_t* __restrict__ col_idx,
                                                          int64_t col_cap, uint32_t* status) {
    const int lane = threadIdx.x & 31;
    const int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (w >= rows) return;
    if (row_ptr[w + 1] > col_cap) {
        if (lane == 0) atomicOr(status, kStatusCapacity);
        return;
    }
    int64_t run = row_ptr[w];
    const int64_t beg = kc_row_ptr[w], end = kc_row_ptr[w + 1];
    for (int64_t e0 = beg; e0 < end; e0 += 32) {
        const int64_t e = e0 + lane;
        int t0 = 0, h0 = 0, w0 = 0, nt = 0, nh = 0, nw = 0;
        if (e < end) key_chunk_boxes(g, kc_col_idx[e], t0, h0, w0, nt, nh, nw);
        const int n = nt * nh * nw;
        int incl = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int64_t pos = run + (incl - n);
        for (int a = 0; a < nt; ++a)
            for (int b = 0; b < nh; ++b)
                for (int c = 0; c < nw; ++c)
                    col_idx[pos++] = ((t0 + a) * g.NH + (h0 + b)) * g.NW + (w0 + c);
        run += __shfl_sync(0xffffffffu, incl, 31);
    }
}

// ------------------------------------------------------------------------
// 64-token query chunks: the attention kernel works on (4,4,8) boxes of
// queries, i.e. on the two w-adjacent query chunks of a box at once. Each box
// row lists the union of the key boxes its two chunks selected, in ascending
// order, with a 4-bit quadrant pattern per entry: bits 0-1 are the key halves
// (lw < 4, lw >= 4) the box's left query chunk attends to, bits 2-3 those of
// its right query chunk. One warp per box row: its lanes read the two chunk
// rows (coalesced) into four bitmaps over the key boxes, one per quadrant, in
// shared memory; the union is their OR, emitted in ascending box order. The
// order of a row's entries does not matter and duplicates collapse.
struct QuadGrid {
    int NH, NW, NWq;   // boxes along h, w; query chunks along w
    int NkW;           // key chunks along w
    int kw64;          // key chunks are (4,4,4) half-boxes (else whole boxes)
    int Nq, Nk, NB;    // query chunks, key chunks, boxes per (batch, head)
    int64_t rows;      // box rows: batch*heads * NB
};

constexpr int kQuadMaxWords = 64;  // 32-bit words per quadrant bitmap: up to 2,048 key boxes

__device__ __forceinline__ void key_box_of(const QuadGrid& g, int kc, int& box, int& bits) {
    if (g.kw64) {
        const int kt = kc / (g.NH * g.NkW), kh = (kc / g.NkW) % g.NH, kw4 = kc % g.NkW;
        box = (kt * g.NH + kh) * g.NW + (kw4 >> 1);
        bits = 1 << (kw4 & 1);
    } else {
        box = kc;
        bits = 3;
    }
}

template <bool kEmit>
__global__ void __launch_bounds__(256) quad_union_kernel(
    const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx, int64_t col_cap,
    QuadGrid g, int32_t* __restrict__ counts, const int32_t* __restrict__ box_row_ptr,
    int32_t* __restrict__ box_col, uint8_t* __restrict__ box_pat, int64_t box_cap,
    uint32_t* status) {
    __shared__ uint32_t bitmap[8][4][kQuadMaxWords];  // [warp][quadrant][word]
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int64_t r = (int64_t)blockIdx.x * 8 + wib;
    if (r >= g.rows) return;  // warp-uniform
    uint32_t (*bm)[kQuadMaxWords] = bitmap[wib];
    const int words = (g.NB + 31) >> 5;
    for (int w = lane; w < words; w += 32)
        for (int qd = 0; qd < 4; ++qd) bm[qd][w] = 0u;
    __syncwarp();
    const int64_t bh = r / g.NB;
    const int b = (int)(r % g.NB);
    const int bt = b / (g.NH * g.NW), bhh = (b / g.NW) % g.NH, bw = b % g.NW;
    const int q0 = (bt * g.NH + bhh) * g.NWq + 2 * bw;  // the box's left query chunk
    bool bad = false;
    for (int side = 0; side < 2; ++side) {
        if (side == 1 && 2 * bw + 1 >= g.NWq) continue;  // no right chunk at the grid edge
        const int64_t row = bh * g.Nq + q0 + side;
        const int64_t beg = row_ptr[row], end = row_ptr[row + 1];
        if (!(beg >= 0 && end >= beg && end <= col_cap && end - beg <= g.Nk)) {
            bad = true;
            continue;
        }
        for (int64_t e = beg + lane; e < end; e += 32) {
            const int c = col_idx[e];
            if (c < 0 || c >= g.Nk) {
                bad = true;
                continue;
            }
            int box, bits;
            key_box_of(g, c, box, bits);
            for (int kh = 0; kh < 2; ++kh)
                if (bits & (1 << kh)) atomicOr(&bm[2 * side + kh][box >> 5], 1u << (box & 31));
        }
    }
    __syncwarp();
    if (kEmit && box_row_ptr[r + 1] > box_cap) {
        if (lane == 0) atomicOr(status, kStatusCapacity);
        return;
    }
    int64_t run = kEmit ? box_row_ptr[r] : 0;
    int total = 0;
    for (int w0 = 0; w0 < words; w0 += 32) {  // ascending: word w0 + lane per round
        const int w = w0 + lane;
        const uint32_t a0 = w < words ? bm[0][w] : 0u, a1 = w < words ? bm[1][w] : 0u;
        const uint32_t a2 = w < words ? bm[2][w] : 0u, a3 = w < words ? bm[3][w] : 0u;
        uint32_t any = a0 | a1 | a2 | a3;
        const int n = __popc(any);
        int incl = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (kEmit) {
            int64_t pos = run + (incl - n);
            while (any) {
                const int bit = __ffs(any) - 1;
                any &= any - 1;
                const uint32_t m = 1u << bit;
                box_col[pos] = w * 32 + bit;
                box_pat[pos] = static_cast<uint8_t>(((a0 & m) ? 1 : 0) | ((a1 & m) ? 2 : 0) |
                                                    ((a2 & m) ? 4 : 0) | ((a3 & m) ? 8 : 0));
                ++pos;
            }
        }
        const int round = __shfl_sync(0xffffffffu, incl, 31);
        run += round;
        total += round;
    }
    if (!kEmit && lane == 0) counts[r] = total;
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(status, kStatusBadIndex);
}

// One CTA waits on an mbarrier that nothing arrives at; the bounded wait
// expires, records the timeout and the kernel returns normally.
__global__ void selftest_timeout_kernel(uint32_t* status, uint64_t timeout_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, &abort_flag, status, timeout_ns);
    __syncthreads();
}

}  // namespace

cudaError_t launch_pool(const Dims& g, const void* x0, const void* x1, float* p0, float* p1,
                        cudaStream_t st) {
    // with two tensors (plan): x0 = Q pools the computed query chunks, x1 = K
    // pools every key chunk; with one tensor it pools every query chunk of x0
    const PoolSide sq{x1 ? g.q_skip : 0, x1 ? g.Nq : g.Nc, 1, 1, 1, g.NH, g.NWq, g.qw};
    const PoolSide sk{0, g.Nk, g.mT, g.mH, g.mW, g.NkH, g.NkW, g.kw64 ? kChunkW / 2 : kChunkW};
    const int nx = x1 ? (g.Nq > g.Nk ? g.Nq : g.Nk) : g.Nc;
    dim3 grid((unsigned)nx, (unsigned)g.BH, x1 ? 2 : 1);
    const auto* a = static_cast<const __nv_bfloat16*>(x0);
    const auto* b = static_cast<const __nv_bfloat16*>(x1 ? x1 : x0);
    if (g.d == 128)
        pool_kernel<128><<<grid, 256, 0, st>>>(a, b, p0, p1 ? p1 : p0, sq, sk, g.T, g.H, g.W, g.N);
    else
        pool_kernel<64><<<grid, 256, 0, st>>>(a, b, p0, p1 ? p1 : p0, sq, sk, g.T, g.H, g.W, g.N);
    return cudaGetLastError();
}

cudaError_t launch_rearrange(const Dims& g, const void* src, void* dst, int inverse,
                             cudaStream_t st) {
    dim3 grid(g.Nc, (unsigned)g.BH);
    const auto* s = static_cast<const __nv_bfloat16*>(src);
    auto* d = static_cast<__nv_bfloat16*>(dst);
    if (g.d == 128)
        rearrange_kernel<128><<<grid, 256, 0, st>>>(s, d, g.T, g.H, g.W, g.NH, g.NW, g.Nc, g.N,
                                                    inverse);
    else
        rearrange_kernel<64><<<grid, 256, 0, st>>>(s, d, g.T, g.H, g.W, g.NH, g.NW, g.Nc, g.N,
                                                   inverse);
    return cudaGetLastError();
}

cudaError_t launch_scores(const Dims& g, const float* qp, const float* kp, float* S,
                          cudaStream_t st, int kshard) {
    dim3 grid((g.Nk + 127) / 128, (g.Nq + 127) / 128, (unsigned)g.BH);
    scores_kernel<<<grid, 256, 0, st>>>(qp, kp, S, g.Nq, g.Nk, kshard > 0 ? kshard : g.Nk, g.d,
                                        g.scale);
    return cudaGetLastError();
}

cudaError_t launch_select(const Dims& g, const bsa_params& p, const float* S, int32_t* row_ptr,
                          int32_t* col_idx, int64_t col_cap, int32_t* counts, int32_t* padded,
                          int pad_stride, uint32_t* status, cudaStream_t st) {
    const unsigned blocks = (unsigned)((g.rows + 7) / 8);
    const int mode = p.mode;
#define BSA_SELECT(MJ)                                                                       \
    select_kernel<MJ><<<blocks, 256, 0, st>>>(S, g.Nc, g.Nk, g.n_cond, g.n_cond_k, g.q_skip,   \
                                              g.Nq, g.rows, mode, p.topk, p.cdf_p,           \
                                              p.cdf_cap_frac, row_ptr, col_idx, col_cap,     \
                                              counts, padded, pad_stride, status)
    // keys per lane: the smallest instantiation that holds the row (the searches
    // cost one compare per key slot and step, so padding slots are not free)
    if (g.Nk <= 32) BSA_SELECT(1);
    else if (g.Nk <= 256) BSA_SELECT(8);
    else if (g.Nk <= 512) BSA_SELECT(16);
    else if (g.Nk <= 768) BSA_SELECT(24);
    else if (g.Nk <= 1024) BSA_SELECT(32);
    else if (g.Nk <= 1280) BSA_SELECT(40);
    else if (g.Nk <= 1536) BSA_SELECT(48);
    else if (g.Nk <= 1792) BSA_SELECT(56);
    else if (g.Nk <= 2048) BSA_SELECT(64);
    else return cudaErrorInvalidValue;
#undef BSA_SELECT
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || mode == BSA_SEL_TOPK) return e;
    scan_counts_kernel<<<1, 1024, 0, st>>>(counts, g.rows, row_ptr);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    compact_kernel<<<blocks, 256, 0, st>>>(counts, padded, pad_stride, g.rows, row_ptr, col_idx,
                                           col_cap, status);
    return cudaGetLastError();
}

cudaError_t launch_scan_counts(const int32_t* counts, int64_t n, int32_t* ptr, cudaStream_t st) {
    scan_counts_kernel<<<1, 1024, 0, st>>>(counts, n, ptr);
    return cudaGetLastError();
}

cudaError_t launch_expand_boxes(const Dims& g, const int32_t* kc_row_ptr,
                                const int32_t* kc_col_idx, int32_t* counts, int32_t* row_ptr,
                                int32_t* col_idx, int64_t col_cap, uint32_t* status,
                                cudaStream_t st) {
    const BoxGrid bg{g.NT, g.NH, g.NW, g.mT, g.mH, g.mW, g.NkH, g.NkW, g.Nk};
    const unsigned blocks = (unsigned)((g.rows + 7) / 8);
    expand_count_kernel<<<blocks, 256, 0, st>>>(kc_row_ptr, kc_col_idx, g.rows, bg, counts);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    scan_counts_kernel<<<1, 1024, 0, st>>>(counts, g.rows, row_ptr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    expand_emit_kernel<<<blocks, 256, 0, st>>>(kc_row_ptr, kc_col_idx, g.rows, bg, row_ptr,
                                               col_idx, col_cap, status);
    return cudaGetLastError();
}

cudaError_t launch_quad_union(const Dims& g, const int32_t* row_ptr, const int32_t* col_idx,
                              int64_t col_cap, int32_t* counts, int32_t* box_row_ptr,
                              int32_t* box_col, uint8_t* box_pat, int64_t box_cap,
                              uint32_t* status, cudaStream_t st) {
    const QuadGrid qg{g.NH, g.NW, g.NWq, g.NkW, g.kw64, g.Nq, g.Nk, g.NB, g.BH * g.NB};
    if (g.NB > 32 * kQuadMaxWords) return cudaErrorInvalidValue;  // not reachable: NB <= Nc
    const unsigned blocks = (unsigned)((qg.rows + 7) / 8);          // a warp per box row
    quad_union_kernel<false><<<blocks, 256, 0, st>>>(row_ptr, col_idx, col_cap, qg, counts,
                                                     nullptr, nullptr, nullptr, 0, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    scan_counts_kernel<<<1, 1024, 0, st>>>(counts, qg.rows, box_row_ptr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    quad_union_kernel<true><<<blocks, 256, 0, st>>>(row_ptr, col_idx, col_cap, qg, counts,
                                                    box_row_ptr, box_col, box_pat, box_cap,
                                                    status);
    return cudaGetLastError();
}

cudaError_t launch_selftest_timeout(uint32_t* status, uint64_t timeout_ns, cudaStream_t st) {
    selftest_timeout_kernel<<<1, 32, 0, st>>>(status, timeout_ns);
    return cudaGetLastError();
}

}  // namespace bsa
