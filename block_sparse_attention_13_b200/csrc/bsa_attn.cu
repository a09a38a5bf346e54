// Block-sparse attention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// Method ("LongCat-Video Technical Report", section "Block Sparse Attention
// (BSA)", "Sparse attention computation"): O = softmax(QK^T/sqrt(d)) V with
// the logits of non-selected key blocks at -inf, i.e. for each query chunk an
// exact softmax over the 128-token key chunks its CSR row lists. Evaluated with
// an online softmax across the chunks ("LongCat-Video Technical Report #",
// section "3D Block Sparse Attention": online softmax over variable-length
// block lists), bf16 tensor-core products and fp32 accumulation.
//
// One CTA owns one query chunk (128 queries = one M=128 MMA tile). Q, K, V and
// O are addressed directly in [T,H,W] token order through 5-D TMA maps whose
// box (64 ch, 8 w, 4 h, 4 t) lands a (4,4,8) chunk in shared memory already in
// chunk-local order, so neither the forward rearrangement nor its inverse
// costs a pass over HBM.
//
// Roles (192 threads): warps 0-3 softmax + epilogue (thread m owns query row m
// = TMEM lane m); warp 4 TMA producer; warp 5 TMEM allocator + MMA issuer.
// TMEM (256 columns): S = Q K^T at [0,128) fp32; P = softmax numerators are
// written back over S as packed bf16 (64 columns) and feed the PV MMA as the
// TMEM A operand; O accumulates at [128, 128+d). Per chunk the MMA warp issues
// S (SS MMA), waits for P, issues O += P V (TS MMA) and waits for it before
// the next S overwrites P. Two CTAs share an SM (<100 KB smem, 256 TMEM
// columns, <=168 registers each), so one CTA's softmax overlaps the other's
// MMAs. O is rescaled in TMEM only when the running max grows by more than
// 2^8 (exact: the final normalisation uses the same reference max).
//
// Every mbarrier wait is bounded; on expiry the CTA records a timeout in the
// status word, drains its in-flight TMA and MMA work, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bsa_internal.cuh"
#include "bsa_ptx.cuh"

namespace bsa {

namespace {

template <int D>
struct AttnCfg {
    static constexpr int kHalfBytes = 128 * 64 * 2;  // one TMA box: 128 tokens x 64 channels
    static constexpr int kHalves = D / 64;
    static constexpr int kTileBytes = kHalves * kHalfBytes;
    static constexpr int kQ = 0;
    static constexpr int kK = kTileBytes;
    static constexpr int kV = 2 * kTileBytes;
    static constexpr int kCtl = 3 * kTileBytes;
    static constexpr int kSmemBytes = kCtl + 256 + 1024;  // + control block + alignment slack
    static constexpr uint32_t kTmemCols = 256;
    static constexpr uint32_t kSCol = 0;
    static constexpr uint32_t kOCol = 128;
    static constexpr int kThreads = 192;
};

struct FwdArgs {
    const int32_t* row_ptr;
    const int32_t* col_idx;
    int64_t col_cap;
    __nv_bfloat16* out;
    float* lse;
    uint32_t* status;
    int H, W, NH, NW, Nc;
    int64_t N;
    float scale_log2;  // softmax scale * log2(e)
    uint64_t timeout_ns;
    int debug_flags;   // bit 0: withhold the first S-ready signal (timeout test)
};

struct __align__(8) Ctl {
    uint64_t q_full, k_full, k_empty, v_full, v_empty, s_full, p_full, o_full, aux;
    uint32_t tmem_base;
    int abort_flag;
    int n_valid;
};

// Wait used only while draining after an abort: ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > timeout_ns) return;
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ bool bar_red_and(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"(pred ? 1u : 0u), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

template <int D>
__global__ void __launch_bounds__(192, 2)
    bsa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const FwdArgs a) {
    using C = AttnCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    Ctl* ctl = reinterpret_cast<Ctl*>(smem + C::kCtl);
    const uint32_t sQ = smem_u32(smem + C::kQ);
    const uint32_t sK = smem_u32(smem + C::kK);
    const uint32_t sV = smem_u32(smem + C::kV);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t row = blockIdx.x;
    const int64_t bh = row / a.Nc;
    const int qc = static_cast<int>(row % a.Nc);
    const int q_t = (qc / (a.NH * a.NW)) * kChunkT;
    const int q_h = ((qc / a.NW) % a.NH) * kChunkH;
    const int q_w = (qc % a.NW) * kChunkW;

    // Row extent; an invalid row is treated as empty and reported.
    int64_t beg = a.row_ptr[row], end = a.row_ptr[row + 1];
    const bool row_ok = beg >= 0 && end >= beg && end <= a.col_cap && end - beg <= a.Nc;
    if (!row_ok) beg = end = 0;

    if (threadIdx.x == 0) {
        mbar_init(&ctl->q_full, 1);
        mbar_init(&ctl->k_full, 1);
        mbar_init(&ctl->k_empty, 1);
        mbar_init(&ctl->v_full, 1);
        mbar_init(&ctl->v_empty, 1);
        mbar_init(&ctl->s_full, 1);
        mbar_init(&ctl->p_full, 128);
        mbar_init(&ctl->o_full, 1);
        mbar_init(&ctl->aux, 1);
        ctl->abort_flag = 0;
        int nv = 0;
        bool bad = !row_ok;
        for (int64_t e = beg; e < end; ++e) {
            const int c = a.col_idx[e];
            if (c >= 0 && c < a.Nc) ++nv; else bad = true;
        }
        ctl->n_valid = nv;
        if (bad) atomicOr(a.status, kStatusBadIndex);
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 5) {
        tmem_alloc(&ctl->tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    if (warp == 4 && lane == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_o);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    const int n_valid = ctl->n_valid;
    volatile int* abort_flag = &ctl->abort_flag;
    const uint64_t tmo = a.timeout_ns;

    if (warp == 4) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && n_valid > 0) {
            mbar_arrive_expect_tx(&ctl->q_full, C::kTileBytes);
#pragma unroll
            for (int h = 0; h < C::kHalves; ++h)
                tma_load_5d(&tm_q, sQ + h * C::kHalfBytes, &ctl->q_full, h * 64, q_w, q_h, q_t,
                            static_cast<int>(bh));
            int nk = 0, nv = 0;
            bool aborted = false;
            for (int64_t e = beg; e < end; ++e) {
                const int c = a.col_idx[e];
                if (c < 0 || c >= a.Nc) continue;
                const int kt = (c / (a.NH * a.NW)) * kChunkT;
                const int kh = ((c / a.NW) % a.NH) * kChunkH;
                const int kw = (c % a.NW) * kChunkW;
                if (nk > 0 && !mbar_wait(&ctl->k_empty, (nk - 1) & 1, abort_flag, a.status, tmo)) {
                    aborted = true;
                    break;
                }
                mbar_arrive_expect_tx(&ctl->k_full, C::kTileBytes);
#pragma unroll
                for (int h = 0; h < C::kHalves; ++h)
                    tma_load_5d(&tm_k, sK + h * C::kHalfBytes, &ctl->k_full, h * 64, kw, kh, kt,
                                static_cast<int>(bh));
                ++nk;
                if (nv > 0 && !mbar_wait(&ctl->v_empty, (nv - 1) & 1, abort_flag, a.status, tmo)) {
                    aborted = true;
                    break;
                }
                mbar_arrive_expect_tx(&ctl->v_full, C::kTileBytes);
#pragma unroll
                for (int h = 0; h < C::kHalves; ++h)
                    tma_load_5d(&tm_v, sV + h * C::kHalfBytes, &ctl->v_full, h * 64, kw, kh, kt,
                                static_cast<int>(bh));
                ++nv;
            }
            if (aborted || *abort_flag) {
                // let the copies already issued land before shared memory is released
                drain_wait(&ctl->q_full, 0, tmo);
                if (nk > 0) drain_wait(&ctl->k_full, (nk - 1) & 1, tmo);
                if (nv > 0) drain_wait(&ctl->v_full, (nv - 1) & 1, tmo);
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n_valid > 0) {
            constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, 0, 0);  // Q, K both K-major
            constexpr uint32_t kIdO = idesc_bf16_f32(128, D, 0, 1);    // P from TMEM, V MN-major
            const uint32_t tS = tmem + C::kSCol;
            const uint32_t tO = tmem + C::kOCol;
            bool aborted = !mbar_wait(&ctl->q_full, 0, abort_flag, a.status, tmo);
            bool issued = false;
            for (int it = 0; it < n_valid && !aborted; ++it) {
                if (!mbar_wait(&ctl->k_full, it & 1, abort_flag, a.status, tmo)) { aborted = true; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kHalfBytes + (kk & 3) * 32;
                    mma_ss(tS, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(sK + off, 16, 1024),
                           kIdS, kk > 0 ? 1u : 0u);
                }
                issued = true;
                tc_commit(&ctl->k_empty);
                if (!((a.debug_flags & 1) && it == 0)) tc_commit(&ctl->s_full);
                if (!mbar_wait(&ctl->p_full, it & 1, abort_flag, a.status, tmo)) { aborted = true; break; }
                tc_fence_after();
                if (!mbar_wait(&ctl->v_full, it & 1, abort_flag, a.status, tmo)) { aborted = true; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tO, tS + kk * 8, sdesc_sw128(sV + kk * 2048, C::kHalfBytes, 1024), kIdO,
                           (it > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&ctl->v_empty);
                // P lives in the S columns: the next S may only start once PV has read it.
                if (it + 1 < n_valid &&
                    !mbar_wait(&ctl->v_empty, it & 1, abort_flag, a.status, tmo)) { aborted = true; break; }
            }
            if (!aborted) {
                tc_commit(&ctl->o_full);
            } else if (issued) {
                tc_commit(&ctl->aux);
                drain_wait(&ctl->aux, 0, tmo);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int m = threadIdx.x;  // query row = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t tS = tmem + lane_off + C::kSCol;
        const uint32_t tO = tmem + lane_off + C::kOCol;
        const float c2 = a.scale_log2;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int it = 0; it < n_valid; ++it) {
            const bool got = mbar_wait(&ctl->s_full, it & 1, abort_flag, a.status, tmo);
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
            float mx = -INFINITY;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                uint32_t s[32];
                tmem_ld32(tS + g * 32, s);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) mx = fmaxf(mx, __uint_as_float(s[j]));
            }
            const float m_new = mx * c2;
            if (it == 0) {
                m_run = m_new;
            } else if (m_new > m_run + 8.0f) {
                // O holds the chunks before this one (their PV completed before S was
                // signalled); rescale it to the new reference max.
                const float alpha = ex2_approx(m_run - m_new);
                l_run *= alpha;
#pragma unroll
                for (int g = 0; g < D / 32; ++g) {
                    uint32_t o[32];
                    tmem_ld32(tO + g * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                    tmem_st32(tO + g * 32, o);
                }
                tmem_wait_st();
                m_run = m_new;
            }
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                uint32_t s[32];
                tmem_ld32(tS + g * 32, s);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float p0 = ex2_approx(fmaf(__uint_as_float(s[2 * j]), c2, -m_run));
                    const float p1 = ex2_approx(fmaf(__uint_as_float(s[2 * j + 1]), c2, -m_run));
                    l_run += p0 + p1;
                    pk[j] = pack_bf16x2(p0, p1);
                }
                tmem_st16(tS + g * 16, pk);  // P columns [16g, 16g+16) were read as S already
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&ctl->p_full);
        }
        if (ok && n_valid > 0) {
            const bool got = mbar_wait(&ctl->o_full, 0, abort_flag, a.status, tmo);
            ok = __all_sync(0xffffffffu, got);
        }
        const bool all_ok = bar_red_and(1, 128, ok);
        const int lt = m >> 5, lh = (m >> 3) & 3, lw = m & 7;
        const int64_t tok = (static_cast<int64_t>(q_t + lt) * a.H + (q_h + lh)) * a.W + q_w + lw;
        if (all_ok && n_valid > 0) {
            tc_fence_after();
            const float inv_l = 1.0f / l_run;
            uint8_t* stage = smem + C::kQ;  // Q is dead once O is final
#pragma unroll
            for (int g = 0; g < D / 32; ++g) {
                uint32_t o[32];
                tmem_ld32(tO + g * 32, o);
                tmem_wait_ld();
                const int half = (g * 32) / 64;
                const int chunk0 = ((g * 32) % 64) / 8;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    uint4 val;
                    val.x = pack_bf16x2(__uint_as_float(o[c4 * 8 + 0]) * inv_l, __uint_as_float(o[c4 * 8 + 1]) * inv_l);
                    val.y = pack_bf16x2(__uint_as_float(o[c4 * 8 + 2]) * inv_l, __uint_as_float(o[c4 * 8 + 3]) * inv_l);
                    val.z = pack_bf16x2(__uint_as_float(o[c4 * 8 + 4]) * inv_l, __uint_as_float(o[c4 * 8 + 5]) * inv_l);
                    val.w = pack_bf16x2(__uint_as_float(o[c4 * 8 + 6]) * inv_l, __uint_as_float(o[c4 * 8 + 7]) * inv_l);
                    const int chunk = chunk0 + c4;
                    *reinterpret_cast<uint4*>(stage + half * C::kHalfBytes + m * 128 +
                                              ((chunk ^ (m & 7)) << 4)) = val;
                }
            }
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (m == 0) {
#pragma unroll
                for (int h = 0; h < C::kHalves; ++h)
                    tma_store_5d(&tm_o, sQ + h * C::kHalfBytes, h * 64, q_w, q_h, q_t,
                                 static_cast<int>(bh));
                tma_store_commit_and_wait_all();
            }
            if (a.lse) a.lse[bh * a.N + tok] = (m_run + __log2f(l_run)) * 0.69314718055994530942f;
        } else if (all_ok) {
            // empty (or rejected) row: zeros, lse = -inf
            uint4 z = make_uint4(0u, 0u, 0u, 0u);
            uint4* dst = reinterpret_cast<uint4*>(a.out + (bh * a.N + tok) * D);
#pragma unroll
            for (int j = 0; j < D / 8; ++j) dst[j] = z;
            if (a.lse) a.lse[bh * a.N + tok] = -INFINITY;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// 5-D tiled map over a [BH][T][H][W][D] bf16 tensor with a (64,8,4,4,1) box and
// 128-byte swizzle: one box is 128 tokens of one chunk x 64 channels.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

bool make_chunk_map(CUtensorMap* tm, const void* base, const Dims& g) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[5] = {(cuuint64_t)g.d, (cuuint64_t)g.W, (cuuint64_t)g.H,
                                (cuuint64_t)g.T, (cuuint64_t)g.BH};
    const cuuint64_t strides[4] = {(cuuint64_t)g.d * 2, (cuuint64_t)g.W * g.d * 2,
                                   (cuuint64_t)g.H * g.W * g.d * 2,
                                   (cuuint64_t)g.T * g.H * g.W * g.d * 2};
    const cuuint32_t box[5] = {64, kChunkW, kChunkH, kChunkT, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_fwd_d(const Dims& g, const CUtensorMap& mq, const CUtensorMap& mk,
                         const CUtensorMap& mv, const CUtensorMap& mo, const FwdArgs& args,
                         cudaStream_t st) {
    using C = AttnCfg<D>;
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(bsa_fwd_kernel<D>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    bsa_fwd_kernel<D><<<(unsigned)g.rows, C::kThreads, C::kSmemBytes, st>>>(mq, mk, mv, mo, args);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_forward(const Dims& g, const void* q, const void* k, const void* v,
                           const int32_t* row_ptr, const int32_t* col_idx, int64_t col_cap,
                           void* out, float* lse, uint32_t* status, uint64_t timeout_ns,
                           int debug_flags, cudaStream_t st) {
    CUtensorMap mq, mk, mv, mo;
    if (!make_chunk_map(&mq, q, g) || !make_chunk_map(&mk, k, g) || !make_chunk_map(&mv, v, g) ||
        !make_chunk_map(&mo, out, g))
        return cudaErrorInvalidValue;
    FwdArgs args;
    args.row_ptr = row_ptr;
    args.col_idx = col_idx;
    args.col_cap = col_cap;
    args.out = static_cast<__nv_bfloat16*>(out);
    args.lse = lse;
    args.status = status;
    args.H = g.H;
    args.W = g.W;
    args.NH = g.NH;
    args.NW = g.NW;
    args.Nc = g.Nc;
    args.N = g.N;
    args.scale_log2 = g.scale * 1.4426950408889634f;
    args.timeout_ns = timeout_ns;
    args.debug_flags = debug_flags;
    return g.d == 128 ? launch_fwd_d<128>(g, mq, mk, mv, mo, args, st)
                      : launch_fwd_d<64>(g, mq, mk, mv, mo, args, st);
}

}  // namespace bsa
