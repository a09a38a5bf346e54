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
// A query chunk (128 queries) is one M=128 MMA tile. Q, K, V and O are
// addressed directly in [T,H,W] token order through 5-D TMA maps whose box
// (64 ch, 8 w, 4 h, 4 t) lands a (4,4,8) chunk in shared memory already in
// chunk-local order, so neither the forward rearrangement nor its inverse
// costs a pass over HBM.
//
// One CTA per SM holds two query chunks (tiles 0 and 1: consecutive CSR rows,
// so usually neighbours in the same head, whose key chunks share L2). Roles
// (320 threads): warps 0-3 and 4-7 are the softmax + epilogue warpgroups of
// tiles 0 and 1 (thread m of a group owns query row m = TMEM lane m); warp 8
// is the TMA producer; warp 9 allocates TMEM and issues the MMAs.
// TMEM (512 columns): S0, S1 = Q K^T fp32 at [0,128) and [128,256); the
// softmax numerators P are written back over the first 64 columns of S as
// packed bf16 and feed the PV MMA as its TMEM A operand; O0, O1 accumulate at
// [256,384) and [384,512). The MMA warp alternates tiles (PV0, S0', PV1, S1'),
// so one tile's softmax overlaps the other tile's MMAs. O is rescaled in TMEM
// only when the running max grows by more than 2^8 (exact: the final
// normalisation uses the same reference max).
//
// Every mbarrier wait is bounded; on expiry the CTA records a timeout in the
// status word, drains its in-flight TMA and MMA work, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "bsa_internal.cuh"
#include "bsa_ptx.cuh"

namespace bsa {

namespace {

// Every kPolyEvery-th pair of softmax exponentials is evaluated by the FMA-pipe
// polynomial instead of the MUFU unit (0 = all on MUFU).
#ifndef BSA_POLY_EVERY
#define BSA_POLY_EVERY 4
#endif
constexpr int kPolyEvery = BSA_POLY_EVERY;

template <int D>
struct AttnCfg {
    static constexpr int kHalfBytes = 128 * 64 * 2;  // one TMA box: 128 tokens x 64 channels
    static constexpr int kHalves = D / 64;
    static constexpr int kTileBytes = kHalves * kHalfBytes;
    // shared memory: Q0 Q1 K0 K1 V0 V1 (one buffer each per tile), control block
    static constexpr int q_off(int t) { return t * kTileBytes; }
    static constexpr int k_off(int t) { return (2 + t) * kTileBytes; }
    static constexpr int v_off(int t) { return (4 + t) * kTileBytes; }
    static constexpr int kCtl = 6 * kTileBytes;
    static constexpr int kMaxChunks = 2048;                // Nc limit of the library
    static constexpr int kList = kCtl + 512;               // uint16 chunk lists of both tiles
    // Grids with partial edge chunks: the edge pattern of every listed chunk (uint8),
    // then the operands of the masking product (see bsa_fwd_kernel): a ones tile and
    // one bias tile per edge pattern 1..7, each 128 rows x 8 bf16 (2 KB), K-major
    // without swizzle.
    static constexpr int kPat = kList + 2 * kMaxChunks * 2;
    static constexpr int kBias = kPat + 2 * kMaxChunks;
    static constexpr int kBiasTile = 128 * 16;
    static constexpr int kSmemBytes = kBias + 8 * kBiasTile + 1024;  // + alignment slack
    // tensor memory: S0 S1 (fp32 128x128; P is written over S as bf16) O0 O1
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t s_col(int t) { return t * 128; }
    static constexpr uint32_t o_col(int t) { return 256 + t * 128; }
    static constexpr int kThreads = 320;  // softmax WG0, softmax WG1, TMA warp, MMA warp
    static constexpr int kTmaWarp = 8;
    static constexpr int kMmaWarp = 9;
};

struct FwdArgs {
    const int32_t* row_ptr;
    const int32_t* col_idx;
    int64_t col_cap;
    __nv_bfloat16* out;
    float* out_f32;    // non-null: O is written here in fp32 instead of bf16 to `out`
    const uint8_t* quad;  // 64-token query chunks: quadrant pattern of every CSR entry
    float* lse;
    uint32_t* status;
    int T, H, W, NH, NW, Nc;
    int q_skip, Nq;    // CSR row r is query chunk q_skip + r % Nq of (batch, head) r / Nq
    int64_t N;
    int64_t rows;
    float scale_log2;  // softmax scale * log2(e)
    uint64_t timeout_ns;
    int debug_flags;   // bit 0: withhold the first S-ready signal (timeout test);
                       // bit 1: count finished CTAs in status[8]
};

struct __align__(8) TileBars {
    uint64_t q_full, k_full, k_empty, v_full, v_empty, s_full, p_full, o_full;
};

struct __align__(8) Ctl {
    TileBars tb[2];
    uint64_t aux;
    int n_valid[2];
    uint32_t tmem_base;
    int abort_flag;
};

// Two query chunks ("tiles" 0 and 1, CSR rows 2*blockIdx.x and 2*blockIdx.x+1)
// per CTA, one CTA per SM. The MMA warp issues, per key-chunk step j,
//   PV0(j), S0(j+1), PV1(j), S1(j+1)
// so each tile's softmax runs while the tensor core works on the other tile.
// S(j+1) is queued right behind the PV(j) that reads P from the same TMEM
// columns: tcgen05 MMAs of one CTA execute in issue order.
// kPartial: the grid has partial edge chunks. The key slots of such a chunk past
// the grid (zero-filled by TMA) must not take part in the softmax, so S of a
// partial key chunk gets one more K = 16 product, ones x bias: A has a 1 in
// column 0 of every row, B has -inf in column 0 of the rows of missing key
// slots and 0 elsewhere (one B tile per edge pattern: partial in t, h, w or a
// combination). Existing slots get exactly +0 and missing ones -inf, as a mask
// would give, and the softmax loop is the same as for full grids.
// kQuad: 64-token query (and key) chunks. A tile is a (4,4,8) box of queries, i.e.
// two w-adjacent query chunks (rows with lw < 4 and lw >= 4), and its CSR row is the
// union of the key boxes they selected; each entry's quadrant pattern says which key
// halves (key slots with lw < 4, lw >= 4) each query half attends to. The softmax
// threads set the logits of the other key halves to -inf before the row max, so the
// result is exactly the attention of each query chunk over its own key chunks.
template <int D, bool kPartial, bool kQuad>
__global__ void __launch_bounds__(320, 1)
    bsa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const FwdArgs a) {
    using C = AttnCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    Ctl* ctl = reinterpret_cast<Ctl*>(smem + C::kCtl);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    uint16_t* lists = reinterpret_cast<uint16_t*>(smem + C::kList);  // [2][kMaxChunks]
    uint8_t* pats = smem + C::kPat;                                   // [2][kMaxChunks]

    if constexpr (kPartial) {
        // ones tile (tile 0) and bias tiles of edge patterns 1..7: row r (key slot r of a
        // chunk: frame r / 32, row (r / 8) % 4, column r % 8) holds 8 bf16, only the
        // first nonzero. Rows are 16 bytes apart, so 8-row core matrices are 128 bytes
        // apart (SBO); both K groups of the product read the same 8 columns (LBO 0).
        const int et = a.T % kChunkT, eh = a.H % kChunkH, ew = a.W % kChunkW;
        for (int i = threadIdx.x; i < 8 * 128; i += blockDim.x) {
            const int tile = i >> 7, r = i & 127;
            const int lt = r >> 5, lh = (r >> 3) & 3, lw = r & 7;
            const bool missing = ((tile & 1) && lt >= et) || ((tile & 2) && lh >= eh) ||
                                 ((tile & 4) && lw >= ew);
            // bf16 bits: 1.0 = 0x3f80, -inf = 0xff80
            const uint32_t first = tile == 0 ? 0x3f80u : (missing ? 0xff80u : 0u);
            *reinterpret_cast<uint4*>(smem + C::kBias + i * 16) = make_uint4(first, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
    }

    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            TileBars& b = ctl->tb[t];
            mbar_init(&b.q_full, 1);
            mbar_init(&b.k_full, 1);
            mbar_init(&b.k_empty, 1);
            mbar_init(&b.v_full, 1);
            mbar_init(&b.v_empty, 1);
            mbar_init(&b.s_full, 1);
            mbar_init(&b.p_full, 128);
            mbar_init(&b.o_full, 1);
        }
        mbar_init(&ctl->aux, 1);
        ctl->abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == C::kTmaWarp) {
        // Stage each tile's chunk list in shared memory (coalesced reads, out-of-range
        // rows and columns dropped and reported), so no global load sits between a
        // freed K/V buffer and the TMA load that refills it.
        bool bad = false;
        for (int t = 0; t < 2; ++t) {
            const int64_t row = 2 * static_cast<int64_t>(blockIdx.x) + t;
            int64_t beg = 0, end = 0;
            if (row < a.rows) {
                beg = a.row_ptr[row];
                end = a.row_ptr[row + 1];
                if (!(beg >= 0 && end >= beg && end <= a.col_cap && end - beg <= a.Nc)) {
                    bad = true;
                    beg = end = 0;
                }
            }
            int cnt = 0;
            for (int64_t e0 = beg; e0 < end; e0 += 32) {
                const int64_t e = e0 + lane;
                const int c = e < end ? a.col_idx[e] : 0;
                const bool valid = e < end && c >= 0 && c < a.Nc;
                if (e < end && !valid) bad = true;
                const uint32_t vb = __ballot_sync(0xffffffffu, valid);
                const int slot = t * C::kMaxChunks + cnt + __popc(vb & ((1u << lane) - 1u));
                if (valid) {
                    lists[slot] = static_cast<uint16_t>(c);
                    // bits 0-2: edge pattern of a partial key box; bits 3-6: quadrant pattern
                    uint32_t pv = 0;
                    if constexpr (kPartial) {
                        int kt, kh, kw;
                        chunk_origin(c, a.NH, a.NW, kt, kh, kw);
                        pv = (kt + kChunkT > a.T ? 1u : 0u) | (kh + kChunkH > a.H ? 2u : 0u) |
                             (kw + kChunkW > a.W ? 4u : 0u);
                    }
                    if constexpr (kQuad) pv |= static_cast<uint32_t>(a.quad[e] & 15u) << 3;
                    if constexpr (kPartial || kQuad) pats[slot] = static_cast<uint8_t>(pv);
                }
                cnt += __popc(vb);
            }
            if (lane == 0) ctl->n_valid[t] = cnt;
        }
        if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(a.status, kStatusBadIndex);
        if (lane == 0) {
            prefetch_tensormap(&tm_q);
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
            prefetch_tensormap(&tm_o);
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
    const int n0 = ctl->n_valid[0], n1 = ctl->n_valid[1];
    const int nmax = n0 > n1 ? n0 : n1;
    volatile int* abort_flag = &ctl->abort_flag;
    const uint64_t tmo = a.timeout_ns;
    // what this thread put in flight (K and V copies per tile; any product), for
    // the drain after an abort
    int nk[2] = {0, 0}, nvv[2] = {0, 0};
    bool issued = false;

    if (warp == C::kTmaWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && nmax > 0) {
            const int n[2] = {n0, n1};
            int bh[2], ct[2], chh[2], cw[2];
            for (int t = 0; t < 2; ++t) {
                const int64_t row = 2 * static_cast<int64_t>(blockIdx.x) + t;
                bh[t] = static_cast<int>(row / a.Nq);
                if (n[t] == 0) continue;
                chunk_origin(a.q_skip + static_cast<int>(row % a.Nq), a.NH, a.NW, ct[t], chh[t], cw[t]);
                mbar_arrive_expect_tx(&ctl->tb[t].q_full, C::kTileBytes);
#pragma unroll
                for (int h = 0; h < C::kHalves; ++h)
                    tma_load_5d(&tm_q, smem_u32(smem + C::q_off(t)) + h * C::kHalfBytes,
                                &ctl->tb[t].q_full, h * 64, cw[t], chh[t], ct[t], bh[t]);
            }
            // The MMA warp frees buffers in the order PV0(j-1), S0(j), PV1(j-1), S1(j)
            // (its issue order), so the loads go out in that order too: V0(j),
            // K0(j+1), V1(j), K1(j+1). Each wait depends only on loads issued by
            // earlier steps of this loop.
            auto load_k = [&](int t, int j) -> bool {
                if (j >= n[t]) return true;
                TileBars& b = ctl->tb[t];
                if (j > 0 && !mbar_wait(&b.k_empty, (j - 1) & 1, abort_flag, a.status, tmo,
                                        site(1, 1, t, j)))
                    return false;
                int kt, kh, kw;
                chunk_origin(lists[t * C::kMaxChunks + j], a.NH, a.NW, kt, kh, kw);
                mbar_arrive_expect_tx(&b.k_full, C::kTileBytes);
#pragma unroll
                for (int h = 0; h < C::kHalves; ++h)
                    tma_load_5d(&tm_k, smem_u32(smem + C::k_off(t)) + h * C::kHalfBytes, &b.k_full,
                                h * 64, kw, kh, kt, bh[t]);
                ++nk[t];
                return true;
            };
            auto load_v = [&](int t, int j) -> bool {
                if (j >= n[t]) return true;
                TileBars& b = ctl->tb[t];
                if (j > 0 && !mbar_wait(&b.v_empty, (j - 1) & 1, abort_flag, a.status, tmo,
                                        site(1, 2, t, j)))
                    return false;
                int vt, vh, vw;
                chunk_origin(lists[t * C::kMaxChunks + j], a.NH, a.NW, vt, vh, vw);
                mbar_arrive_expect_tx(&b.v_full, C::kTileBytes);
#pragma unroll
                for (int h = 0; h < C::kHalves; ++h)
                    tma_load_5d(&tm_v, smem_u32(smem + C::v_off(t)) + h * C::kHalfBytes, &b.v_full,
                                h * 64, vw, vh, vt, bh[t]);
                ++nvv[t];
                return true;
            };
            bool aborted = !(load_k(0, 0) && load_k(1, 0));
            for (int j = 0; j < nmax && !aborted; ++j)
                aborted = !(load_v(0, j) && load_k(0, j + 1) && load_v(1, j) && load_k(1, j + 1));
        }
        __syncwarp();
    } else if (warp == C::kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && nmax > 0) {
            constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, 0, 0);  // Q, K both K-major
            constexpr uint32_t kIdO = idesc_bf16_f32(128, D, 0, 1);    // P from TMEM, V MN-major
            const int n[2] = {n0, n1};
            bool aborted = false;
            for (int t = 0; t < 2 && !aborted; ++t)
                if (n[t] > 0 && !mbar_wait(&ctl->tb[t].q_full, 0, abort_flag, a.status, tmo, site(2, 0, t, 0)))
                    aborted = true;
            auto issue_s = [&](int t, int j) -> bool {
                TileBars& b = ctl->tb[t];
                if (!mbar_wait(&b.k_full, j & 1, abort_flag, a.status, tmo, site(2, 1, t, j))) return false;
                tc_fence_after();
                const uint32_t sq = smem_u32(smem + C::q_off(t));
                const uint32_t sk = smem_u32(smem + C::k_off(t));
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kHalfBytes + (kk & 3) * 32;
                    mma_ss(tmem + C::s_col(t), sdesc_sw128(sq + off, 16, 1024),
                           sdesc_sw128(sk + off, 16, 1024), kIdS, kk > 0 ? 1u : 0u);
                }
                if constexpr (kPartial) {
                    const int pat = pats[t * C::kMaxChunks + j] & 7;
                    if (pat) {
                        const uint32_t sb = smem_u32(smem + C::kBias);
                        mma_ss(tmem + C::s_col(t), sdesc_plain(sb, 0, 128),
                               sdesc_plain(sb + pat * C::kBiasTile, 0, 128), kIdS, 1u);
                    }
                }
                issued = true;
                tc_commit(&b.k_empty);
                if (!((a.debug_flags & 1) && j == 0 && t == 0)) tc_commit(&b.s_full);
                return true;
            };
            auto issue_pv = [&](int t, int j) -> bool {
                TileBars& b = ctl->tb[t];
                if (!mbar_wait(&b.p_full, j & 1, abort_flag, a.status, tmo, site(2, 3, t, j))) return false;
                tc_fence_after();
                if (!mbar_wait(&b.v_full, j & 1, abort_flag, a.status, tmo, site(2, 2, t, j))) return false;
                tc_fence_after();
                const uint32_t sv = smem_u32(smem + C::v_off(t));
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tmem + C::o_col(t), tmem + C::s_col(t) + kk * 8,
                           sdesc_sw128(sv + kk * 2048, C::kHalfBytes, 1024), kIdO,
                           (j > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&b.v_empty);
                return true;
            };
            for (int t = 0; t < 2 && !aborted; ++t)
                if (n[t] > 0 && !issue_s(t, 0)) aborted = true;
            for (int j = 0; j < nmax && !aborted; ++j) {
                for (int t = 0; t < 2 && !aborted; ++t) {
                    if (j >= n[t]) continue;
                    if (!issue_pv(t, j)) { aborted = true; break; }
                    if (j + 1 < n[t]) {
                        if (!issue_s(t, j + 1)) { aborted = true; break; }
                    } else {
                        tc_commit(&ctl->tb[t].o_full);
                    }
                }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int t = warp >> 2;                     // tile of this warpgroup
        const int m = threadIdx.x & 127;             // query row = TMEM lane
        const int n_t = t ? n1 : n0;
        TileBars& b = ctl->tb[t];
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + C::s_col(t);
        const uint32_t tO = tmem + lane_off + C::o_col(t);
        const float c2 = a.scale_log2;
        float m_run = -INFINITY;
        bool has_key = false;  // a step with keys for this row has been seen
        float2 l2 = make_float2(0.f, 0.f), l2b = make_float2(0.f, 0.f);
        bool ok = true;
        for (int it = 0; it < n_t; ++it) {
            const bool got = mbar_wait(&b.s_full, it & 1, abort_flag, a.status, tmo, site(3, 4, t, it));
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
            uint32_t s[128];
            tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(s + 0));
            tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(s + 32));
            tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(s + 64));
            tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(s + 96));
#pragma unroll
            for (int c = 0; c < 4; ++c)
                tmem_wait_ld_tie(*reinterpret_cast<uint32_t(*)[32]>(s + 32 * c));
            // Row max in four chains: key slots with lw in {0,1}, {2,3} (the key box's
            // left half, lw < 4) and {4,5}, {6,7} (its right half).
            float ha0 = fmaxf(__uint_as_float(s[0]), __uint_as_float(s[1]));
            float ha1 = fmaxf(__uint_as_float(s[2]), __uint_as_float(s[3]));
            float hb0 = fmaxf(__uint_as_float(s[4]), __uint_as_float(s[5]));
            float hb1 = fmaxf(__uint_as_float(s[6]), __uint_as_float(s[7]));
#pragma unroll
            for (int j = 8; j < 128; j += 8) {
                ha0 = fmax3(ha0, __uint_as_float(s[j]), __uint_as_float(s[j + 1]));
                ha1 = fmax3(ha1, __uint_as_float(s[j + 2]), __uint_as_float(s[j + 3]));
                hb0 = fmax3(hb0, __uint_as_float(s[j + 4]), __uint_as_float(s[j + 5]));
                hb1 = fmax3(hb1, __uint_as_float(s[j + 6]), __uint_as_float(s[j + 7]));
            }
            const float mx_a = fmaxf(ha0, ha1), mx_b = fmaxf(hb0, hb1);
            // kQuad: the key halves this query row attends to in this box (its query
            // half is the lw of row m). The masked logits never enter any arithmetic:
            // the max is taken over the kept halves and masked numerators are zeroed.
            bool keep_a = true, keep_b = true;
            if constexpr (kQuad) {
                const uint32_t qp = pats[t * C::kMaxChunks + it] >> 3;
                const uint32_t mine = (qp >> ((m & 4) ? 2 : 0)) & 3u;
                keep_a = mine & 1u;
                keep_b = mine & 2u;
            }
            const bool step_has = keep_a || keep_b;
            const float m_new =
                (keep_a && keep_b ? fmaxf(mx_a, mx_b) : (keep_a ? mx_a : mx_b)) * c2;
            // Lazy rescale: move the reference max only when it grows by > 2^8. The
            // first step with a key sets it (it == 0 unless rows skip steps).
            const bool first = !has_key && step_has;
            const bool rescale = has_key && step_has && m_new > m_run + 8.0f;
            const float alpha = rescale ? ex2_approx(m_run - m_new) : 1.0f;
            if (first || rescale) m_run = m_new;
            has_key = has_key || step_has;
            l2.x *= alpha;
            l2.y *= alpha;
            l2b.x *= alpha;
            l2b.y *= alpha;
            const float2 cc = make_float2(c2, c2);
            // no key yet (kQuad): every numerator of this step is zeroed below
            const float m_ref = has_key ? m_run : 0.0f;
            const float2 nm = make_float2(-m_ref, -m_ref);
            const bool masked = kQuad && __any_sync(0xffffffffu, !(keep_a && keep_b));
            uint32_t pk[64];
            auto exp_pairs = [&](auto mask_tag) {
                constexpr bool kMask = decltype(mask_tag)::value;
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    const float2 x = __ffma2_rn(
                        make_float2(__uint_as_float(s[2 * j]), __uint_as_float(s[2 * j + 1])), cc,
                        nm);
                    // alternate pairs between the MUFU unit and the FMA-pipe polynomial
                    float2 pp = (kPolyEvery > 0 && j % kPolyEvery == 0)
                                    ? exp2_poly2(x)
                                    : make_float2(ex2_approx(x.x), ex2_approx(x.y));
                    // pair j holds key slots 2j, 2j+1: lw of both is < 4 iff (j & 2) == 0
                    if constexpr (kMask)
                        if (!((j & 2) ? keep_b : keep_a)) pp = make_float2(0.0f, 0.0f);
                    if (j & 1) l2b = __fadd2_rn(l2b, pp); else l2 = __fadd2_rn(l2, pp);
                    pk[j] = pack_bf16x2(pp.x, pp.y);
                }
            };
            if (masked)
                exp_pairs(std::true_type{});
            else
                exp_pairs(std::false_type{});
            // P over S columns [0, 64): every S value is already in registers
            tmem_st32(tS + 0, *reinterpret_cast<const uint32_t(*)[32]>(pk + 0));
            tmem_st32(tS + 32, *reinterpret_cast<const uint32_t(*)[32]>(pk + 32));
            // tcgen05.ld/st are warp-collective (.sync.aligned): the branch must be
            // taken by the whole warp, each row scaling by its own alpha (1 if its
            // reference max did not move).
            if (__any_sync(0xffffffffu, rescale)) {
                // O holds the chunks before this one (their PV completed before S was
                // signalled, and the next PV waits for P): rescale it to the new max.
#pragma unroll 1
                for (int g = 0; g < D / 32; ++g) {
                    uint32_t o[32];
                    tmem_ld32(tO + g * 32, o);
                    tmem_wait_ld_tie(o);
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                    tmem_st32(tO + g * 32, o);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&b.p_full);
        }
        const float l_run = (l2.x + l2.y) + (l2b.x + l2b.y);
        if (ok && n_t > 0) {
            const bool got = mbar_wait(&b.o_full, 0, abort_flag, a.status, tmo, site(3, 5, t, 0));
            ok = __all_sync(0xffffffffu, got);
        }
        const bool all_ok = bar_red_and(1 + t, 128, ok);
        const int64_t row = 2 * static_cast<int64_t>(blockIdx.x) + t;
        if (row < a.rows) {
            const int64_t bh = row / a.Nq;
            int q_t, q_h, q_w;
            chunk_origin(a.q_skip + static_cast<int>(row % a.Nq), a.NH, a.NW, q_t, q_h, q_w);
            const int lt = m >> 5, lh = (m >> 3) & 3, lw = m & 7;
            // a query slot of a partial edge chunk past the grid has no output (the TMA
            // store clips those rows; the direct stores below skip them)
            const bool q_exists = q_t + lt < a.T && q_h + lh < a.H && q_w + lw < a.W;
            const int64_t tok =
                (static_cast<int64_t>(q_t + lt) * a.H + (q_h + lh)) * a.W + q_w + lw;
            if (all_ok && n_t > 0 && a.out_f32) {
                // fp32 output (a partial result that is merged later): each thread
                // stores its own row, 128-bit stores; tcgen05.ld is warp-collective,
                // so every lane loads and only existing query slots store
                tc_fence_after();
                // a row without any key (kQuad: its query chunk kept none of the box's
                // keys): zeros, lse = -inf
                const float inv_l = has_key ? 1.0f / l_run : 0.0f;
                float4* dst = reinterpret_cast<float4*>(a.out_f32 + (bh * a.N + tok) * D);
#pragma unroll
                for (int g = 0; g < D / 32; ++g) {
                    uint32_t o[32];
                    tmem_ld32(tO + g * 32, o);
                    tmem_wait_ld_tie(o);
                    if (q_exists) {
#pragma unroll
                        for (int c4 = 0; c4 < 8; ++c4)
                            dst[g * 8 + c4] = make_float4(__uint_as_float(o[c4 * 4 + 0]) * inv_l,
                                                          __uint_as_float(o[c4 * 4 + 1]) * inv_l,
                                                          __uint_as_float(o[c4 * 4 + 2]) * inv_l,
                                                          __uint_as_float(o[c4 * 4 + 3]) * inv_l);
                    }
                }
                if (a.lse && q_exists)
                    a.lse[bh * a.N + tok] =
                        has_key ? (m_run + __log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
            } else if (all_ok && n_t > 0) {
                tc_fence_after();
                const float inv_l = has_key ? 1.0f / l_run : 0.0f;
                uint8_t* stage = smem + C::q_off(t);  // Q of this tile is dead once O is final
#pragma unroll
                for (int g = 0; g < D / 32; ++g) {
                    uint32_t o[32];
                    tmem_ld32(tO + g * 32, o);
                    tmem_wait_ld_tie(o);
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
                named_bar_sync(1 + t, 128);
                if (m == 0) {
#pragma unroll
                    for (int h = 0; h < C::kHalves; ++h)
                        tma_store_5d(&tm_o, smem_u32(stage) + h * C::kHalfBytes, h * 64, q_w, q_h,
                                     q_t, static_cast<int>(bh));
                    tma_store_commit_and_wait_all();
                }
                if (a.lse && q_exists)
                    a.lse[bh * a.N + tok] =
                        has_key ? (m_run + __log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
            } else if (all_ok && q_exists) {
                // empty (or rejected) row: zeros, lse = -inf
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                if (a.out_f32) {
                    uint4* dst = reinterpret_cast<uint4*>(a.out_f32 + (bh * a.N + tok) * D);
#pragma unroll
                    for (int j = 0; j < D / 4; ++j) dst[j] = z;
                } else {
                    uint4* dst = reinterpret_cast<uint4*>(a.out + (bh * a.N + tok) * D);
#pragma unroll
                    for (int j = 0; j < D / 8; ++j) dst[j] = z;
                }
                if (a.lse) a.lse[bh * a.N + tok] = -INFINITY;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    // After an abort (the flag no longer changes here, whichever role gave up and
    // whenever), the copies and products still in flight land before the CTA's
    // shared memory and TMEM are released.
    if (*abort_flag) {
        if (warp == C::kTmaWarp && lane == 0) {
            for (int t = 0; t < 2; ++t) {
                if ((t ? n1 : n0) == 0) continue;
                drain_wait(&ctl->tb[t].q_full, 0, tmo);
                if (nk[t] > 0) drain_wait(&ctl->tb[t].k_full, (nk[t] - 1) & 1, tmo);
                if (nvv[t] > 0) drain_wait(&ctl->tb[t].v_full, (nvv[t] - 1) & 1, tmo);
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
    if ((a.debug_flags & 2) && threadIdx.x == 0) atomicAdd(a.status + 8, 1u);
}

}  // namespace

// 5-D tiled map over a [BH][T][H][W][D] bf16 tensor with a (64,8,4,4,1) box and
// 128-byte swizzle: one box is 128 tokens of one chunk x 64 channels.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver entry point is looked up once per process (a function-local static
// is initialised exactly once, also under concurrent first calls).
static EncodeTiledFn get_encode_fn() {
    static const EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(p);
        return static_cast<EncodeTiledFn>(nullptr);
    }();
    return fn;
}

bool make_chunk_map(CUtensorMap* tm, const void* base, const Dims& g, int box_t) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[5] = {(cuuint64_t)g.d, (cuuint64_t)g.W, (cuuint64_t)g.H,
                                (cuuint64_t)g.T, (cuuint64_t)g.BH};
    const cuuint64_t strides[4] = {(cuuint64_t)g.d * 2, (cuuint64_t)g.W * g.d * 2,
                                   (cuuint64_t)g.H * g.W * g.d * 2,
                                   (cuuint64_t)g.T * g.H * g.W * g.d * 2};
    const cuuint32_t box[5] = {64, kChunkW, kChunkH, (cuuint32_t)box_t, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

namespace {

template <int D, bool kPartial, bool kQuad>
cudaError_t launch_fwd_dp(const Dims& g, const CUtensorMap& mq, const CUtensorMap& mk,
                          const CUtensorMap& mv, const CUtensorMap& mo, const FwdArgs& args,
                          cudaStream_t st) {
    using C = AttnCfg<D>;
    static std::atomic<uint64_t> attr_done{0};
    const cudaError_t e =
        raise_smem_limit(bsa_fwd_kernel<D, kPartial, kQuad>, C::kSmemBytes, attr_done);
    if (e != cudaSuccess) return e;
    const unsigned grid = static_cast<unsigned>((g.rows + 1) / 2);
    bsa_fwd_kernel<D, kPartial, kQuad>
        <<<grid, C::kThreads, C::kSmemBytes, st>>>(mq, mk, mv, mo, args);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_fwd_d(const Dims& g, const CUtensorMap& mq, const CUtensorMap& mk,
                         const CUtensorMap& mv, const CUtensorMap& mo, const FwdArgs& args,
                         cudaStream_t st) {
    const bool partial = g.T % kChunkT || g.H % kChunkH || g.W % kChunkW;
    if (args.quad)
        return partial ? launch_fwd_dp<D, true, true>(g, mq, mk, mv, mo, args, st)
                       : launch_fwd_dp<D, false, true>(g, mq, mk, mv, mo, args, st);
    return partial ? launch_fwd_dp<D, true, false>(g, mq, mk, mv, mo, args, st)
                   : launch_fwd_dp<D, false, false>(g, mq, mk, mv, mo, args, st);
}

__global__ void exp2_selftest_kernel(const float* __restrict__ x, float* __restrict__ y_poly,
                                     float* __restrict__ y_mufu, int64_t n) {
    const int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 2;
    if (i + 1 < n) {
        const float2 v = make_float2(x[i], x[i + 1]);
        const float2 p = exp2_poly2(v);
        y_poly[i] = p.x;
        y_poly[i + 1] = p.y;
        y_mufu[i] = ex2_approx(v.x);
        y_mufu[i + 1] = ex2_approx(v.y);
    }
}

}  // namespace

cudaError_t launch_exp2_selftest(const float* x, float* y_poly, float* y_mufu, int64_t n,
                                 cudaStream_t st) {
    const int64_t pairs = n / 2;
    if (pairs == 0) return cudaSuccess;
    exp2_selftest_kernel<<<(unsigned)((pairs + 255) / 256), 256, 0, st>>>(x, y_poly, y_mufu, n);
    return cudaGetLastError();
}

cudaError_t launch_forward(const Dims& g, const void* q, const void* k, const void* v,
                           const int32_t* row_ptr, const int32_t* col_idx, int64_t col_cap,
                           void* out, float* lse, uint32_t* status, uint64_t timeout_ns,
                           int debug_flags, cudaStream_t st, float* out_f32,
                           const uint8_t* quad) {
    if (!out && !out_f32) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv, mo;
    // with an fp32 output the bf16 output map is never used (built over q)
    if (!make_chunk_map(&mq, q, g) || !make_chunk_map(&mk, k, g) || !make_chunk_map(&mv, v, g) ||
        !make_chunk_map(&mo, out_f32 ? q : out, g))
        return cudaErrorInvalidValue;
    FwdArgs args;
    args.row_ptr = row_ptr;
    args.col_idx = col_idx;
    args.col_cap = col_cap;
    args.out = static_cast<__nv_bfloat16*>(out);
    args.out_f32 = out_f32;
    args.quad = quad;
    args.lse = lse;
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
    args.rows = g.rows;
    args.scale_log2 = g.scale * 1.4426950408889634f;
    args.timeout_ns = timeout_ns;
    args.debug_flags = debug_flags;
    return g.d == 128 ? launch_fwd_d<128>(g, mq, mk, mv, mo, args, st)
                      : launch_fwd_d<64>(g, mq, mk, mv, mo, args, st);
}

}  // namespace bsa
