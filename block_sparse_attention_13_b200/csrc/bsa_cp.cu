// Context parallelism for block sparse attention ("LongCat-Video Technical
// Report", section "Block Sparse Attention (BSA)", ring block sparse
// attention; "LongCat-Video Technical Report #", section "开源实现": LSE and
// output correction kernels). The sequence is split across ranks along the
// latent frames; every rank selects among the pooled keys of all ranks, then
// attends over each rank's K/V shard in turn and folds the partial results
// together with their log-sum-exps. This file holds the two device steps that
// are specific to that: slicing the selection to one shard's key chunks, and
// merging a partial result into the running one.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bsa_internal.cuh"
#include "bsa_ptx.cuh"

namespace bsa {

namespace {

// One warp per row: number of entries with lo <= c < hi.
__global__ void __launch_bounds__(256) csr_slice_count_kernel(const int32_t* __restrict__ row_ptr,
                                                              const int32_t* __restrict__ col_idx,
                                                              int64_t rows, int64_t col_cap,
                                                              int lo, int hi,
                                                              int32_t* __restrict__ counts,
                                                              uint32_t* status) {
    const int lane = threadIdx.x & 31;
    const int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (w >= rows) return;
    const int64_t beg = row_ptr[w], end = row_ptr[w + 1];
    int n = 0;
    if (beg >= 0 && end >= beg && end <= col_cap) {
        for (int64_t e = beg + lane; e < end; e += 32) {
            const int c = col_idx[e];
            n += (c >= lo && c < hi);
        }
    } else if (lane == 0) {
        atomicOr(status, kStatusBadIndex);
    }
    n = __reduce_add_sync(0xffffffffu, n);
    if (lane == 0) counts[w] = n;
}

// One warp per row: the kept entries, in their row order, re-indexed.
__global__ void __launch_bounds__(256) csr_slice_emit_kernel(const int32_t* __restrict__ row_ptr,
                                                             const int32_t* __restrict__ col_idx,
                                                             int64_t rows, int64_t col_cap,
                                                             int lo, int hi,
                                                             const int32_t* __restrict__ out_row_ptr,
                                                             int32_t* __restrict__ out_col_idx,
                                                             int64_t out_cap, uint32_t* status) {
    const int lane = threadIdx.x & 31;
    const int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (w >= rows) return;
    const int64_t beg = row_ptr[w], end = row_ptr[w + 1];
    if (!(beg >= 0 && end >= beg && end <= col_cap)) return;  // reported by the count pass
    if (out_row_ptr[w + 1] > out_cap) {
        if (lane == 0) atomicOr(status, kStatusCapacity);
        return;
    }
    int64_t run = out_row_ptr[w];
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int64_t e0 = beg; e0 < end; e0 += 32) {
        const int64_t e = e0 + lane;
        const int c = e < end ? col_idx[e] : lo - 1;
        const bool keep = c >= lo && c < hi;
        const uint32_t kb = __ballot_sync(0xffffffffu, keep);
        if (keep) out_col_idx[run + __popc(kb & lt_mask)] = c - lo;
        run += __popc(kb);
    }
}

// out = merge(out, part) by log-sum-exp for every token; one thread per 8
// channels of a token. A token whose part has lse = -inf keeps its value; one
// whose accumulator has lse = -inf takes the part.
template <int D>
__global__ void __launch_bounds__(256) lse_merge_kernel(__nv_bfloat16* __restrict__ out,
                                                        float* __restrict__ lse,
                                                        const __nv_bfloat16* __restrict__ part,
                                                        const float* __restrict__ lse_part,
                                                        int64_t tokens) {
    constexpr int VPT = D / 8;
    const int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const bool valid = v < tokens * VPT;
    const int64_t tok = valid ? v / VPT : 0;
    const float a = valid ? lse[tok] : 0.f, b = valid ? lse_part[tok] : -INFINITY;
    // every lane of a token (VPT consecutive lanes of one warp) has read lse[tok]
    // before its first lane overwrites it
    __syncwarp();
    if (!valid || b == -INFINITY) return;
    uint4* po = reinterpret_cast<uint4*>(out) + v;
    const uint4 pb = reinterpret_cast<const uint4*>(part)[v];
    float l;
    uint4 r;
    if (a == -INFINITY) {
        r = pb;
        l = b;
    } else {
        const float m = fmaxf(a, b);
        const float ea = __expf(a - m), eb = __expf(b - m);
        const float inv = 1.0f / (ea + eb);
        const float wa = ea * inv, wb = eb * inv;
        l = m + __logf(ea + eb);
        const uint4 pa = *po;
        const uint32_t av[4] = {pa.x, pa.y, pa.z, pa.w}, bv[4] = {pb.x, pb.y, pb.z, pb.w};
        uint32_t rv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&av[e]));
            const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bv[e]));
            rv[e] = pack_bf16x2(fmaf(wa, x.x, wb * y.x), fmaf(wa, x.y, wb * y.y));
        }
        r = make_uint4(rv[0], rv[1], rv[2], rv[3]);
    }
    *po = r;
    if (v % VPT == 0) lse[tok] = l;
}

}  // namespace

cudaError_t launch_csr_slice(int64_t rows, const int32_t* row_ptr, const int32_t* col_idx,
                             int64_t col_cap, int lo, int hi, int32_t* counts, int32_t* out_row_ptr,
                             int32_t* out_col_idx, int64_t out_cap, uint32_t* status,
                             cudaStream_t st) {
    const unsigned blocks = static_cast<unsigned>((rows + 7) / 8);
    csr_slice_count_kernel<<<blocks, 256, 0, st>>>(row_ptr, col_idx, rows, col_cap, lo, hi, counts,
                                                   status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if ((e = launch_scan_counts(counts, rows, out_row_ptr, st)) != cudaSuccess) return e;
    csr_slice_emit_kernel<<<blocks, 256, 0, st>>>(row_ptr, col_idx, rows, col_cap, lo, hi,
                                                  out_row_ptr, out_col_idx, out_cap, status);
    return cudaGetLastError();
}

cudaError_t launch_lse_merge(const Dims& g, void* out, float* lse, const void* out_part,
                             const float* lse_part, cudaStream_t st) {
    const int64_t tokens = g.BH * g.N;
    const int64_t vecs = tokens * (g.d / 8);
    const unsigned blocks = static_cast<unsigned>((vecs + 255) / 256);
    auto* o = static_cast<__nv_bfloat16*>(out);
    const auto* p = static_cast<const __nv_bfloat16*>(out_part);
    if (g.d == 128)
        lse_merge_kernel<128><<<blocks, 256, 0, st>>>(o, lse, p, lse_part, tokens);
    else
        lse_merge_kernel<64><<<blocks, 256, 0, st>>>(o, lse, p, lse_part, tokens);
    return cudaGetLastError();
}

}  // namespace bsa
