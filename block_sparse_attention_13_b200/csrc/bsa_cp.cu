// Context parallelism for block sparse attention ("LongCat-Video Technical
// Report", section "Block Sparse Attention (BSA)", ring block sparse
// attention; "LongCat-Video Technical Report #", section "开源实现": LSE and
// output correction kernels). The sequence is split across ranks along the
// latent frames; every rank selects among the pooled keys of all ranks, then
// attends over each rank's K/V shard in turn and folds the partial results
// together with their log-sum-exps. This file holds the two device steps that
// are specific to that: slicing the selection to one shard's key chunks, and
// merging a partial result into the running one. For the backward of the ring
// it holds the fp32 accumulation of the per-shard gradient contributions and
// their final rounding to bf16.
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

// The same merge with an fp32 accumulator and an fp32 partial result (4
// elements per thread): the partial outputs are rounded only once, when the
// merged result is finally converted to bf16.
template <int D>
__global__ void __launch_bounds__(256) lse_merge_f32_kernel(float* __restrict__ out,
                                                            float* __restrict__ lse,
                                                            const float* __restrict__ part,
                                                            const float* __restrict__ lse_part,
                                                            int64_t tokens) {
    constexpr int VPT = D / 4;
    const int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const bool valid = v < tokens * VPT;
    const int64_t tok = valid ? v / VPT : 0;
    const float a = valid ? lse[tok] : 0.f, b = valid ? lse_part[tok] : -INFINITY;
    // every lane of a token (VPT consecutive lanes of one warp) has read lse[tok]
    // before its first lane overwrites it
    __syncwarp();
    if (!valid || b == -INFINITY) return;
    float4* po = reinterpret_cast<float4*>(out) + v;
    const float4 y = reinterpret_cast<const float4*>(part)[v];
    float l;
    float4 r;
    if (a == -INFINITY) {
        r = y;
        l = b;
    } else {
        const float m = fmaxf(a, b);
        const float ea = __expf(a - m), eb = __expf(b - m);
        const float inv = 1.0f / (ea + eb);
        const float wa = ea * inv, wb = eb * inv;
        l = m + __logf(ea + eb);
        const float4 x = *po;
        r = make_float4(fmaf(wa, x.x, wb * y.x), fmaf(wa, x.y, wb * y.y), fmaf(wa, x.z, wb * y.z),
                        fmaf(wa, x.w, wb * y.w));
    }
    *po = r;
    if (v % VPT == 0) lse[tok] = l;
}

// acc (fp32) = part (bf16), or acc += part; 8 elements per thread and step.
__global__ void __launch_bounds__(256) grad_accumulate_kernel(const uint4* __restrict__ part,
                                                              float4* __restrict__ acc,
                                                              int64_t n8, int overwrite) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
         i += (int64_t)gridDim.x * blockDim.x) {
        const uint4 pv = part[i];
        const uint32_t w[4] = {pv.x, pv.y, pv.z, pv.w};
        float f[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {  // bf16 -> fp32 is exact: the bits move up 16 places
            f[2 * e] = __uint_as_float(w[e] << 16);
            f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
        }
        float4 a0 = make_float4(f[0], f[1], f[2], f[3]), a1 = make_float4(f[4], f[5], f[6], f[7]);
        if (!overwrite) {
            const float4 b0 = acc[2 * i], b1 = acc[2 * i + 1];
            a0 = make_float4(b0.x + a0.x, b0.y + a0.y, b0.z + a0.z, b0.w + a0.w);
            a1 = make_float4(b1.x + a1.x, b1.y + a1.y, b1.z + a1.z, b1.w + a1.w);
        }
        acc[2 * i] = a0;
        acc[2 * i + 1] = a1;
    }
}

// out (bf16, round to nearest even) = acc (fp32).
__global__ void __launch_bounds__(256) grad_finalize_kernel(const float4* __restrict__ acc,
                                                            uint4* __restrict__ out, int64_t n8) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float4 a0 = acc[2 * i], a1 = acc[2 * i + 1];
        out[i] = make_uint4(pack_bf16x2(a0.x, a0.y), pack_bf16x2(a0.z, a0.w),
                            pack_bf16x2(a1.x, a1.y), pack_bf16x2(a1.z, a1.w));
    }
}

// Elementwise passes over HBM: at most 8 resident 256-thread blocks per SM,
// grid-striding over the rest.
unsigned stream_blocks(int64_t n8) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (n8 + 255) / 256, cap = static_cast<int64_t>(sms) * 8;
    return static_cast<unsigned>(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

cudaError_t launch_grad_accumulate(int64_t n, const void* part, float* acc, int overwrite,
                                   cudaStream_t st) {
    const int64_t n8 = n / 8;
    if (n8 == 0) return cudaSuccess;
    grad_accumulate_kernel<<<stream_blocks(n8), 256, 0, st>>>(
        static_cast<const uint4*>(part), reinterpret_cast<float4*>(acc), n8, overwrite);
    return cudaGetLastError();
}

cudaError_t launch_grad_finalize(int64_t n, const float* acc, void* out, cudaStream_t st) {
    const int64_t n8 = n / 8;
    if (n8 == 0) return cudaSuccess;
    grad_finalize_kernel<<<stream_blocks(n8), 256, 0, st>>>(reinterpret_cast<const float4*>(acc),
                                                            static_cast<uint4*>(out), n8);
    return cudaGetLastError();
}

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

cudaError_t launch_lse_merge_f32(const Dims& g, float* out, float* lse, const float* out_part,
                                 const float* lse_part, cudaStream_t st) {
    const int64_t tokens = g.BH * g.N;
    const int64_t vecs = tokens * (g.d / 4);
    const unsigned blocks = static_cast<unsigned>((vecs + 255) / 256);
    if (g.d == 128)
        lse_merge_f32_kernel<128><<<blocks, 256, 0, st>>>(out, lse, out_part, lse_part, tokens);
    else
        lse_merge_f32_kernel<64><<<blocks, 256, 0, st>>>(out, lse, out_part, lse_part, tokens);
    return cudaGetLastError();
}

}  // namespace bsa
