// compress.cuh -- HCA block compression (official blog "ERNIE 5.5 Flash Base . ERNIE",
// section 2.1: every 128 tokens are compressed into a single cached entry).
//
// Entry j of sequence b, KV head g:  Kc = sum_i alpha_i K[b, blk*j+i, g, :],
// alpha = softmax over the block of the per-position weights w[b, blk*j+i]
// (all-zero / absent weights give the mean); Vc likewise with the same alpha.
//
// The kernel is a pure HBM stream: one CTA per (b, j, g) entry reads blk raw rows of
// K and of V with 16-byte coalesced loads (evict-first), accumulates in fp32 and
// writes two bf16 rows.  The block softmax of the weights is one warp with shuffle
// reductions.  No shared-memory staging is needed: every raw byte is read once.
#pragma once

#include "common.cuh"

namespace hca {

constexpr int kCompressThreads = 256;
constexpr int kCompressUnroll = 8;

// Weighted sum over `blk` rows of one tensor with D channels.  Each thread owns 8
// consecutive channels of rows r0, r0 + R, ...; the R partial sums are then added
// through shared memory and rounded once to bf16.
template <int D>
__device__ __forceinline__ void pool_rows(const __nv_bfloat16* __restrict__ src, int64_t row_stride,
                                          const float* __restrict__ alpha, int blk, float* __restrict__ red,
                                          __nv_bfloat16* __restrict__ dst) {
    constexpr int TPR = D / 8;                   // threads per row (16 bytes each)
    constexpr int R = kCompressThreads / TPR;    // rows in flight per pass
    const int tid = threadIdx.x;
    const int c0 = (tid % TPR) * 8;
    const int r0 = tid / TPR;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;

    for (int r = r0; r < blk; r += R * kCompressUnroll) {
        uint4 x[kCompressUnroll];
#pragma unroll
        for (int u = 0; u < kCompressUnroll; ++u) {
            const int rr = r + u * R;
            if (rr < blk) x[u] = __ldcs(reinterpret_cast<const uint4*>(src + rr * row_stride + c0));
        }
#pragma unroll
        for (int u = 0; u < kCompressUnroll; ++u) {
            const int rr = r + u * R;
            if (rr < blk) {
                const float a = alpha[rr];
                acc[0] = fmaf(a, bf16lo(x[u].x), acc[0]);
                acc[1] = fmaf(a, bf16hi(x[u].x), acc[1]);
                acc[2] = fmaf(a, bf16lo(x[u].y), acc[2]);
                acc[3] = fmaf(a, bf16hi(x[u].y), acc[3]);
                acc[4] = fmaf(a, bf16lo(x[u].z), acc[4]);
                acc[5] = fmaf(a, bf16hi(x[u].z), acc[5]);
                acc[6] = fmaf(a, bf16lo(x[u].w), acc[6]);
                acc[7] = fmaf(a, bf16hi(x[u].w), acc[7]);
            }
        }
    }
    float4* o = reinterpret_cast<float4*>(red + r0 * D + c0);
    o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    __syncthreads();
    for (int c2 = tid; c2 < D / 2; c2 += kCompressThreads) {
        float s0 = 0.f, s1 = 0.f;
#pragma unroll 4
        for (int r = 0; r < R; ++r) {
            const float2 p = *reinterpret_cast<const float2*>(red + r * D + 2 * c2);
            s0 += p.x;
            s1 += p.y;
        }
        reinterpret_cast<uint32_t*>(dst)[c2] = pack_bf16x2(s0, s1);
    }
    __syncthreads();
}

template <int DK, int DV>
__global__ void __launch_bounds__(kCompressThreads)
compress_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                const float* __restrict__ w, __nv_bfloat16* __restrict__ kc, __nv_bfloat16* __restrict__ vc,
                int T, int Hkv, int blk, int Nc) {
    __shared__ float alpha[128];
    __shared__ __align__(16) float red[kCompressThreads * 8];

    const int e = blockIdx.x;                 // entry index, KV head fastest
    const int g = e % Hkv;
    const int bj = e / Hkv;
    const int j = bj % Nc;
    const int b = bj / Nc;
    const int64_t pos0 = (int64_t)b * T + (int64_t)blk * j;

    if (threadIdx.x < 32) {
        // alpha = softmax of the block's weights (max subtracted), one warp
        const int lane = threadIdx.x;
        float wv[4];
        float m = -INFINITY;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int idx = lane + 32 * i;
            wv[i] = idx < blk ? (w ? w[pos0 + idx] : 0.f) : -INFINITY;
            m = fmaxf(m, wv[i]);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            wv[i] = (lane + 32 * i) < blk ? expf(wv[i] - m) : 0.f;
            s += wv[i];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        const float inv = 1.f / s;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (lane + 32 * i < blk) alpha[lane + 32 * i] = wv[i] * inv;
    }
    __syncthreads();

    const int64_t out_row = ((int64_t)b * Nc + j) * Hkv + g;
    pool_rows<DK>(k + (pos0 * Hkv + g) * DK, (int64_t)Hkv * DK, alpha, blk, red, kc + out_row * DK);
    pool_rows<DV>(v + (pos0 * Hkv + g) * DV, (int64_t)Hkv * DV, alpha, blk, red, vc + out_row * DV);
}

}  // namespace hca
