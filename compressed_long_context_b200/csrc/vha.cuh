// vha.cuh -- Virtual Head Attention applied to an attention output (official blog "ERNIE 5.5
// Flash Base . ERNIE", section 2.1, and the Zhidx article, section "1. Latent-Gated Sparse
// Attention": a lightweight cross-head low-rank mixing with an identity skip after the
// attention).  Reading: per token and per channel c, o'[:, c] = (I + U V^T) o[:, c] over the
// token's Hq heads, with U, V of shape [Hq, r].
//
// In place on out [n, Hq, dv] (bf16 or fp32).  One CTA per (token, 64-channel slice): the
// slice's Hq x 64 values go to shared memory with 16-byte loads, t = V^T o (r x 64) is
// reduced over the heads, and o + U t is written back.  The kernel reads and writes the
// output once: it is bound by HBM bandwidth.
#pragma once

#include "common.cuh"

namespace hca {

constexpr int kVhaThreads = 256;
constexpr int kVhaCh = 64;          // channels per CTA
constexpr int kVhaMaxHeads = 64;
constexpr int kVhaMaxRank = 32;

struct VhaParams {
    void* out;               // [n, Hq, dv]
    const float* U;          // [Hq, r]
    const float* V;          // [Hq, r]
    long long n;
    int Hq, dv, r;
};

template <bool F32>
__global__ void __launch_bounds__(kVhaThreads) vha_kernel(const VhaParams p) {
    __shared__ __align__(16) float o_s[kVhaMaxHeads * kVhaCh];
    __shared__ float t_s[kVhaMaxRank * kVhaCh];
    __shared__ float u_s[kVhaMaxHeads * kVhaMaxRank];
    __shared__ float v_s[kVhaMaxHeads * kVhaMaxRank];
    const int slices = p.dv / kVhaCh;
    const long long tok = blockIdx.x / slices;
    const int c0 = (int)(blockIdx.x - tok * slices) * kVhaCh;
    const int tid = threadIdx.x;
    const int hr = p.Hq * p.r;
    for (int i = tid; i < hr; i += kVhaThreads) {
        u_s[i] = __ldg(p.U + i);
        v_s[i] = __ldg(p.V + i);
    }
    // the slice: head h, channels c0 .. c0+63, 16 bytes per load
    const size_t base = (size_t)tok * p.Hq * p.dv + c0;
    constexpr int vec = F32 ? 4 : 8;                  // channels per 16-byte load
    constexpr int per_row = kVhaCh / vec;
    for (int i = tid; i < p.Hq * per_row; i += kVhaThreads) {
        const int h = i / per_row, c = (i - h * per_row) * vec;
        if constexpr (F32) {
            const float4 x = *reinterpret_cast<const float4*>(static_cast<const float*>(p.out) + base +
                                                              (size_t)h * p.dv + c);
            *reinterpret_cast<float4*>(o_s + h * kVhaCh + c) = x;
        } else {
            const uint4 x = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.out) + base +
                                                            (size_t)h * p.dv + c);
            float* d = o_s + h * kVhaCh + c;
            d[0] = bf16lo(x.x); d[1] = bf16hi(x.x); d[2] = bf16lo(x.y); d[3] = bf16hi(x.y);
            d[4] = bf16lo(x.z); d[5] = bf16hi(x.z); d[6] = bf16lo(x.w); d[7] = bf16hi(x.w);
        }
    }
    __syncthreads();
    // t[k][c] = sum_h V[h][k] o[h][c]
    for (int i = tid; i < p.r * kVhaCh; i += kVhaThreads) {
        const int k = i / kVhaCh, c = i - k * kVhaCh;
        float acc = 0.f;
        for (int h = 0; h < p.Hq; ++h) acc = fmaf(v_s[h * p.r + k], o_s[h * kVhaCh + c], acc);
        t_s[i] = acc;
    }
    __syncthreads();
    // o'[h][c] = o[h][c] + sum_k U[h][k] t[k][c], written back in the output's type
    for (int i = tid; i < p.Hq * per_row; i += kVhaThreads) {
        const int h = i / per_row, c = (i - h * per_row) * vec;
        float y[vec];
#pragma unroll
        for (int e = 0; e < vec; ++e) y[e] = o_s[h * kVhaCh + c + e];
        for (int k = 0; k < p.r; ++k) {
            const float u = u_s[h * p.r + k];
#pragma unroll
            for (int e = 0; e < vec; ++e) y[e] = fmaf(u, t_s[k * kVhaCh + c + e], y[e]);
        }
        if constexpr (F32) {
            *reinterpret_cast<float4*>(static_cast<float*>(p.out) + base + (size_t)h * p.dv + c) =
                make_float4(y[0], y[1], y[2], y[3]);
        } else {
            *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + base + (size_t)h * p.dv + c) =
                make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                           pack_bf16x2(y[6], y[7]));
        }
    }
}

}  // namespace hca
