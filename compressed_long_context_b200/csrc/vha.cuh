// vha.cuh -- Virtual Head Attention applied to an attention output (official blog "ERNIE 5.5
// Flash Base . ERNIE", section 2.1, and the Zhidx article, section "1. Latent-Gated Sparse
// Attention": a lightweight cross-head low-rank mixing with an identity skip after the
// attention).  Reading: per token and per channel c, o'[:, c] = (I + U V^T) o[:, c] over the
// token's Hq heads, with U, V of shape [Hq, r].
//
// In place on out [n, Hq, dv] (bf16 or fp32).  Work item = (token, slice of 64 bf16 or 32
// fp32 channels), one warp each: lane l holds one 32-bit word of every head row (two bf16
// channels, or one fp32 channel) in registers, so the reduction over heads, t = V^T o
// (r values per channel), runs inside the lane with no shared-memory traffic for the data;
// o + U t is written back over the same words.  U and V sit in shared memory, padded with
// zeros to a power-of-two rank RP >= 4 (zero terms add nothing), and are read as
// broadcasts.  Both products use the two-wide fp32 FMA, each lane of which rounds like
// fmaf.  The output is read and written once: HBM-bound when the FMA work per byte is small
// (2 Hq r FMAs per channel; at Hq 64 the rank-8 mixing is about 1000 FMAs per 2-byte
// channel).  The fp32 path also prefetches each warp's next item into L2.
#pragma once

#include "common.cuh"

namespace hca {

constexpr int kVhaThreads = 128;    // 4 warps, each its own work item
constexpr int kVhaCh = 64;          // dv must be a multiple of this
constexpr int kVhaMaxHeads = 64;
constexpr int kVhaMaxRank = 32;

struct VhaParams {
    void* out;               // [n, Hq, dv]
    const float* U;          // [Hq, r]
    const float* V;          // [Hq, r]
    long long n;
    int Hq, dv, r;
};

// Factor copies in shared memory: [Hq][RP] each, and for bf16 every value twice, so that one
// 16-byte broadcast load yields the (u, u) pairs the two-channel FMA takes.
__host__ __device__ inline int vha_smem_bytes(int Hq, int rp, bool f32) { return 2 * Hq * rp * (f32 ? 1 : 2) * 4; }

// 16-byte shared-memory load kept where it is written: the factors are loop-invariant, and a
// compiler that hoists their Hq * RP values out of the work-item loop spills.
__device__ __forceinline__ float4 vha_lds4(uint32_t addr) {
    float4 f;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(f.x), "=f"(f.y), "=f"(f.z), "=f"(f.w) : "r"(addr));
    return f;
}

template <bool F32, int RP>
__global__ void __launch_bounds__(kVhaThreads) vha_kernel(const VhaParams p) {
    // RP * kS a multiple of 4: whole 16-byte loads per head row, and v_s (after Hq rows of
    // u_s) 16-byte aligned for any Hq
    static_assert(RP >= 4 && RP % 4 == 0, "rank padded to a multiple of 4");
    constexpr int kS = F32 ? 1 : 2;                  // stored copies of each factor value
    constexpr int kQ = RP * kS / 4;                  // float4 loads per head row of a factor
    constexpr int kT = F32 ? RP / 2 : RP;            // float2 accumulators of t per lane
    extern __shared__ __align__(16) float vsm[];
    float* u_s = vsm;
    float* v_s = vsm + p.Hq * RP * kS;
    for (int i = threadIdx.x; i < p.Hq * RP; i += kVhaThreads) {
        const int h = i / RP, k = i - h * RP;
        const float u = k < p.r ? __ldg(p.U + h * p.r + k) : 0.f;
        const float v = k < p.r ? __ldg(p.V + h * p.r + k) : 0.f;
#pragma unroll
        for (int e = 0; e < kS; ++e) {
            u_s[i * kS + e] = u;
            v_s[i * kS + e] = v;
        }
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int slices = p.dv / (F32 ? 32 : 64);
    const long long items = p.n * slices;
    const long long stride = (long long)gridDim.x * (kVhaThreads / 32);
    const int row_words = F32 ? p.dv : p.dv / 2;     // 32-bit words per head row
    uint32_t* out = static_cast<uint32_t*>(p.out);
    for (long long item = (long long)blockIdx.x * (kVhaThreads / 32) + (threadIdx.x >> 5); item < items;
         item += stride) {
        // factor bases re-derived per item (opaque to the compiler), so that their per-head
        // addresses are not hoisted out of the loop and kept live in registers
        uint32_t vb = smem_u32(v_s), ub = smem_u32(u_s);
        asm volatile("" : "+r"(vb), "+r"(ub));
        const long long tok = item / slices;
        uint32_t* row = out + tok * p.Hq * row_words + (item - tok * slices) * 32 + lane;
        // fp32: the warp's next item into L2 (lane l: head rows l and l + 32, 128 bytes each),
        // so its DRAM latency overlaps this item's arithmetic without holding registers.  An
        // fp32 item is half as many channels per byte as a bf16 one; for bf16 the prefetch
        // measured slower (its items are already long enough to hide the loads).
        if (F32 && item + stride < items) {
            const long long nt = (item + stride) / slices;
            const uint32_t* nrow = out + nt * p.Hq * row_words + (item + stride - nt * slices) * 32;
#pragma unroll
            for (int h = lane; h < kVhaMaxHeads; h += 32)
                if (h < p.Hq) asm volatile("prefetch.global.L2 [%0];" :: "l"(nrow + (size_t)h * row_words));
        }
        uint32_t x[kVhaMaxHeads];
        {
            const uint32_t* src = row;
#pragma unroll
            for (int h = 0; h < kVhaMaxHeads; ++h) {
                if (h < p.Hq) x[h] = *src;
                src += row_words;
                asm volatile("" : "+l"(src));      // one live address: the chain is not unrolled into 64

            }
        }
        // t = V^T o.  bf16: t[k] = (t_k at channel 2l, at 2l+1); fp32: t[j] = (t_2j, t_2j+1).
        float2 t[kT];
#pragma unroll
        for (int j = 0; j < kT; ++j) t[j] = make_float2(0.f, 0.f);
#pragma unroll
        for (int h = 0; h < kVhaMaxHeads; ++h) {
            if (h < p.Hq) {
                const uint32_t vh = vb + h * RP * kS * 4;
                const float2 xx = F32 ? make_float2(__uint_as_float(x[h]), __uint_as_float(x[h]))
                                      : make_float2(__uint_as_float(x[h] << 16), __uint_as_float(x[h] & 0xffff0000u));
#pragma unroll
                for (int q = 0; q < kQ; ++q) {
                    const float4 f = vha_lds4(vh + 16 * q);
                    t[2 * q] = __ffma2_rn(make_float2(f.x, f.y), xx, t[2 * q]);
                    t[2 * q + 1] = __ffma2_rn(make_float2(f.z, f.w), xx, t[2 * q + 1]);
                }
            }
        }
        // o' = o + U t, over the words just read
        uint32_t* dst = row;
#pragma unroll
        for (int h = 0; h < kVhaMaxHeads; ++h) {
            if (h < p.Hq) {
                const uint32_t uh = ub + h * RP * kS * 4;
                if constexpr (F32) {
                    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                    for (int q = 0; q < kQ; ++q) {
                        const float4 f = vha_lds4(uh + 16 * q);
                        acc = __ffma2_rn(make_float2(f.x, f.y), t[2 * q], acc);
                        acc = __ffma2_rn(make_float2(f.z, f.w), t[2 * q + 1], acc);
                    }
                    *dst = __float_as_uint(__uint_as_float(x[h]) + (acc.x + acc.y));
                } else {
                    float2 y = make_float2(__uint_as_float(x[h] << 16), __uint_as_float(x[h] & 0xffff0000u));
#pragma unroll
                    for (int q = 0; q < kQ; ++q) {
                        const float4 f = vha_lds4(uh + 16 * q);
                        y = __ffma2_rn(make_float2(f.x, f.y), t[2 * q], y);
                        y = __ffma2_rn(make_float2(f.z, f.w), t[2 * q + 1], y);
                    }
                    *dst = pack_bf16x2(y.x, y.y);
                }
            }
            dst += row_words;
            asm volatile("" : "+l"(dst));
        }
    }
}

}  // namespace hca
