// append.cuh -- one decode step's cache update for HCA: the newest token of every sequence
// goes into the raw window, and a block that it completes is pooled into the compressed
// cache (official blog "ERNIE 5.5 Flash Base . ERNIE", section 2.1: every 128 tokens are
// compressed into a single cached entry; attention reads the entries plus a window of
// recent raw tokens).
//
// The window is a ring: position p of sequence b lives in slot p % W.  Attention over the
// window does not depend on the order of its keys, so decode reads the ring as it is
// (HCA_WINDOW_RING), with no copy to restore the oldest-first order.
//
// The pooling is the compressor's softmax-weighted mean (weights w, one per position,
// shared by K, V and every KV head), computed online so that no raw token has to stay
// resident after it leaves the window: per (sequence, KV head) a running state holds the
// block's largest weight m, the sum s = sum exp(w_i - m) and the fp32 accumulators
// sum exp(w_i - m) k_i (and v_i).  A new token with weight w moves the reference to
// m' = max(m, w), rescales the state by exp(m - m') and adds exp(w - m') k.  When the
// token completes a block, the entry acc / s is rounded to bf16 once and written, and
// the state returns to all zeros -- which is also the state of an empty block (s = 0).
#pragma once

#include "common.cuh"

namespace hca {

constexpr int kAppendThreads = 128;
constexpr int kAppendHeader = 4;            // state floats before the accumulators: m, s, 2 unused

struct AppendParams {
    const __nv_bfloat16* k_new;   // [B, Hkv, d]
    const __nv_bfloat16* v_new;   // [B, Hkv, dv]
    const float* w;               // [B] or null (weight 0)
    const int* seqlens;           // [B], length including the new token
    __nv_bfloat16* kw;            // [B, W, Hkv, d] ring
    __nv_bfloat16* vw;            // [B, W, Hkv, dv] ring
    __nv_bfloat16* kc;            // [B, Nmax, Hkv, d] or pool [P, ps, Hkv, d]
    __nv_bfloat16* vc;
    const int* page_table;        // [B, max_pages] or null
    float* state;                 // [B, Hkv, kAppendHeader + d + dv]
    int B, Hkv, d, dv, blk, W, Nmax, page_size, max_pages, num_pages;
};

// Channels c .. c+3 of one tensor (K or V), already loaded: ring write, state update and,
// when the block completes, the entry.
__device__ __forceinline__ void append_channels(uint2 x, float4 t, __nv_bfloat16* ring, float* acc,
                                                __nv_bfloat16* entry, int c, float a, float e, float inv_s,
                                                bool complete) {
    *reinterpret_cast<uint2*>(ring + c) = x;
    t.x = fmaf(e, bf16lo(x.x), t.x * a);
    t.y = fmaf(e, bf16hi(x.x), t.y * a);
    t.z = fmaf(e, bf16lo(x.y), t.z * a);
    t.w = fmaf(e, bf16hi(x.y), t.w * a);
    if (complete) {
        if (entry)
            *reinterpret_cast<uint2*>(entry + c) =
                make_uint2(pack_bf16x2(t.x * inv_s, t.y * inv_s), pack_bf16x2(t.z * inv_s, t.w * inv_s));
        t = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    *reinterpret_cast<float4*>(acc + c) = t;
}

// One CTA per (sequence, KV head); thread i owns channels 4i .. 4i+3 of K and of V (d, dv <=
// 512).  Every load is issued before any result is needed -- the new token, the pooling
// state, the weight and the length do not depend on one another -- so a call costs one
// memory round trip after launch.
__global__ void __launch_bounds__(kAppendThreads) append_kernel(const AppendParams p) {
    const int u = blockIdx.x;
    const int b = u / p.Hkv, g = u - b * p.Hkv;
    const int c = 4 * threadIdx.x;
    const bool hk = c < p.d, hv = c < p.dv;
    float* st = p.state + (size_t)u * (kAppendHeader + p.d + p.dv);
    float* acc_k = st + kAppendHeader;
    float* acc_v = st + kAppendHeader + p.d;
    const int L = __ldg(p.seqlens + b);
    const float w = p.w ? __ldg(p.w + b) : 0.f;
    const float2 ms = *reinterpret_cast<const float2*>(st);
    const uint2 xk = hk ? *reinterpret_cast<const uint2*>(p.k_new + (size_t)u * p.d + c) : make_uint2(0u, 0u);
    const uint2 xv = hv ? *reinterpret_cast<const uint2*>(p.v_new + (size_t)u * p.dv + c) : make_uint2(0u, 0u);
    const float4 tk = hk ? *reinterpret_cast<const float4*>(acc_k + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 tv = hv ? *reinterpret_cast<const float4*>(acc_v + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    if (L < 1) {
        if (threadIdx.x == 0) record_error(HCA_ERR_DEVICE_INPUT);
        return;
    }
    const long long pos = (long long)L - 1;
    const int slot = (int)(pos % p.W);
    const float m_old = ms.x, s_old = ms.y;
    const bool empty = !(s_old > 0.f);
    const float m_new = empty ? w : fmaxf(m_old, w);
    const float a = empty ? 0.f : expf(m_old - m_new);
    const float e = expf(w - m_new);
    const float s_new = fmaf(s_old, a, e);
    const bool complete = (pos + 1) % p.blk == 0;
    // destination of a completed block's entry (null: out of the cache, reported)
    __nv_bfloat16 *ek = nullptr, *ev = nullptr;
    if (complete) {
        const long long j = pos / p.blk;
        long long row = -1;
        if (p.page_table) {
            const long long pi = j / p.page_size;
            if (pi < p.max_pages) {
                const int pg = __ldg(p.page_table + (size_t)b * p.max_pages + pi);
                if (pg >= 0 && pg < p.num_pages) row = (long long)pg * p.page_size + j % p.page_size;
            }
        } else if (j < p.Nmax) {
            row = (long long)b * p.Nmax + j;
        }
        if (row >= 0) {
            ek = p.kc + ((size_t)row * p.Hkv + g) * p.d;
            ev = p.vc + ((size_t)row * p.Hkv + g) * p.dv;
        } else if (threadIdx.x == 0) {
            record_error(HCA_ERR_DEVICE_INPUT);
        }
    }
    const float inv_s = 1.f / s_new;
    const size_t ring_row = (size_t)b * p.W + slot;
    if (hk) append_channels(xk, tk, p.kw + (ring_row * p.Hkv + g) * p.d, acc_k, ek, c, a, e, inv_s, complete);
    if (hv) append_channels(xv, tv, p.vw + (ring_row * p.Hkv + g) * p.dv, acc_v, ev, c, a, e, inv_s, complete);
    __syncthreads();      // every thread has read m and s
    if (threadIdx.x == 0) *reinterpret_cast<float2*>(st) = complete ? make_float2(0.f, 0.f) : make_float2(m_new, s_new);
}

}  // namespace hca
