// prefill.cuh -- HCA prefill on tcgen05 tensor cores (sm_100a).
//
// Every query row (token t, head h) attends, in one online softmax, to the compressed
// entries j < n_c(t) and then to the raw window t-W+1 .. t (official blog "ERNIE 5.5
// Flash Base . ERNIE", section 2.1; Zhidx article, section "1. Latent-Gated Sparse
// Attention").  The two segments are two runs of key tiles through the same (m, l, O)
// state, with a per-row mask on each tile.
//
// This single-CTA kernel serves 64-dim heads (512-dim heads run on the SM pair of
// prefill_pair.cuh, which also takes PrefillParams and the tile helpers from here).
//
// Tiling.  The 128 MMA rows of a tile are (token, head) pairs of one KV group: 128 / G
// tokens x G heads (G = Hq / Hkv), so all rows of a tile share their keys.  S (two
// 128-column buffers), P and the 64-column O of a row tile all fit one SM's tensor memory.
//
// Per work item (row tile), warp-specialised, persistent over a heavy-first schedule:
//   warp 0 (1 thread)  TMA: Q tile (d/64 slabs), then K and V tiles as 64-channel slabs
//                      (128 keys each, 128-byte swizzle) through a ring of 16 KB slots;
//   warp 1 (1 thread)  tcgen05.mma: S = Q K^T into TMEM (double-buffered), then
//                      O += P V with P read from TMEM (written over its S buffer);
//   warps 2-5          softmax, thread = row: mask, running max with lazy rescaling
//                      (only when the max grows by more than 2^8), P in bf16 back to
//                      TMEM; epilogue O / l (+ LSE) to global memory.
#pragma once

#include "common.cuh"

namespace hca {

constexpr int kPfThreads = 192;
constexpr int kPfRows = 128;
constexpr float kPfRescale = 8.0f;   // log2 units
constexpr uint32_t kPfSlab = 128 * 128;

template <int D>
struct PfCfg {
    static_assert(D == 64, "prefill_kernel serves 64-dim heads; 512-dim heads use prefill_pair_kernel");
    static constexpr int kSlabs = D / 64;                 // Q / K slabs per row
    static constexpr int kDVC = D;                        // value columns
    static constexpr int kVSlabs = kDVC / 64;
    static constexpr int kRing = 8;
    static constexpr uint32_t kSmQ = 0;
    static constexpr uint32_t kSmRing = kSmQ + kSlabs * kPfSlab;
    static constexpr uint32_t kSmBar = kSmRing + kRing * kPfSlab;
    static constexpr int kNumBars = 2 * kRing + 10;
    static constexpr uint32_t kSmMisc = kSmBar + kNumBars * 8;
    static constexpr uint32_t kSmem = kSmMisc + 64 + 1024;
    static_assert(kSmem <= 232448, "prefill shared memory exceeds the 227 KB per-block limit");
    static_assert(kSmRing % 1024 == 0 && kSmBar % 8 == 0, "operand tiles 1024-aligned, barriers 8-aligned");
    static constexpr uint32_t kTmS = 0;       // 2 x 128 columns
    static constexpr uint32_t kTmO = 256;     // kDVC columns (after the two S buffers)
};

struct PrefillParams {
    void* out;          // [B, T, Hq, dv] bf16 or fp32
    float* lse;         // [B, Hq, T] or null
    int B, T, Hq, Hkv, G, tpt, blk, W, Nc, ntile_t, flags;
    long long items;
    float scale_log2;
};

struct PfItem {
    int b, g, t0, tlast;
    int nc_hi, ncomp, nct, wlo, nwin, nwt;
};

__device__ __forceinline__ int pf_visible(int t, int W, int blk) {
    const int a = t - W + 1;
    return a > 0 ? a / blk : 0;
}

template <int D>
__device__ __forceinline__ PfItem pf_item(const PrefillParams& p, long long i) {
    PfItem it;
    long long r = i;
    it.g = (int)(r % p.Hkv);
    r /= p.Hkv;
    it.b = (int)(r % p.B);
    r /= p.B;
    const int tt = p.ntile_t - 1 - (int)r;        // heavy (late) token tiles first
    it.t0 = tt * p.tpt;
    it.tlast = min(it.t0 + p.tpt, p.T) - 1;
    it.nc_hi = pf_visible(it.tlast, p.W, p.blk);
    it.ncomp = it.nc_hi;
    it.nct = (it.ncomp + 127) / 128;
    it.wlo = max(0, it.t0 - p.W + 1);
    it.nwin = it.tlast - it.wlo + 1;
    it.nwt = (it.nwin + 127) / 128;
    return it;
}

// keys in tile j of an item, and the MMA N (multiple of 16)
__device__ __forceinline__ int pf_tile_keys(const PfItem& it, int j) {
    return j < it.nct ? min(128, it.ncomp - 128 * j) : min(128, it.nwin - 128 * (j - it.nct));
}

template <int D>
__global__ void __launch_bounds__(kPfThreads, 1)
prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tm_q,
               const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
               const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_vc) {
    using C = PfCfg<D>;
    extern __shared__ uint8_t dsmem[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::kSmBar);
    uint64_t* full = bars;
    uint64_t* empty = bars + C::kRing;
    uint64_t* q_full = bars + 2 * C::kRing;
    uint64_t* q_empty = q_full + 1;
    uint64_t* s_full = q_full + 2;     // [2]
    uint64_t* p_full = q_full + 4;     // [2]
    uint64_t* pv_done = q_full + 6;    // [2]
    uint64_t* o_full = q_full + 8;
    uint64_t* o_empty = q_full + 9;
    int* misc = reinterpret_cast<int*>(sm + C::kSmMisc);
    volatile int* abort_flag = misc;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int i = 0; i < C::kRing; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 4);
            mbar_init(&pv_done[i], 1);
        }
        mbar_init(o_full, 1);
        mbar_init(o_empty, 4);
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_kc);
        prefetch_tmap(&tm_vc);
    }
    if (warp == 1) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const long long stride = gridDim.x;

    if (warp == 0) {
        // ===================================================== TMA producer
        if (lane == 0) {
            uint32_t ring = 0;
            int item_n = 0;
            bool ok = true;
            auto load_slab = [&](const CUtensorMap* m, int c0, int g, int row, int b) -> bool {
                const uint32_t st = ring % C::kRing;
                if (!mbar_wait(&empty[st], ((ring / C::kRing) & 1) ^ 1, abort_flag)) return false;
                mbar_arrive_expect_tx(&full[st], kPfSlab);
                tma_load_4d(sm + C::kSmRing + st * kPfSlab, m, &full[st], c0, g, row, b);
                ++ring;
                return true;
            };
            auto load_k = [&](const PfItem& it, int j) -> bool {
                const bool comp = j < it.nct;
                const int row = comp ? 128 * j : it.wlo + 128 * (j - it.nct);
                for (int s = 0; s < C::kSlabs; ++s)
                    if (!load_slab(comp ? &tm_kc : &tm_k, 64 * s, it.g, row, it.b)) return false;
                return true;
            };
            auto load_v = [&](const PfItem& it, int j) -> bool {
                const bool comp = j < it.nct;
                const int row = comp ? 128 * j : it.wlo + 128 * (j - it.nct);
                for (int s = 0; s < C::kVSlabs; ++s)
                    if (!load_slab(comp ? &tm_vc : &tm_v, 64 * s, it.g, row, it.b)) return false;
                return true;
            };
            for (long long i = blockIdx.x; ok && i < p.items; i += stride, ++item_n) {
                const PfItem it = pf_item<D>(p, i);
                // Q tile: rows (token, head) = (t0 + r / G, g*G + r % G)
                if (!mbar_wait(q_empty, (item_n & 1) ^ 1, abort_flag)) break;
                mbar_arrive_expect_tx(q_full, C::kSlabs * kPfSlab);
                for (int s = 0; s < C::kSlabs; ++s)
                    tma_load_4d(sm + C::kSmQ + s * kPfSlab, &tm_q, q_full, 64 * s, it.g * p.G, it.t0, it.b);
                const int nt = it.nct + it.nwt;
                ok = load_k(it, 0);
                for (int j = 0; ok && j < nt; ++j) {
                    if (j + 1 < nt) ok = load_k(it, j + 1);
                    if (ok) ok = load_v(it, j);
                }
            }
        }
    } else if (warp == 1) {
        // ===================================================== MMA issuer
        uint32_t ring = 0;
        int n = 0;            // global tile counter (S/P buffer parity)
        int item_n = 0;
        bool ok = true;
        const uint32_t q_base = smem_u32(sm + C::kSmQ);
        for (long long i = blockIdx.x; ok && i < p.items; i += stride, ++item_n) {
            const PfItem it = pf_item<D>(p, i);
            const int nt = it.nct + it.nwt;
            if (!warp_wait(q_full, item_n & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            auto issue_qk = [&](int j, int nn) -> bool {
                const int N = (pf_tile_keys(it, j) + 15) & ~15;
                const uint32_t id = idesc_bf16(128, N, 0, 0);
                const uint32_t dst = tmem + C::kTmS + 128 * (nn & 1);
                for (int s = 0; s < C::kSlabs; ++s) {
                    const uint32_t st = ring % C::kRing;
                    if (!warp_wait(&full[st], (ring / C::kRing) & 1, abort_flag)) return false;
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t kb = smem_u32(sm + C::kSmRing + st * kPfSlab);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t ad = smem_desc_sw128(q_base + s * kPfSlab + kk * 32, 16, 1024);
                            const uint64_t bd = smem_desc_sw128(kb + kk * 32, 16, 1024);
                            mma_ss(dst, ad, bd, id, (s | kk) ? 1u : 0u);
                        }
                        mma_commit(&empty[st]);
                    }
                    __syncwarp();
                    ++ring;
                }
                if (lane == 0) {
                    mma_commit(&s_full[nn & 1]);
                    if (j == nt - 1) mma_commit(q_empty);
                }
                __syncwarp();
                return true;
            };
            auto issue_pv = [&](int j, int nn) -> bool {
                const int ksteps = (pf_tile_keys(it, j) + 15) >> 4;
                const uint32_t id = idesc_bf16(128, 64, 0, 1);
                const uint32_t pa = tmem + C::kTmS + 128 * (nn & 1);
                if (!warp_wait(&p_full[nn & 1], (nn >> 1) & 1, abort_flag)) return false;
                if (j == 0 && !warp_wait(o_empty, (item_n & 1) ^ 1, abort_flag)) return false;
                tc_fence_after();
                for (int v = 0; v < C::kVSlabs; ++v) {
                    const uint32_t st = ring % C::kRing;
                    if (!warp_wait(&full[st], (ring / C::kRing) & 1, abort_flag)) return false;
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t vb = smem_u32(sm + C::kSmRing + st * kPfSlab);
                        for (int kk = 0; kk < ksteps; ++kk) {
                            const uint64_t bd = smem_desc_sw128(vb + kk * 2048, 8192, 1024);
                            mma_ts(tmem + C::kTmO + 64 * v, pa + kk * 8, bd, id, (j == 0 && kk == 0) ? 0u : 1u);
                        }
                        mma_commit(&empty[st]);
                    }
                    __syncwarp();
                    ++ring;
                }
                if (lane == 0) {
                    mma_commit(&pv_done[nn & 1]);
                    if (j == nt - 1) mma_commit(o_full);
                }
                __syncwarp();
                return true;
            };
            if (!issue_qk(0, n)) { ok = false; break; }
            for (int j = 0; j < nt; ++j) {
                if (j + 1 < nt && !issue_qk(j + 1, n + j + 1)) { ok = false; break; }
                if (!issue_pv(j, n + j)) { ok = false; break; }
            }
            n += nt;
        }
    } else {
        // ===================================================== softmax / epilogue (warps 2-5)
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;                 // row of the tile
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        int n = 0, item_n = 0;
        bool ok = true;
        for (long long i = blockIdx.x; ok && i < p.items; i += stride, ++item_n) {
            const PfItem it = pf_item<D>(p, i);
            const int nt = it.nct + it.nwt;
            const int tok = it.t0 + r / p.G;
            const bool row_live = tok < p.T;
            const int t = row_live ? tok : p.T - 1;
            const int head = it.g * p.G + (r % p.G);
            const int nc_t = pf_visible(t, p.W, p.blk);
            float m = -INFINITY, l = 0.f;
            for (int j = 0; j < nt; ++j, ++n) {
                const int sb = n & 1;
                const int nk = pf_tile_keys(it, j);
                const int ncol = (nk + 15) & ~15;
                // valid columns of this row: [lo, hi)
                int lo, hi;
                if (j < it.nct) {
                    lo = 0;
                    hi = min(nk, nc_t - 128 * j);
                } else {
                    const int u0 = it.wlo + 128 * (j - it.nct);
                    lo = max(0, t - p.W + 1 - u0);
                    hi = min(nk, t - u0 + 1);
                }
                if (!warp_wait(&s_full[sb], (n >> 1) & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                float s[128];
                const uint32_t sa = tmem + lane_off + C::kTmS + 128 * sb;
#pragma unroll
                for (int c = 0; c < 128; c += 16)
                    if (c < ncol) tmem_ld16(sa + c, s + c);
                tmem_wait_ld();
                float tmax = -INFINITY;
#pragma unroll
                for (int c = 0; c < 128; ++c) {
                    const bool v = c >= lo && c < hi;
                    s[c] = v ? s[c] * p.scale_log2 : -INFINITY;
                    tmax = fmaxf(tmax, s[c]);
                }
                // lazy max: a row moves its reference only when the new max exceeds it by
                // 2^8 (or on its first visible key).  tcgen05.ld/st are warp-collective, so the
                // O rescale runs for the whole warp whenever any of its rows needs it, with
                // factor 1 for the others.
                const bool rescale = m != -INFINITY && tmax > m + kPfRescale;
                float al = 1.f;
                if (rescale) {
                    al = ex2(m - tmax);
                    l *= al;
                }
                if (rescale || (m == -INFINITY && tmax > -INFINITY)) m = tmax;
                if (__any_sync(0xffffffffu, rescale)) {
                    // O, once the previous PV has landed
                    if (!warp_wait(&pv_done[(n - 1) & 1], ((n - 1) >> 1) & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < C::kDVC; c += 16) {
                        float o[16];
                        uint32_t w[16];
                        tmem_ld16(tmem + lane_off + C::kTmO + c, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 16; ++k) w[k] = __float_as_uint(o[k] * al);
                        tmem_st16(tmem + lane_off + C::kTmO + c, w);
                    }
                    tmem_wait_st();
                }
                const float mref = m == -INFINITY ? 0.f : m;
                float rs = 0.f;
#pragma unroll
                for (int c = 0; c < 128; c += 32) {
                    if (c < ncol) {
                        uint32_t pk[16];
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const float a = ex2(s[c + 2 * k] - mref);
                            const float b2 = ex2(s[c + 2 * k + 1] - mref);
                            rs += a + b2;
                            pk[k] = pack_bf16x2(a, b2);
                        }
                        tmem_st16(sa + c / 2, pk);
                    }
                }
                l += rs;
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[sb]);
            }
            if (!ok) break;
            // ---- epilogue: out = O / l, lse = ln(sum exp(logits))
            if (!warp_wait(o_full, item_n & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const float inv = 1.f / l;
            const size_t orow = (((size_t)it.b * p.T + tok) * p.Hq + head) * (size_t)C::kDVC;
#pragma unroll 1
            for (int c = 0; c < C::kDVC; c += 16) {
                float o[16];
                tmem_ld16(tmem + lane_off + C::kTmO + c, o);
                tmem_wait_ld();
                if (row_live) {
                    if (p.flags & HCA_OUT_F32) {
                        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow + c);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            dst[k] = make_float4(o[4 * k] * inv, o[4 * k + 1] * inv, o[4 * k + 2] * inv,
                                                 o[4 * k + 3] * inv);
                    } else {
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + orow + c);
#pragma unroll
                        for (int k = 0; k < 2; ++k)
                            dst[k] = make_uint4(pack_bf16x2(o[8 * k] * inv, o[8 * k + 1] * inv),
                                                pack_bf16x2(o[8 * k + 2] * inv, o[8 * k + 3] * inv),
                                                pack_bf16x2(o[8 * k + 4] * inv, o[8 * k + 5] * inv),
                                                pack_bf16x2(o[8 * k + 6] * inv, o[8 * k + 7] * inv));
                    }
                }
            }
            if (row_live && p.lse)
                p.lse[((size_t)it.b * p.Hq + head) * p.T + tok] = (m + log2f(l)) * 0.6931471805599453f;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_empty);
        }
    }

    __syncwarp();      // every role reconverges its warp before the CTA-wide barrier
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace hca
