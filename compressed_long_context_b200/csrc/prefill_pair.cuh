// prefill_pair.cuh -- HCA prefill for 512-dim heads on a pair of SMs (a thread-block
// cluster of two CTAs).
//
// What is computed is the same as prefill.cuh (official blog "ERNIE 5.5 Flash Base .
// ERNIE", section 2.1; Zhidx article, section "1. Latent-Gated Sparse Attention"): every
// query row (token t, head h) attends, in one online softmax, to the compressed entries
// j < n_c(t) and to the raw window t-W+1 .. t.
//
// Why a pair.  A row tile of 128 (token, head) rows with 512-dim values needs a 128 x 512
// fp32 accumulator: all 512 columns of one SM's tensor memory.  The logits of a 256-key
// tile need 256 more.  So the work is split by stage, not by value columns:
//   S-CTA (cluster rank 0): Q resident in shared memory, K tiles streamed by TMA,
//       S = Q K^T with N = 256 keys into a double-buffered S (2 x 256 TMEM columns), softmax
//       (thread = row), and P (bf16) stored straight into the O-CTA's shared memory in the
//       non-swizzled K-major layout the tensor core reads (8 keys of row r at
//       (key / 8) * 2048 + r * 16, so the 32 rows of a warp fill 512 contiguous bytes per
//       store instruction: remote stores need that to stream), together with the per-row
//       rescale factors (and, after the last tile, the row sums);
//   O-CTA (cluster rank 1): V tiles streamed by TMA, O += P V with N = 256 value columns
//       (two MMAs per 16 keys cover the 512 columns), rescale of O rows when the S-CTA moved
//       a row's reference maximum, and the epilogue out = O / l.
// Every MMA is M = 128, N = 256 (or the 16-rounded key count of a short tile): the tcgen05
// issue cost of one M = 128 MMA does not shrink with N, so narrow MMAs waste the pipe.
//
// Warps (224 threads, same kernel for both ranks):
//   S-CTA: 0 TMA (Q, K) | 1 MMA + TMEM | 2-5 softmax | 6 idle
//   O-CTA: 0 TMA (V)    | 1 MMA + TMEM | 2-5 rescale + epilogue | 6 forwards "P slot
//          consumed" to the S-CTA
//
// Tiles of one row tile (item): the compressed segment in tiles of 256 entries, then the
// raw window [wlo, tlast] in tiles of 256 tokens; per-row masks [lo, hi) as in prefill.cuh.
// Lazy rescaling: a row moves its reference maximum only when a tile's maximum exceeds it
// by 2^8, so the O-CTA rarely touches O between MMAs.
#pragma once

#include "common.cuh"
#include "prefill.cuh"

namespace hca {

constexpr int kPpThreads = 224;
constexpr int kPpKeys = 256;                     // keys per tile (MMA N of S)
constexpr int kPpD = 512;
constexpr int kPpRing = 3;                       // K units (S-CTA) / V units (O-CTA)
constexpr uint32_t kPpQSlab = 128 * 128;         // Q: 128 rows x 64 channels
constexpr uint32_t kPpUnit = 32768;              // K: 256 keys x 64 ch; V: 64 keys x 256 ch
constexpr uint32_t kPpVSub = 8192;               // V unit = 4 channel slabs of 64 keys x 64 ch
constexpr uint32_t kPpPBuf = 65536;              // P: 128 rows x 256 keys, 32 key chunks of 2 KB
constexpr uint32_t kPpHdrBytes = 1040;           // alpha[128], l[128], flag[4]
// shared-memory layout (offsets from a 1024-aligned base); the two ranks reuse offsets
constexpr uint32_t kPpSmQ = 0;                   // S-CTA: Q, 8 slabs (128 KB)
constexpr uint32_t kPpSmP = 0;                   // O-CTA: P, 2 buffers (128 KB)
constexpr uint32_t kPpSmRing = 131072;           // both: ring of 3 units (96 KB)
constexpr uint32_t kPpSmHdr = kPpSmRing + kPpRing * kPpUnit;     // O-CTA: 2 headers
constexpr uint32_t kPpSmBar = kPpSmHdr + 2 * kPpHdrBytes;
constexpr int kPpNumBars = 32;
constexpr uint32_t kPpSmMisc = kPpSmBar + kPpNumBars * 8;
constexpr uint32_t kPpSmem = kPpSmMisc + 64;
static_assert(kPpSmem <= 232448, "pair prefill shared memory exceeds the 227 KB per-block limit");
static_assert(kPpSmHdr % 16 == 0 && kPpSmBar % 8 == 0, "header 16-aligned, barriers 8-aligned");

// barrier indices (both ranks initialise all of them; each rank uses its own)
enum : int {
    kBarKFull = 0, kBarKEmpty = 3, kBarQFull = 6, kBarQEmpty = 7, kBarSFull = 8, kBarSEmpty = 10,
    kBarPEmpty = 12,                                           // S-CTA
    kBarVFull = 14, kBarVEmpty = 17, kBarPFull = 20, kBarCorr = 22, kBarPCons = 24, kBarOFull = 26,
    kBarOEmpty = 27,                                           // O-CTA
    kBarDrain = 28
};

struct PpItem {
    int b, g, t0, tlast;
    int ncomp, nct, wlo, nwin, nwt;
};

__device__ __forceinline__ PpItem pp_item(const PrefillParams& p, long long i) {
    PpItem it;
    it.g = (int)(i % p.Hkv);
    long long r = i / p.Hkv;
    it.b = (int)(r % p.B);
    r /= p.B;
    const int tt = p.ntile_t - 1 - (int)r;        // heavy (late) token tiles first
    it.t0 = tt * p.tpt;
    it.tlast = min(it.t0 + p.tpt, p.T) - 1;
    it.ncomp = pf_visible(it.tlast, p.W, p.blk);
    it.nct = (it.ncomp + kPpKeys - 1) / kPpKeys;
    it.wlo = max(0, it.t0 - p.W + 1);
    it.nwin = it.tlast - it.wlo + 1;
    it.nwt = (it.nwin + kPpKeys - 1) / kPpKeys;
    return it;
}

__device__ __forceinline__ int pp_tile_keys(const PpItem& it, int j) {
    return j < it.nct ? min(kPpKeys, it.ncomp - kPpKeys * j) : min(kPpKeys, it.nwin - kPpKeys * (j - it.nct));
}
__device__ __forceinline__ int pp_tile_row(const PpItem& it, int j) {
    return j < it.nct ? kPpKeys * j : it.wlo + kPpKeys * (j - it.nct);
}

// ------------------------------------------------------------------ cluster helpers

__device__ __forceinline__ uint32_t pp_cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// shared::cluster address of the same shared-memory offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t pp_mapa(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void pp_cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void pp_remote_arrive(uint32_t rbar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" :: "r"(rbar) : "memory");
}
__device__ __forceinline__ void pp_st_cluster_v4(uint32_t raddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" :: "r"(raddr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}
__device__ __forceinline__ void pp_st_cluster_u32(uint32_t raddr, uint32_t v) {
    asm volatile("st.shared::cluster.b32 [%0], %1;" :: "r"(raddr), "r"(v) : "memory");
}
__device__ __forceinline__ void pp_fence_proxy_async_cluster() {
    asm volatile("fence.proxy.async.shared::cluster;" ::: "memory");
}
// try_wait with acquire at cluster scope: for barriers the peer CTA arrives on
__device__ __forceinline__ bool pp_try_wait_cl(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool pp_wait_cl(uint64_t* bar, uint32_t parity, volatile int* abort) {
    if (pp_try_wait_cl(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (pp_try_wait_cl(bar, parity)) return true;
        if ((i & 63u) == 0) {
            if (*abort) return false;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                *abort = 1;
                record_error(HCA_ERR_TIMEOUT);
                return false;
            }
        }
    }
}
__device__ __forceinline__ bool pp_warp_wait_cl(uint64_t* bar, uint32_t parity, volatile int* abort) {
    const bool ok = pp_wait_cl(bar, parity, abort);
    return __all_sync(0xffffffffu, ok);
}
// Wait for a phase at exit, ignoring the abort flag (copies already issued still land);
// bounded by the same wall-clock limit.
__device__ __forceinline__ void pp_drain_wait(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            record_error(HCA_ERR_TIMEOUT);
            return;
        }
}

// Shared-memory matrix descriptor for the non-swizzled K-major layout: core matrices of
// 8 rows x 16 bytes (rows 16 bytes apart), `lbo` bytes between core matrices adjacent in K,
// `sbo` bytes between core matrices adjacent in M/N; swizzle field 0.
__device__ __forceinline__ uint64_t pp_desc_noswz(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;
    return d;
}

__device__ __forceinline__ uint32_t pp_ld_cluster_u32(uint32_t raddr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(raddr) : "memory");
    return v;
}

// Producer-side drain: wait until the last load issued into every slot of a ring has landed.
__device__ __forceinline__ void pp_drain_ring(uint64_t* full, uint32_t issued) {
    for (uint32_t st = 0; st < (uint32_t)kPpRing; ++st)
        if (issued > st) pp_drain_wait(&full[st], ((issued - 1 - st) / kPpRing) & 1);
}

__global__ void __launch_bounds__(kPpThreads, 1)
prefill_pair_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_vc) {
    extern __shared__ __align__(1024) uint8_t dsmem[];
    uint8_t* sm = dsmem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kPpSmBar);
    int* misc = reinterpret_cast<int*>(sm + kPpSmMisc);
    volatile int* abort_flag = misc;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = pp_cluster_rank();
    const bool s_cta = rank == 0;
    // the swizzled operand tiles need a 1024-byte aligned base; there is no room for slack
    const bool aligned = (smem_u32(dsmem) & 1023u) == 0;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        misc[2] = aligned ? 1 : 0;
        for (int i = 0; i < kPpRing; ++i) {
            mbar_init(&bars[kBarKFull + i], 1);
            mbar_init(&bars[kBarKEmpty + i], 1);
            mbar_init(&bars[kBarVFull + i], 1);
            mbar_init(&bars[kBarVEmpty + i], 1);
        }
        mbar_init(&bars[kBarQFull], 1);
        mbar_init(&bars[kBarQEmpty], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars[kBarSFull + i], 1);
            mbar_init(&bars[kBarSEmpty + i], 4);
            mbar_init(&bars[kBarPEmpty + i], 1);
            mbar_init(&bars[kBarPFull + i], 4);
            mbar_init(&bars[kBarCorr + i], 4);
            mbar_init(&bars[kBarPCons + i], 1);
        }
        mbar_init(&bars[kBarOFull], 1);
        mbar_init(&bars[kBarOEmpty], 4);
        mbar_init(&bars[kBarDrain], 1);
        fence_mbar_init();
        if (s_cta) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_kc);
        } else {
            prefetch_tmap(&tm_v);
            prefetch_tmap(&tm_vc);
        }
    }
    if (warp == 1) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    pp_cluster_sync();      // barriers of both CTAs are initialised before any remote arrive
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t peer_base = pp_mapa(smem_u32(sm), rank ^ 1u);
    const bool go = aligned && pp_ld_cluster_u32(peer_base + kPpSmMisc + 8) != 0;
    if (!go && threadIdx.x == 0) record_error(HCA_ERR_INTERNAL);
    const long long npairs = gridDim.x >> 1;
    const long long pair = blockIdx.x >> 1;

    if (s_cta && warp == 0) {
        // ===================================================== S-CTA: TMA of Q and K
        if (lane == 0 && go) {
            uint32_t kr = 0, qn = 0;
            bool ok = true;
            for (long long i = pair; ok && i < p.items; i += npairs) {
                const PpItem it = pp_item(p, i);
                if (!mbar_wait(&bars[kBarQEmpty], (qn & 1) ^ 1, abort_flag)) break;
                mbar_arrive_expect_tx(&bars[kBarQFull], 8 * kPpQSlab);
                for (int s = 0; s < 8; ++s)
                    tma_load_4d(sm + kPpSmQ + s * kPpQSlab, &tm_q, &bars[kBarQFull], 64 * s, it.g * p.G, it.t0, it.b);
                ++qn;
                const int nt = it.nct + it.nwt;
                for (int j = 0; ok && j < nt; ++j) {
                    const bool comp = j < it.nct;
                    const int row = pp_tile_row(it, j);
                    for (int s = 0; s < 8; ++s) {
                        const uint32_t st = kr % kPpRing;
                        if (!mbar_wait(&bars[kBarKEmpty + st], ((kr / kPpRing) & 1) ^ 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&bars[kBarKFull + st], kPpUnit);
                        tma_load_4d(sm + kPpSmRing + st * kPpUnit, comp ? &tm_kc : &tm_k, &bars[kBarKFull + st],
                                    64 * s, it.g, row, it.b);
                        ++kr;
                    }
                }
            }
            pp_drain_ring(&bars[kBarKFull], kr);
            if (qn) pp_drain_wait(&bars[kBarQFull], (qn - 1) & 1);
        }
    } else if (s_cta && warp == 1) {
        // ===================================================== S-CTA: S = Q K^T
        if (go) {
            uint32_t kr = 0;
            int n = 0, item_n = 0;
            bool ok = true;
            const uint32_t q_base = smem_u32(sm + kPpSmQ);
            for (long long i = pair; ok && i < p.items; i += npairs, ++item_n) {
                const PpItem it = pp_item(p, i);
                const int nt = it.nct + it.nwt;
                if (!warp_wait(&bars[kBarQFull], item_n & 1, abort_flag)) break;
                for (int j = 0; ok && j < nt; ++j, ++n) {
                    const int sb = n & 1;
                    if (!warp_wait(&bars[kBarSEmpty + sb], ((n >> 1) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int N = (pp_tile_keys(it, j) + 15) & ~15;
                    const uint32_t id = idesc_bf16(128, N, 0, 0);
                    const uint32_t dst = tmem + sb * kPpKeys;
                    for (int s = 0; s < 8; ++s) {
                        const uint32_t st = kr % kPpRing;
                        if (!warp_wait(&bars[kBarKFull + st], (kr / kPpRing) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        if (lane == 0) {
                            const uint32_t kb = smem_u32(sm + kPpSmRing + st * kPpUnit);
                            const uint32_t qa = q_base + s * kPpQSlab;
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_ss(dst, smem_desc_sw128(qa + kk * 32, 16, 1024),
                                       smem_desc_sw128(kb + kk * 32, 16, 1024), id, (s | kk) ? 1u : 0u);
                            mma_commit(&bars[kBarKEmpty + st]);
                        }
                        __syncwarp();
                        ++kr;
                    }
                    if (!ok) break;
                    if (lane == 0) {
                        mma_commit(&bars[kBarSFull + sb]);
                        if (j == nt - 1) mma_commit(&bars[kBarQEmpty]);
                    }
                    __syncwarp();
                }
            }
            if (lane == 0) {
                mma_commit(&bars[kBarDrain]);
                pp_drain_wait(&bars[kBarDrain], 0);
            }
            __syncwarp();
        }
    } else if (s_cta && warp >= 2 && warp <= 5) {
        // ===================================================== S-CTA: softmax, P to the O-CTA
        if (go) {
            const int q4 = warp & 3;
            const int r = q4 * 32 + lane;
            const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
            const uint32_t rP = peer_base + kPpSmP + (uint32_t)r * 16u;
            const uint32_t rHdr = peer_base + kPpSmHdr;
            const uint32_t rPFull = peer_base + kPpSmBar + kBarPFull * 8;
            const float sl2 = p.scale_log2;
            int n = 0;
            bool ok = true;
            for (long long i = pair; ok && i < p.items; i += npairs) {
                const PpItem it = pp_item(p, i);
                const int nt = it.nct + it.nwt;
                const int tok = it.t0 + r / p.G;
                const bool row_live = tok < p.T;
                const int t = row_live ? tok : p.T - 1;
                const int head = it.g * p.G + (r % p.G);
                const int nc_t = pf_visible(t, p.W, p.blk);
                float m = -INFINITY, l = 0.f;
                for (int j = 0; j < nt; ++j, ++n) {
                    const int sb = n & 1;
                    const int nk = pp_tile_keys(it, j);
                    const int ncol = (nk + 15) & ~15;
                    int lo, hi;               // valid columns of this row: [lo, hi)
                    if (j < it.nct) {
                        lo = 0;
                        hi = min(nk, nc_t - kPpKeys * j);
                    } else {
                        const int u0 = it.wlo + kPpKeys * (j - it.nct);
                        lo = max(0, t - p.W + 1 - u0);
                        hi = min(nk, t - u0 + 1);
                    }
                    if (!warp_wait(&bars[kBarSFull + sb], (n >> 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = tmem + lane_off + sb * kPpKeys;
                    // The reference maximum m of a row is lazy: P = 2^(logit - m) is computed
                    // against the reference of the earlier tiles, and m moves only when a tile
                    // exceeds it by 2^8 -- the tile is then redone against the new reference.  A
                    // warp in which some row has no reference yet takes the tile maximum first.
                    const bool need_max = __any_sync(0xffffffffu, m == -INFINITY);
                    float tmax = -INFINITY;
                    if (need_max) {
#pragma unroll 1
                        for (int c0 = 0; c0 < ncol; c0 += 64) {
                            float v[64];
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                if (c0 + 16 * k < ncol) tmem_ld16(sa + c0 + 16 * k, v + 16 * k);
                            tmem_wait_ld();
#pragma unroll
                            for (int k = 0; k < 64; ++k) {
                                const int c = c0 + k;
                                if (c >= lo && c < hi) tmax = fmaxf(tmax, v[k] * sl2);
                            }
                        }
                    }
                    bool resc = false;
                    float al = 1.f;
                    if (need_max) {
                        resc = m != -INFINITY && tmax > m + kPfRescale;
                        if (resc) {
                            al = ex2(m - tmax);
                            l *= al;
                        }
                        if (resc || (m == -INFINITY && tmax > -INFINITY)) m = tmax;
                    }
                    // the O-CTA's P slot is free once the PV of tile n-2 has landed
                    if (!pp_warp_wait_cl(&bars[kBarPEmpty + sb], ((n >> 1) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    // P in bf16, stored into the peer: keys 8c..8c+7 of this row at chunk c
                    // (2 KB per chunk of 8 keys x 128 rows)
                    const uint32_t pbase = rP + sb * kPpPBuf;
                    float rs;
                    for (int attempt = 0;; ++attempt) {
                        const float mref = m == -INFINITY ? 0.f : m;
                        float dmax = -INFINITY;
                        rs = 0.f;
#pragma unroll 1
                        for (int c0 = 0; c0 < ncol; c0 += 64) {
                            float v[64];
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                if (c0 + 16 * k < ncol) tmem_ld16(sa + c0 + 16 * k, v + 16 * k);
                            tmem_wait_ld();
#pragma unroll
                            for (int k16 = 0; k16 < 4; ++k16) {
                                const int cb = c0 + 16 * k16;
                                if (cb < ncol) {
                                    uint32_t pk[8];
#pragma unroll
                                    for (int e = 0; e < 8; ++e) {
                                        const int c = cb + 2 * e;
                                        const float d0 = (c >= lo && c < hi) ? fmaf(v[16 * k16 + 2 * e], sl2, -mref)
                                                                             : -INFINITY;
                                        const float d1 = (c + 1 >= lo && c + 1 < hi)
                                                             ? fmaf(v[16 * k16 + 2 * e + 1], sl2, -mref) : -INFINITY;
                                        dmax = fmaxf(dmax, fmaxf(d0, d1));
                                        const float a = ex2(d0), b2 = ex2(d1);
                                        rs += a + b2;
                                        pk[e] = pack_bf16x2(a, b2);
                                    }
                                    const uint32_t ra = pbase + ((uint32_t)cb >> 3) * 2048u;
                                    pp_st_cluster_v4(ra, pk[0], pk[1], pk[2], pk[3]);
                                    pp_st_cluster_v4(ra + 2048u, pk[4], pk[5], pk[6], pk[7]);
                                }
                            }
                        }
                        if (need_max || attempt) break;
                        // every row of this warp has a reference here; redo if one was exceeded
                        const bool over = dmax > kPfRescale;
                        if (!__any_sync(0xffffffffu, over)) break;
                        if (over) {
                            al = ex2(-dmax);
                            l *= al;
                            m += dmax;
                            resc = true;
                        }
                    }
                    l += rs;
                    // every TMEM load of this warp has completed: S may be overwritten
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars[kBarSEmpty + sb]);
                    // header of the slot: rescale factor per row, per-warp flag, row sums
                    const uint32_t hdr = rHdr + sb * kPpHdrBytes;
                    pp_st_cluster_u32(hdr + r * 4, __float_as_uint(al));
                    if (j == nt - 1) pp_st_cluster_u32(hdr + 512 + r * 4, __float_as_uint(l));
                    const bool any = __any_sync(0xffffffffu, resc);
                    if (lane == 0) pp_st_cluster_u32(hdr + 1024 + q4 * 4, any ? 1u : 0u);
                    pp_fence_proxy_async_cluster();
                    __syncwarp();
                    if (lane == 0) pp_remote_arrive(rPFull + sb * 8);
                }
                if (!ok) break;
                if (row_live && p.lse)
                    p.lse[((size_t)it.b * p.Hq + head) * p.T + tok] = (m + log2f(l)) * 0.6931471805599453f;
            }
        }
    }
    else if (!s_cta && warp == 0) {
        // ===================================================== O-CTA: TMA of V
        if (lane == 0 && go) {
            uint32_t vr = 0;
            bool ok = true;
            for (long long i = pair; ok && i < p.items; i += npairs) {
                const PpItem it = pp_item(p, i);
                const int nt = it.nct + it.nwt;
                for (int j = 0; ok && j < nt; ++j) {
                    const bool comp = j < it.nct;
                    const int row = pp_tile_row(it, j);
                    const int nu = (pp_tile_keys(it, j) + 63) >> 6;
                    for (int h = 0; ok && h < 2; ++h)
                        for (int u = 0; u < nu; ++u) {
                            const uint32_t st = vr % kPpRing;
                            if (!mbar_wait(&bars[kBarVEmpty + st], ((vr / kPpRing) & 1) ^ 1, abort_flag)) {
                                ok = false;
                                break;
                            }
                            mbar_arrive_expect_tx(&bars[kBarVFull + st], kPpUnit);
                            for (int c = 0; c < 4; ++c)
                                tma_load_4d(sm + kPpSmRing + st * kPpUnit + c * kPpVSub, comp ? &tm_vc : &tm_v,
                                            &bars[kBarVFull + st], 256 * h + 64 * c, it.g, row + 64 * u, it.b);
                            ++vr;
                        }
                }
            }
            pp_drain_ring(&bars[kBarVFull], vr);
        }
    } else if (!s_cta && warp == 1) {
        // ===================================================== O-CTA: O += P V
        if (go) {
            uint32_t vr = 0;
            int n = 0, item_n = 0;
            bool ok = true;
            const uint32_t p_base = smem_u32(sm + kPpSmP);
            const uint32_t id = idesc_bf16(128, 256, 0, 1);
            for (long long i = pair; ok && i < p.items; i += npairs, ++item_n) {
                const PpItem it = pp_item(p, i);
                const int nt = it.nct + it.nwt;
                for (int j = 0; ok && j < nt; ++j, ++n) {
                    const int sb = n & 1;
                    if (!pp_warp_wait_cl(&bars[kBarPFull + sb], (n >> 1) & 1, abort_flag) ||
                        !warp_wait(&bars[kBarCorr + sb], (n >> 1) & 1, abort_flag) ||
                        (j == 0 && !warp_wait(&bars[kBarOEmpty], (item_n & 1) ^ 1, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nk = pp_tile_keys(it, j);
                    const int nu = (nk + 63) >> 6;
                    for (int h = 0; ok && h < 2; ++h)
                        for (int u = 0; u < nu; ++u) {
                            const uint32_t st = vr % kPpRing;
                            if (!warp_wait(&bars[kBarVFull + st], (vr / kPpRing) & 1, abort_flag)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            if (lane == 0) {
                                const uint32_t vb = smem_u32(sm + kPpSmRing + st * kPpUnit);
                                const uint32_t pa = p_base + sb * kPpPBuf + u * 16384;   // 16 keys = 4 KB
#pragma unroll
                                for (int kk = 0; kk < 4; ++kk)
                                    if (64 * u + 16 * kk < nk)
                                        mma_ss(tmem + 256 * h, pp_desc_noswz(pa + kk * 4096, 2048, 128),
                                               smem_desc_sw128(vb + kk * 2048, kPpVSub, 1024), id,
                                               (j == 0 && u == 0 && kk == 0) ? 0u : 1u);
                                mma_commit(&bars[kBarVEmpty + st]);
                            }
                            __syncwarp();
                            ++vr;
                        }
                    if (!ok) break;
                    if (lane == 0) {
                        mma_commit(&bars[kBarPCons + sb]);
                        if (j == nt - 1) mma_commit(&bars[kBarOFull]);
                    }
                    __syncwarp();
                }
            }
            if (lane == 0) {
                mma_commit(&bars[kBarDrain]);
                pp_drain_wait(&bars[kBarDrain], 0);
            }
            __syncwarp();
        }
    } else if (!s_cta && warp >= 2 && warp <= 5) {
        // ===================================================== O-CTA: rescale, epilogue
        if (go) {
            const int q4 = warp & 3;
            const int r = q4 * 32 + lane;
            const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
            int n = 0, item_n = 0;
            bool ok = true;
            for (long long i = pair; ok && i < p.items; i += npairs, ++item_n) {
                const PpItem it = pp_item(p, i);
                const int nt = it.nct + it.nwt;
                const int tok = it.t0 + r / p.G;
                const bool row_live = tok < p.T;
                const int head = it.g * p.G + (r % p.G);
                float lfin = 1.f;
                for (int j = 0; j < nt; ++j, ++n) {
                    const int sb = n & 1;
                    if (!pp_warp_wait_cl(&bars[kBarPFull + sb], (n >> 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint8_t* hdr = sm + kPpSmHdr + sb * kPpHdrBytes;
                    const int flag = *reinterpret_cast<const volatile int*>(hdr + 1024 + q4 * 4);
                    const float al = *reinterpret_cast<const volatile float*>(hdr + r * 4);
                    if (j == nt - 1) lfin = *reinterpret_cast<const volatile float*>(hdr + 512 + r * 4);
                    if (flag) {
                        // a row of this warp moved its reference maximum (never on a first
                        // tile): scale O once the PV of tile n-1 has landed
                        if (!warp_wait(&bars[kBarPCons + ((n - 1) & 1)], ((n - 1) >> 1) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll 1
                        for (int c0 = 0; c0 < kPpD; c0 += 64) {
                            float o[64];
#pragma unroll
                            for (int k = 0; k < 4; ++k) tmem_ld16(tmem + lane_off + c0 + 16 * k, o + 16 * k);
                            tmem_wait_ld();
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                uint32_t w[16];
#pragma unroll
                                for (int e = 0; e < 16; ++e) w[e] = __float_as_uint(o[16 * k + e] * al);
                                tmem_st16(tmem + lane_off + c0 + 16 * k, w);
                            }
                        }
                        tmem_wait_st();
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars[kBarCorr + sb]);
                }
                if (!ok) break;
                // ---- epilogue: out = O / l
                if (!warp_wait(&bars[kBarOFull], item_n & 1, abort_flag)) break;
                tc_fence_after();
                const float inv = 1.f / lfin;
                const size_t orow = (((size_t)it.b * p.T + tok) * p.Hq + head) * (size_t)kPpD;
#pragma unroll 1
                for (int c0 = 0; c0 < kPpD; c0 += 32) {
                    float o[32];
                    tmem_ld16(tmem + lane_off + c0, o);
                    tmem_ld16(tmem + lane_off + c0 + 16, o + 16);
                    tmem_wait_ld();
                    if (row_live) {
                        if (p.flags & HCA_OUT_F32) {
                            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow + c0);
#pragma unroll
                            for (int k = 0; k < 8; ++k)
                                dst[k] = make_float4(o[4 * k] * inv, o[4 * k + 1] * inv, o[4 * k + 2] * inv,
                                                     o[4 * k + 3] * inv);
                        } else {
                            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + orow + c0);
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                dst[k] = make_uint4(pack_bf16x2(o[8 * k] * inv, o[8 * k + 1] * inv),
                                                    pack_bf16x2(o[8 * k + 2] * inv, o[8 * k + 3] * inv),
                                                    pack_bf16x2(o[8 * k + 4] * inv, o[8 * k + 5] * inv),
                                                    pack_bf16x2(o[8 * k + 6] * inv, o[8 * k + 7] * inv));
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[kBarOEmpty]);
            }
        }
    } else if (!s_cta && warp == 6) {
        // ===================================================== O-CTA: P slot consumed -> S-CTA
        if (lane == 0 && go) {
            const uint32_t rPEmpty = peer_base + kPpSmBar + kBarPEmpty * 8;
            int n = 0;
            bool ok = true;
            for (long long i = pair; ok && i < p.items; i += npairs) {
                const PpItem it = pp_item(p, i);
                const int nt = it.nct + it.nwt;
                for (int j = 0; j < nt; ++j, ++n) {
                    if (!mbar_wait(&bars[kBarPCons + (n & 1)], (n >> 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    pp_remote_arrive(rPEmpty + (n & 1) * 8);
                }
            }
        }
    }

    __syncwarp();           // every role reconverges its warp before the CTA-wide barrier
    tc_fence_before();
    __syncthreads();
    pp_cluster_sync();      // no remote store or arrive is still aimed at a CTA that leaves
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace hca
