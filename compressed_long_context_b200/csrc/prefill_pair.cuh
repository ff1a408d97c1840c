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
//       (thread = row), and P (bf16) stored straight into a slot of the O-CTA's shared
//       memory with st.async, in the non-swizzled K-major layout the tensor core reads (8 keys
//       of row r at (key / 8) * 2048 + r * 16).  Every such store counts its bytes on the
//       O-CTA's slot barrier (mbarrier::complete_tx), and each lane quarter arms that barrier
//       with the byte total it stored, so the writers never wait for completion.  A per-unit
//       header (each row's rescale factor, a flag per lane quarter) travels the same way.  The
//       hand-off granule is a P unit of 128 keys (half an S tile), three slots in flight;
//   O-CTA (cluster rank 1): V tiles streamed by TMA, O += P V with N = 256 value columns
//       (two MMAs per 16 keys cover the 512 columns), rescale of O rows when the S-CTA moved
//       a row's reference maximum, and the epilogue out = O / l.
// Every MMA is M = 128, N = 256 (or the 16-rounded key count of a short tile): the tcgen05
// issue cost of one M = 128 MMA does not shrink with N, so narrow MMAs waste the pipe.
//
// Warps (320 threads, same kernel for both ranks):
//   S-CTA: 0 TMA (Q, K) | 1 MMA + TMEM | 2-9 softmax (two warps per TMEM lane quarter)
//   O-CTA: 0 TMA (V)    | 1 MMA + TMEM | 2-5 rescale + epilogue | 7 "P slot consumed"
//          forwarded to the S-CTA (its own warp, so that a slot is returned the moment its
//          PV lands, whatever else is waiting) | 6, 8, 9 idle
//
// Tiles of one row tile (item): the compressed segment in tiles of 256 entries, then the
// raw window [wlo, tlast] in tiles of 256 tokens; per-row masks [lo, hi) as in prefill.cuh.
// Lazy rescaling: a row moves its reference maximum only when a tile's maximum exceeds it
// by 2^8, so the O-CTA rarely touches O between MMAs.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "prefill.cuh"

namespace hca {

constexpr int kPpThreads = 320;
constexpr int kPpSoftWarps = 8;                 // S-CTA softmax warps (2..9)
constexpr int kPpKeys = 256;                     // keys per S tile (MMA N of S)
constexpr int kPpUKeys = 128;                    // keys per P unit (the hand-off granule)
#ifndef HCA_PP_SLOTS
#define HCA_PP_SLOTS 3
#endif
#ifndef HCA_PP_VRING
#define HCA_PP_VRING 3
#endif
constexpr int kPpSlots = HCA_PP_SLOTS;           // P units in flight between the two CTAs
constexpr int kPpD = 512;
constexpr int kPpRingK = 3;                      // K units in flight (S-CTA)
constexpr int kPpRingV = HCA_PP_VRING;           // V units in flight (O-CTA)
constexpr uint32_t kPpQSlab = 128 * 128;         // Q: 128 rows x 64 channels
constexpr uint32_t kPpUnit = 32768;              // K: 256 keys x 64 ch; V: 64 keys x 256 ch
constexpr uint32_t kPpVSub = 8192;               // V unit = 4 channel slabs of 64 keys x 64 ch
constexpr uint32_t kPpPBuf = 32768;              // P unit: 128 rows x 128 keys, 16 key chunks of 2 KB
constexpr uint32_t kPpHdrBytes = 528;            // per P unit: alpha[128], flag[4]
// shared-memory layout (offsets from a 1024-aligned base); the two ranks reuse offsets
constexpr uint32_t kPpSmQ = 0;                   // S-CTA: Q, 8 slabs (128 KB)
constexpr uint32_t kPpSmP = 0;                   // O-CTA: P units
constexpr uint32_t kPpSmStage = kPpSmP + kPpSlots * kPpPBuf;   // O-CTA: output staging, 4 warps x 8 KB
constexpr uint32_t kPpStageWarp = 8192;          // 2 pieces of 4 KB: 32 rows x 64 bf16 or 32 fp32 columns
constexpr uint32_t kPpSmRing = 131072;           // S-CTA: K ring (after Q)
constexpr uint32_t kPpSmVRing = kPpSmStage + 4 * kPpStageWarp;  // O-CTA: V ring (after staging)
constexpr uint32_t kPpSmHdr = kPpSmRing + kPpRingK * kPpUnit;    // O-CTA: unit headers
constexpr uint32_t kPpSmXch = kPpSmHdr;          // S-CTA: softmax exchange, 2 x 2 x 128 floats
constexpr uint32_t kPpHdrArea = kPpSlots * kPpHdrBytes > 2048 ? kPpSlots * kPpHdrBytes : 2048;
constexpr uint32_t kPpSmBar = kPpSmHdr + kPpHdrArea;
constexpr int kPpNumBars = 56;                  // 56 used; even count keeps misc 16-aligned
constexpr uint32_t kPpSmMisc = kPpSmBar + kPpNumBars * 8;
constexpr uint32_t kPpSmem = kPpSmMisc + 16;
static_assert(kPpSmem <= 232448, "pair prefill shared memory exceeds the 227 KB per-block limit");
static_assert(kPpSmHdr % 16 == 0 && kPpSmBar % 8 == 0 && kPpSmMisc % 16 == 0,
              "header 16-aligned, barriers 8-aligned");
static_assert(kPpKeys == 2 * kPpUKeys, "an S tile is two P units");
static_assert(kPpSlots <= 4 && kPpRingV <= 4 && kPpRingK == 3, "barrier index ranges");
static_assert(kPpSmVRing + kPpRingV * kPpUnit <= kPpSmHdr, "O-CTA: P, staging and the V ring fit");
static_assert(kPpSmVRing % 1024 == 0, "V units 1024-aligned");

// barrier indices (both ranks initialise all of them; each rank uses its own)
enum : int {
    kBarKFull = 0, kBarKEmpty = 3, kBarSFull = 8, kBarSEmpty = 10,      // (6, 7 unused)
    kBarPEmpty = 12,                                                       // S-CTA (+ [<= 4])
    kBarVFull = 16, kBarVEmpty = 20, kBarPFull = 24, kBarCorr = 28, kBarPCons = 32,
    kBarOFull = 36, kBarOEmpty = 37,                                       // O-CTA
    kBarDrain = 38,
    kBarQSFull = 40, kBarQSEmpty = 48                                      // S-CTA: per Q slab [8]
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
// P units of a tile with nk keys, and the keys / 16-rounded columns of unit hh
__device__ __forceinline__ int pp_units(int nk) { return (nk + kPpUKeys - 1) / kPpUKeys; }
__device__ __forceinline__ int pp_unit_keys(int nk, int hh) { return min(kPpUKeys, nk - hh * kPpUKeys); }
__device__ __forceinline__ int pp_unit_cols(int nk, int hh) { return min(kPpUKeys, ((nk + 15) & ~15) - hh * kPpUKeys); }

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
// Asynchronous stores into a peer CTA's shared memory; each completes `bytes` of the peer's
// mbarrier transaction count (release at cluster scope), so the writer never waits.
__device__ __forceinline__ void pp_st_async_v4(uint32_t raddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                                               uint32_t rbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];"
                 :: "r"(raddr), "r"(a), "r"(b), "r"(c), "r"(d), "r"(rbar) : "memory");
}
__device__ __forceinline__ void pp_st_async_u32(uint32_t raddr, uint32_t v, uint32_t rbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];"
                 :: "r"(raddr), "r"(v), "r"(rbar) : "memory");
}
// Arrival + expected bytes on a peer's barrier.  Relaxed: the bytes carry their own release
// (complete_tx of st.async), and a release here would wait for every store still in flight.
__device__ __forceinline__ void pp_remote_arrive_expect_tx(uint32_t rbar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.relaxed.cluster.shared::cluster.b64 _, [%0], %1;"
                 :: "r"(rbar), "r"(bytes) : "memory");
}
// TMA tensor store (shared -> global) of one box, tracked by the issuing thread's bulk groups
__device__ __forceinline__ void pp_tma_store_4d(const CUtensorMap* m, const void* src, int c0, int c1, int c2,
                                                int c3) {
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];"
                 :: "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}
__device__ __forceinline__ void pp_bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void pp_bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void pp_bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void pp_bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void pp_st_cluster_u32(uint32_t raddr, uint32_t v) {
    asm volatile("st.shared::cluster.b32 [%0], %1;" :: "r"(raddr), "r"(v) : "memory");
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
            if (globaltimer_ns() - t0 > wait_limit_ns()) {
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
        if (globaltimer_ns() - t0 > wait_limit_ns()) {
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
__device__ __forceinline__ void pp_drain_ring(uint64_t* full, uint32_t issued, uint32_t ring) {
    for (uint32_t st = 0; st < ring; ++st)
        if (issued > st) pp_drain_wait(&full[st], ((issued - 1 - st) / ring) & 1);
}

__global__ void __launch_bounds__(kPpThreads, 1)   // 10 warps: at most 168 registers (3 warps per SMSP)
prefill_pair_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_vc,
                    const __grid_constant__ CUtensorMap tm_out) {
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
        for (int i = 0; i < kPpRingK; ++i) {
            mbar_init(&bars[kBarKFull + i], 1);
            mbar_init(&bars[kBarKEmpty + i], 1);
        }
        for (int i = 0; i < kPpRingV; ++i) {
            mbar_init(&bars[kBarVFull + i], 1);
            mbar_init(&bars[kBarVEmpty + i], 1);
        }
        for (int i = 0; i < 8; ++i) {
            mbar_init(&bars[kBarQSFull + i], 1);
            mbar_init(&bars[kBarQSEmpty + i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars[kBarSFull + i], 1);
            mbar_init(&bars[kBarSEmpty + i], kPpSoftWarps);
        }
        for (int i = 0; i < kPpSlots; ++i) {
            mbar_init(&bars[kBarPEmpty + i], 1);
            mbar_init(&bars[kBarPFull + i], 4);        // armed by each TMEM lane quarter
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
            prefetch_tmap(&tm_out);
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
                const int nt = it.nct + it.nwt;
                for (int j = 0; ok && j < nt; ++j) {
                    const bool comp = j < it.nct;
                    const int row = pp_tile_row(it, j);
                    for (int s = 0; s < 8; ++s) {
                        if (j == 0) {
                            // Q slab s of this row tile, as soon as the previous row tile's last
                            // MMAs on slab s have completed (not after its whole last tile)
                            if (!mbar_wait(&bars[kBarQSEmpty + s], (qn & 1) ^ 1, abort_flag)) {
                                ok = false;
                                break;
                            }
                            mbar_arrive_expect_tx(&bars[kBarQSFull + s], kPpQSlab);
                            tma_load_4d(sm + kPpSmQ + s * kPpQSlab, &tm_q, &bars[kBarQSFull + s], 64 * s,
                                        it.g * p.G, it.t0, it.b);
                        }
                        const uint32_t st = kr % kPpRingK;
                        if (!mbar_wait(&bars[kBarKEmpty + st], ((kr / kPpRingK) & 1) ^ 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&bars[kBarKFull + st], kPpUnit);
                        tma_load_4d(sm + kPpSmRing + st * kPpUnit, comp ? &tm_kc : &tm_k, &bars[kBarKFull + st],
                                    64 * s, it.g, row, it.b);
                        ++kr;
                    }
                }
                ++qn;
            }
            pp_drain_ring(&bars[kBarKFull], kr, kPpRingK);
            if (qn)
                for (int s = 0; s < 8; ++s) pp_drain_wait(&bars[kBarQSFull + s], (qn - 1) & 1);
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
                        const uint32_t st = kr % kPpRingK;
                        // Q slab s of this row tile (landed once per item, used by every tile)
                        if ((j == 0 && !warp_wait(&bars[kBarQSFull + s], item_n & 1, abort_flag)) ||
                            !warp_wait(&bars[kBarKFull + st], (kr / kPpRingK) & 1, abort_flag)) {
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
                            // the row tile's last use of Q slab s: the next row tile's slab s
                            // may land once these MMAs have completed
                            if (j == nt - 1) mma_commit(&bars[kBarQSEmpty + s]);
                        }
                        __syncwarp();
                        ++kr;
                    }
                    if (!ok) break;
                    if (lane == 0) mma_commit(&bars[kBarSFull + sb]);
                    __syncwarp();
                }
            }
            if (lane == 0) {
                mma_commit(&bars[kBarDrain]);
                pp_drain_wait(&bars[kBarDrain], 0);
            }
            __syncwarp();
        }
    } else if (s_cta && warp >= 2 && warp < 2 + kPpSoftWarps) {
        // ===================================================== S-CTA: softmax, P to the O-CTA
        // Eight warps: warp w owns the 32 rows of TMEM lane quarter w % 4 and one half of the
        // columns of every unit (hw = 0: the first 64, hw = 1: the last 64).  The two warps of
        // a quarter keep identical per-row references m (they take the same decisions from
        // the same exchanged maxima) and their own partial row sums.
        if (go) {
            const int q4 = warp & 3;
            const int hw = (warp - 2) >> 2;
            const int r = q4 * 32 + lane;
            const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
            float* xch = reinterpret_cast<float*>(sm + kPpSmXch);     // [2 parities][2 halves][128 rows]
            int xpar = 0;
            // a value of this row from both warps of the quarter (64-thread named barrier)
            auto exchange = [&](float mine, float* other) {
                xch[(xpar * 2 + hw) * 128 + r] = mine;
                asm volatile("bar.sync %0, 64;" :: "r"(4 + q4) : "memory");
                *other = xch[(xpar * 2 + (hw ^ 1)) * 128 + r];
                xpar ^= 1;
            };
            // the two warps of a quarter go on or unwind together: a verdict that differed
            // would leave one of them at a named barrier the other never reaches
            auto pair_agree = [&](bool ok_mine) -> bool {
                uint32_t res;
                asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
                             "barrier.red.and.pred q, %2, 64, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                             : "=r"(res) : "r"((uint32_t)ok_mine), "r"(4 + q4) : "memory");
                return res != 0;
            };
            const uint32_t rP = peer_base + kPpSmP + (uint32_t)r * 16u;
            const uint32_t rHdr = peer_base + kPpSmHdr;
            const uint32_t rPFull = peer_base + kPpSmBar + kBarPFull * 8;
            const float sl2 = p.scale_log2;
            int n = 0;            // S tiles
            uint32_t un = 0;      // P units
            bool ok = true;
            for (long long i = pair; ok && i < p.items; i += npairs) {
                const PpItem it = pp_item(p, i);
                const int nt = it.nct + it.nwt;
                const int tok = it.t0 + r / p.G;
                const bool row_live = tok < p.T;
                const int t = row_live ? tok : p.T - 1;
                const int head = it.g * p.G + (r % p.G);
                const int nc_t = pf_visible(t, p.W, p.blk);
                float m = -INFINITY, l = 0.f;     // l: this warp's partial row sum
                for (int j = 0; ok && j < nt; ++j, ++n) {
                    const int sb = n & 1;
                    const int nk = pp_tile_keys(it, j);
                    int lo, hi;               // valid columns of this row in the tile: [lo, hi)
                    if (j < it.nct) {
                        lo = 0;
                        hi = min(nk, nc_t - kPpKeys * j);
                    } else {
                        const int u0 = it.wlo + kPpKeys * (j - it.nct);
                        lo = max(0, t - p.W + 1 - u0);
                        hi = min(nk, t - u0 + 1);
                    }
                    if (!pair_agree(warp_wait(&bars[kBarSFull + sb], (n >> 1) & 1, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = tmem + lane_off + sb * kPpKeys;
                    const int nu = pp_units(nk);
                    for (int hh = 0; hh < nu; ++hh, ++un) {
                        const int us = (int)(un % kPpSlots);
                        const int u_end = hh * kPpUKeys + pp_unit_cols(nk, hh);
                        const int c_beg = hh * kPpUKeys + 64 * hw;            // this warp's columns
                        const int c_end = min(c_beg + 64, u_end);             // (may be empty)
                        // The reference maximum m of a row is lazy: P = 2^(logit - m) is computed
                        // against the reference of the earlier units, and m moves only when a unit
                        // exceeds it by 2^8 -- the unit is then redone against the new reference.
                        // A quarter in which some row has no reference yet takes the maximum first.
                        const bool need_max = __any_sync(0xffffffffu, m == -INFINITY);
                        bool resc = false;
                        float al = 1.f;
                        if (need_max) {
                            float tmax = -INFINITY;
#pragma unroll 1
                            for (int c0 = c_beg; c0 < c_end; c0 += 32) {
                                float v[32];
#pragma unroll
                                for (int k = 0; k < 2; ++k)
                                    if (c0 + 16 * k < c_end) tmem_ld16(sa + c0 + 16 * k, v + 16 * k);
                                tmem_wait_ld();
#pragma unroll
                                for (int k = 0; k < 32; ++k) {
                                    const int c = c0 + k;
                                    if (c >= lo && c < hi) tmax = fmaxf(tmax, v[k] * sl2);
                                }
                            }
                            float tother;
                            exchange(tmax, &tother);
                            tmax = fmaxf(tmax, tother);
                            resc = m != -INFINITY && tmax > m + kPfRescale;
                            if (resc) {
                                al = ex2(m - tmax);
                                l *= al;
                            }
                            if (resc || (m == -INFINITY && tmax > -INFINITY)) m = tmax;
                        }
                        // the O-CTA's slot us is free once the PV of unit un - kPpSlots has landed
                        if (!pair_agree(pp_warp_wait_cl(&bars[kBarPEmpty + us], ((un / kPpSlots) & 1) ^ 1,
                                                        abort_flag))) {
                            ok = false;
                            break;
                        }
                        // P in bf16 straight into the O-CTA's slot us: keys 8c..8c+7 of the unit,
                        // this row, at chunk c (2 KB per chunk of 8 keys x 128 rows).  Every store
                        // counts its bytes on the slot's barrier; each lane quarter arms it once
                        // it knows how many bytes it stored (a redone unit is stored twice).
                        const uint32_t pbar = rPFull + us * 8;
                        const uint32_t pbase = rP + us * kPpPBuf;
                        int attempts = 1;
                        // columns valid for every row of the warp (most compressed units) skip
                        // the per-column mask
                        const bool unmasked = __all_sync(0xffffffffu, lo <= c_beg && hi >= c_end);
                        float rs, dmax;
                        auto pass2 = [&](auto masked_tag, float mref) {
                            constexpr bool kMasked = decltype(masked_tag)::value;
                            dmax = -INFINITY;
                            rs = 0.f;
#pragma unroll 1
                            for (int c0 = c_beg; c0 < c_end; c0 += 32) {
                                float v[32];
#pragma unroll
                                for (int k = 0; k < 2; ++k)
                                    if (c0 + 16 * k < c_end) tmem_ld16(sa + c0 + 16 * k, v + 16 * k);
                                tmem_wait_ld();
#pragma unroll
                                for (int k16 = 0; k16 < 2; ++k16) {
                                    const int cb = c0 + 16 * k16;
                                    if (cb < c_end) {
                                        uint32_t pk[8];
#pragma unroll
                                        for (int e = 0; e < 8; ++e) {
                                            const int c = cb + 2 * e;
                                            float d0 = fmaf(v[16 * k16 + 2 * e], sl2, -mref);
                                            float d1 = fmaf(v[16 * k16 + 2 * e + 1], sl2, -mref);
                                            if (kMasked) {
                                                d0 = (c >= lo && c < hi) ? d0 : -INFINITY;
                                                d1 = (c + 1 >= lo && c + 1 < hi) ? d1 : -INFINITY;
                                            }
                                            dmax = fmaxf(dmax, fmaxf(d0, d1));
                                            const float a = ex2(d0), b2 = ex2(d1);
                                            rs += a + b2;
                                            pk[e] = pack_bf16x2(a, b2);
                                        }
                                        const uint32_t ra = pbase + ((uint32_t)(cb - hh * kPpUKeys) >> 3) * 2048u;
                                        pp_st_async_v4(ra, pk[0], pk[1], pk[2], pk[3], pbar);
                                        pp_st_async_v4(ra + 2048u, pk[4], pk[5], pk[6], pk[7], pbar);
                                    }
                                }
                            }
                        };
                        for (int attempt = 0;; ++attempt) {
                            const float mref = m == -INFINITY ? 0.f : m;
                            if (unmasked)
                                pass2(std::false_type{}, mref);
                            else
                                pass2(std::true_type{}, mref);
                            if (need_max || attempt) break;
                            // every row has a reference here; redo if a unit exceeded it
                            float dother;
                            exchange(dmax, &dother);
                            dmax = fmaxf(dmax, dother);
                            const bool over = dmax > kPfRescale;
                            if (!__any_sync(0xffffffffu, over)) break;
                            if (over) {
                                al = ex2(-dmax);
                                l *= al;
                                m += dmax;
                                resc = true;
                            }
                            attempts = 2;
                        }
                        l += rs;
                        if (hh == nu - 1) {
                            // every TMEM load of this warp from the tile has completed
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&bars[kBarSEmpty + sb]);
                        }
                        const bool last = j == nt - 1 && hh == nu - 1;
                        float lrow = 0.f;
                        if (last) {      // whole-row sums for the epilogue and the LSE
                            float lother;
                            exchange(l, &lother);
                            lrow = l + lother;
                        }
                        if (hw == 0) {
                            // unit header: rescale factor per row, per-quarter flag; then the arm:
                            // this quarter's P bytes (both warps, every attempt) and header bytes
                            const uint32_t hdr = rHdr + us * kPpHdrBytes;
                            pp_st_async_u32(hdr + r * 4, __float_as_uint(al), pbar);
                            const bool any = __any_sync(0xffffffffu, resc);
                            if (lane == 0) {
                                pp_st_async_u32(hdr + 512 + q4 * 4, any ? 1u : 0u, pbar);
                                pp_remote_arrive_expect_tx(
                                    pbar, (uint32_t)attempts * (uint32_t)(u_end - hh * kPpUKeys) * 64u + 32u * 4u + 4u);
                            }
                            if (last && row_live && p.lse)
                                p.lse[((size_t)it.b * p.Hq + head) * p.T + tok] =
                                    (m + log2f(lrow)) * 0.6931471805599453f;
                        }
                    }
                }
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
                    const int nk = pp_tile_keys(it, j);
                    for (int hh = 0; ok && hh < pp_units(nk); ++hh) {
                        const int nv = (pp_unit_keys(nk, hh) + 63) >> 6;
                        for (int h = 0; ok && h < 2; ++h)
                            for (int u = 0; u < nv; ++u) {
                                const uint32_t st = vr % kPpRingV;
                                if (!mbar_wait(&bars[kBarVEmpty + st], ((vr / kPpRingV) & 1) ^ 1, abort_flag)) {
                                    ok = false;
                                    break;
                                }
                                mbar_arrive_expect_tx(&bars[kBarVFull + st], kPpUnit);
                                for (int c = 0; c < 4; ++c)
                                    tma_load_4d(sm + kPpSmVRing + st * kPpUnit + c * kPpVSub, comp ? &tm_vc : &tm_v,
                                                &bars[kBarVFull + st], 256 * h + 64 * c, it.g,
                                                row + kPpUKeys * hh + 64 * u, it.b);
                                ++vr;
                            }
                    }
                }
            }
            pp_drain_ring(&bars[kBarVFull], vr, kPpRingV);
        }
    } else if (!s_cta && warp == 1) {
        // ===================================================== O-CTA: O += P V
        if (go) {
            uint32_t vr = 0, un = 0;
            int item_n = 0;
            bool ok = true;
            const uint32_t p_base = smem_u32(sm + kPpSmP);
            const uint32_t id = idesc_bf16(128, 256, 0, 1);
            for (long long i = pair; ok && i < p.items; i += npairs, ++item_n) {
                const PpItem it = pp_item(p, i);
                const int nt = it.nct + it.nwt;
                for (int j = 0; ok && j < nt; ++j) {
                    const int nk = pp_tile_keys(it, j);
                    const int nu = pp_units(nk);
                    for (int hh = 0; hh < nu; ++hh, ++un) {
                        const int us = (int)(un % kPpSlots);
                        const uint32_t ph = (un / kPpSlots) & 1;
                        const bool first = j == 0 && hh == 0;
                        if (!pp_warp_wait_cl(&bars[kBarPFull + us], ph, abort_flag) ||
                            !warp_wait(&bars[kBarCorr + us], ph, abort_flag) ||
                            (first && !warp_wait(&bars[kBarOEmpty], (item_n & 1) ^ 1, abort_flag))) {
                            ok = false;
                            break;
                        }
                        fence_proxy_async_smem();    // P arrived through the generic proxy
                        tc_fence_after();
                        const int nku = pp_unit_keys(nk, hh);
                        const int nv = (nku + 63) >> 6;
                        for (int h = 0; ok && h < 2; ++h)
                            for (int u = 0; u < nv; ++u) {
                                const uint32_t st = vr % kPpRingV;
                                if (!warp_wait(&bars[kBarVFull + st], (vr / kPpRingV) & 1, abort_flag)) {
                                    ok = false;
                                    break;
                                }
                                tc_fence_after();
                                if (lane == 0) {
                                    const uint32_t vb = smem_u32(sm + kPpSmVRing + st * kPpUnit);
                                    const uint32_t pa = p_base + us * kPpPBuf + u * 16384;   // 16 keys = 4 KB
#pragma unroll
                                    for (int kk = 0; kk < 4; ++kk)
                                        if (64 * u + 16 * kk < nku)
                                            mma_ss(tmem + 256 * h, pp_desc_noswz(pa + kk * 4096, 2048, 128),
                                                   smem_desc_sw128(vb + kk * 2048, kPpVSub, 1024), id,
                                                   (first && u == 0 && kk == 0) ? 0u : 1u);
                                    mma_commit(&bars[kBarVEmpty + st]);
                                }
                                __syncwarp();
                                ++vr;
                            }
                        if (!ok) break;
                        if (lane == 0) {
                            mma_commit(&bars[kBarPCons + us]);
                            if (j == nt - 1 && hh == nu - 1) mma_commit(&bars[kBarOFull]);
                        }
                        __syncwarp();
                    }
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
            uint32_t un = 0;
            int item_n = 0;
            bool ok = true;
            for (long long i = pair; ok && i < p.items; i += npairs, ++item_n) {
                const PpItem it = pp_item(p, i);
                const int nt = it.nct + it.nwt;
                float l = 0.f;            // row sum of the bf16 P this CTA multiplies with
                for (int j = 0; ok && j < nt; ++j) {
                    const int nk = pp_tile_keys(it, j);
                    const int nu = pp_units(nk);
                    for (int hh = 0; hh < nu; ++hh, ++un) {
                        const int us = (int)(un % kPpSlots);
                        if (!pp_warp_wait_cl(&bars[kBarPFull + us], (un / kPpSlots) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        const uint8_t* hdr = sm + kPpSmHdr + us * kPpHdrBytes;
                        const int flag = *reinterpret_cast<const volatile int*>(hdr + 512 + q4 * 4);
                        const float al = *reinterpret_cast<const volatile float*>(hdr + r * 4);
                        // l = l * alpha + the unit's P of this row (8 keys per 16-byte chunk)
                        float us_sum = 0.f;
                        const uint8_t* prow = sm + kPpSmP + us * kPpPBuf + r * 16;
                        const int nch = pp_unit_cols(nk, hh) >> 3;
#pragma unroll 4
                        for (int c = 0; c < nch; ++c) {
                            const uint4 w = *reinterpret_cast<const uint4*>(prow + c * 2048);
                            us_sum += (bf16lo(w.x) + bf16hi(w.x)) + (bf16lo(w.y) + bf16hi(w.y)) +
                                      (bf16lo(w.z) + bf16hi(w.z)) + (bf16lo(w.w) + bf16hi(w.w));
                        }
                        l = l * al + us_sum;
                        if (flag) {
                            // a row of this warp moved its reference maximum (never in the first
                            // unit of an item): scale O once the PV of unit un-1 has landed
                            const uint32_t pu = un - 1;
                            if (!warp_wait(&bars[kBarPCons + pu % kPpSlots], (pu / kPpSlots) & 1, abort_flag)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
#pragma unroll 1
                            for (int c0 = 0; c0 < kPpD; c0 += 32) {
                                float o[32];
#pragma unroll
                                for (int k = 0; k < 2; ++k) tmem_ld16(tmem + lane_off + c0 + 16 * k, o + 16 * k);
                                tmem_wait_ld();
#pragma unroll
                                for (int k = 0; k < 2; ++k) {
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
                        if (lane == 0) mbar_arrive(&bars[kBarCorr + us]);
                    }
                }
                if (!ok) break;
                // ---- epilogue: out = O / l.  Each warp stages 32 rows x 128 bytes at a time in
                // shared memory and writes them with one TMA tensor store (a coalesced box);
                // per-lane row stores would touch 32 lines per instruction.
                if (!warp_wait(&bars[kBarOFull], item_n & 1, abort_flag)) break;
                tc_fence_after();
                const float inv = 1.f / l;
                const bool f32 = (p.flags & HCA_OUT_F32) != 0;
                uint8_t* stg = sm + kPpSmStage + q4 * kPpStageWarp;
                const int r0 = q4 * 32;                       // first row of this warp's box
                const int tok0 = it.t0 + r0 / p.G, head0 = it.g * p.G + r0 % p.G;
                const bool live = tok0 < p.T;                 // rows past T are clipped by the store
                // a piece is 4 KB: 32 rows x 64 columns of bf16, or x 32 columns of fp32
                const int pw = f32 ? 32 : 64;
#pragma unroll 1
                for (int c0 = 0, k = 0; c0 < kPpD; c0 += pw, ++k) {
                    uint8_t* buf = stg + (k & 1) * (kPpStageWarp / 2);
                    if (k >= 2 && lane == 0) pp_bulk_wait_read1();     // the store of piece k-2 read it
                    __syncwarp();
                    if (f32) {
                        float o[32];
                        tmem_ld16(tmem + lane_off + c0, o);
                        tmem_ld16(tmem + lane_off + c0 + 16, o + 16);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 8; ++e)       // 128-byte swizzle: chunk e of row lane
                            *reinterpret_cast<float4*>(buf + lane * 128 + (((e ^ lane) & 7) << 4)) =
                                make_float4(o[4 * e] * inv, o[4 * e + 1] * inv, o[4 * e + 2] * inv,
                                            o[4 * e + 3] * inv);
                    } else {
#pragma unroll
                        for (int hv = 0; hv < 2; ++hv) {
                            float o[32];
                            tmem_ld16(tmem + lane_off + c0 + 32 * hv, o);
                            tmem_ld16(tmem + lane_off + c0 + 32 * hv + 16, o + 16);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 4; ++e)   // 128-byte swizzle: chunk 4 hv + e of row lane
                                *reinterpret_cast<uint4*>(buf + lane * 128 + ((((4 * hv + e) ^ lane) & 7) << 4)) =
                                    make_uint4(pack_bf16x2(o[8 * e] * inv, o[8 * e + 1] * inv),
                                               pack_bf16x2(o[8 * e + 2] * inv, o[8 * e + 3] * inv),
                                               pack_bf16x2(o[8 * e + 4] * inv, o[8 * e + 5] * inv),
                                               pack_bf16x2(o[8 * e + 6] * inv, o[8 * e + 7] * inv));
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0 && live) {
                        pp_tma_store_4d(&tm_out, buf, c0, head0, tok0, it.b);
                        pp_bulk_commit();
                    }
                }
                if (lane == 0) pp_bulk_wait_read0();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[kBarOEmpty]);
            }
            if (lane == 0) pp_bulk_wait_all();     // every output store has completed
            __syncwarp();
        }
    } else if (!s_cta && warp == 7) {
        // ===================================================== O-CTA: P slot consumed -> S-CTA
        if (lane == 0 && go) {
            const uint32_t rPEmpty = peer_base + kPpSmBar + kBarPEmpty * 8;
            uint32_t un = 0;
            bool ok = true;
            for (long long i = pair; ok && i < p.items; i += npairs) {
                const PpItem it = pp_item(p, i);
                const int nt = it.nct + it.nwt;
                for (int j = 0; ok && j < nt; ++j) {
                    const int nu = pp_units(pp_tile_keys(it, j));
                    for (int hh = 0; hh < nu; ++hh, ++un) {
                        const int us = (int)(un % kPpSlots);
                        if (!mbar_wait(&bars[kBarPCons + us], (un / kPpSlots) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        pp_remote_arrive(rPEmpty + us * 8);
                    }
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
