// dsa.cuh -- the sparse-attention layers' decode step (sm_100a): a lightweight indexer scores every
// past position, the top-k positions are kept, and the core attention of the query's heads runs
// over those positions only (Zhidx article "280B Total Parameters, 14B Activated ...", section
// "1. Latent-Gated Sparse Attention", DSA paragraph; wiki summary "Key claims": DeepSeek-style
// DSA in the full-context MLA layers, whose query, key and value are 256-dim).
//
// Forms (the pages leave them open; the oracle takes the same readings):
//   I(s) = sum_j w_j * max(0, q_I[j] . k_I[s])   (H_I indexer heads, one d_I = 64 key per position)
//   keep the k positions of largest I, equal scores in increasing position order
//   out[h] = softmax_s(scale * q[h] . k[s]) v[s] over the kept s, one key / value row per position
//
// Kernels:
//   dsa_index_kernel   two persistent CTAs per SM over all (sequence, 128-position tile) pairs:
//                      a tile's indexer keys (128 x 64 bf16, 16 KB) arrive by TMA into a 6-slot
//                      ring, one tcgen05 MMA chain gives the 128 x H_I dot products in tensor
//                      memory (two buffers), four epilogue warps apply ReLU and the head weights
//                      and write the scores (fp32).  HBM-bound on the keys.
//   dsa_topk_kernel    a cluster of four CTAs per sequence, each over a quarter of the
//                      positions: radix select of the k-th largest score (three digit passes of
//                      11 / 11 / 10 bits over order-preserving integer keys, warp-aggregated
//                      shared-memory histograms summed by rank 0 through distributed shared
//                      memory), then one ordered pass that keeps every larger score and the
//                      first equal ones, positions ascending.
//   dsa_attend_kernel  two CTAs per sequence: the query heads (64 x 256 bf16) stay in shared
//                      memory; per tile of 128 kept positions, the key rows and then the value
//                      rows are gathered by TMA (tile::gather4: four 128-byte row segments per
//                      copy) into 128-byte-swizzled slabs, S^T = K Q^T and
//                      O^T += V^T P^T run on tcgen05 (as in the HCA decode), four warps run an
//                      online softmax with a lazily moved reference maximum, and four more issue
//                      the gathers as soon as a buffer is free.
// Every wait is bounded (common.cuh).
#pragma once

#include "common.cuh"

namespace hca {

constexpr int kDsaDI = 64;                 // indexer key / query dimension (one 128-byte row)
constexpr int kDsaD = 256;                 // core attention head dimension
constexpr int kDsaHeads = 64;              // query heads of a sequence (MMA N, padded)
constexpr int kDsaMaxHI = 64;              // indexer heads (MMA N, multiple of 16)

// Byte offset of 16-byte chunk c of row r in a 128-byte-swizzled slab (the TMA / tcgen05 layout).
__device__ __forceinline__ uint32_t dsa_sw(uint32_t r, uint32_t c) { return r * 128u + (((c ^ r) & 7u) << 4); }

// Bounded wait by a group of 128 threads (named barrier 2) with one verdict for the group, so
// that the group either goes on together or unwinds together.
__device__ __forceinline__ bool dsa_group_wait128(uint64_t* bar, uint32_t parity, volatile int* abort) {
    const bool ok = mbar_wait(bar, parity, abort);
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
                 "barrier.red.and.pred q, 2, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r) : "r"((uint32_t)ok) : "memory");
    return r != 0;
}

// ------------------------------------------------------------------------------------- indexer

constexpr int kIdxThreads = 192;           // producer, MMA issuer, 4 epilogue warps
constexpr int kIdxRing = 6;                // two CTAs per SM: 12 slots per SM
constexpr uint32_t kIdxSlab = 128 * 128;   // 128 positions x 64 dims bf16
constexpr uint32_t kIdxQBytes = kDsaMaxHI * 128;
constexpr uint32_t kIdxSmRing = 0;
constexpr uint32_t kIdxSmQ = kIdxSmRing + kIdxRing * kIdxSlab;          // two query buffers
constexpr uint32_t kIdxSmBar = kIdxSmQ + 2 * kIdxQBytes;
constexpr int kIdxNumBars = 2 * kIdxRing + 9;                           // ring full / empty, q, acc, drain
constexpr uint32_t kIdxSmW = kIdxSmBar + ((kIdxNumBars * 8 + 15) & ~15);  // two weight buffers [64]
constexpr uint32_t kIdxSmem = kIdxSmW + 2 * kDsaMaxHI * 4 + 16;
static_assert(kIdxSmQ % 1024 == 0 && kIdxSlab % 1024 == 0, "swizzled operands 1024-aligned");
static_assert(kIdxSmem <= 232448, "indexer shared memory exceeds the per-block limit");

struct DsaIndexParams {
    const float* w;          // [B, HI]
    const int* seqlens;      // [B]
    float* scores;           // [B, Lmax]
    int B, HI, Lmax, ntile;  // ntile = ceil(Lmax / 128)
    long long total;         // B * ntile
};

__device__ __forceinline__ int dsa_len(const DsaIndexParams& p, int b) {
    const int L = __ldg(p.seqlens + b);
    return L < 0 ? 0 : (L > p.Lmax ? p.Lmax : L);
}

// Walks (sequence, tile) pairs in order from a flat index, with the sequence's length cached.
struct DsaTileWalk {
    int b, t, L;
    __device__ DsaTileWalk(const DsaIndexParams& p, long long i) {
        b = (int)(i / p.ntile);
        t = (int)(i - (long long)b * p.ntile);
        L = b < p.B ? dsa_len(p, b) : 0;
    }
    __device__ void next(const DsaIndexParams& p) {
        if (++t == p.ntile) {
            t = 0;
            ++b;
            L = b < p.B ? dsa_len(p, b) : 0;
        }
    }
};

__global__ void __launch_bounds__(kIdxThreads, 2)
dsa_index_kernel(const DsaIndexParams p, const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k) {
    extern __shared__ __align__(1024) uint8_t dsmem[];
    if (smem_u32(dsmem) & 1023u) {
        if (threadIdx.x == 0) record_error(HCA_ERR_INTERNAL);
        return;
    }
    uint8_t* sm = dsmem;
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kIdxSmBar);
    uint64_t* empty = full + kIdxRing;
    uint64_t* q_full = empty + kIdxRing;       // [2]
    uint64_t* q_empty = q_full + 2;            // [2]
    uint64_t* acc_full = q_full + 4;           // [2]
    uint64_t* acc_empty = q_full + 6;          // [2]
    uint64_t* drain = q_full + 8;
    int* misc = reinterpret_cast<int*>(sm + kIdxSmW + 2 * kDsaMaxHI * 4);
    volatile int* abort_flag = misc;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 1);
    float* wsm = reinterpret_cast<float*>(sm + kIdxSmW);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int i = 0; i < kIdxRing; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], 1);
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 4);
        }
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, 128);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // this CTA's contiguous range of (sequence, tile) pairs
    const long long per = (p.total + gridDim.x - 1) / gridDim.x;
    const long long t_begin = per * blockIdx.x;
    const long long t_end = min(p.total, t_begin + per);

    if (warp == 0) {
        if (lane == 0) {
            uint32_t op = 0, nq = 0;
            int cur_b = -1;
            bool ok = true;
            DsaTileWalk wk(p, t_begin);
            for (long long i = t_begin; ok && i < t_end; ++i, wk.next(p)) {
                const int b = wk.b, t = wk.t;
                if (128 * t >= wk.L) continue;                    // past the sequence: no keys to read
                if (b != cur_b) {
                    const uint32_t qb = nq & 1;
                    if (!mbar_wait(&q_empty[qb], ((nq >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(&q_full[qb], (uint32_t)p.HI * 128);
                    tma_load_4d(sm + kIdxSmQ + qb * kIdxQBytes, &tm_q, &q_full[qb], 0, 0, b, 0);
                    ++nq;
                    cur_b = b;
                }
                const uint32_t st = op % kIdxRing;
                if (!mbar_wait(&empty[st], ((op / kIdxRing) & 1) ^ 1, abort_flag)) { ok = false; break; }
                mbar_arrive_expect_tx(&full[st], kIdxSlab);
                tma_load_4d(sm + kIdxSmRing + st * kIdxSlab, &tm_k, &full[st], 0, 128 * t, b, 0);
                ++op;
            }
            mbar_drain_ring(full, op, kIdxRing);
            // the last query load has landed too (it was consumed unless a wait gave up)
            if (nq) mbar_drain_wait(&q_full[(nq - 1) & 1], ((nq - 1) >> 1) & 1);
        }
    } else if (warp == 1) {
        const uint32_t id = idesc_bf16(128, p.HI, 0, 0);
        uint32_t op = 0, nq = 0, na = 0;
        int cur_b = -1;
        bool ok = true;
        DsaTileWalk wk(p, t_begin);
        for (long long i = t_begin; ok && i < t_end; ++i, wk.next(p)) {
            const int b = wk.b, t = wk.t;
            if (128 * t >= wk.L) continue;
            if (b != cur_b) {
                if (cur_b >= 0 && lane == 0) mma_commit(&q_empty[(nq - 1) & 1]);   // previous query buffer free
                if (!warp_wait(&q_full[nq & 1], (nq >> 1) & 1, abort_flag)) { ok = false; break; }
                ++nq;
                cur_b = b;
            }
            const uint32_t st = op % kIdxRing, ab = na & 1;
            if (!warp_wait(&acc_empty[ab], ((na >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
            if (!warp_wait(&full[st], (op / kIdxRing) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t a = smem_u32(sm + kIdxSmRing + st * kIdxSlab);
                const uint32_t q = smem_u32(sm + kIdxSmQ + ((nq - 1) & 1) * kIdxQBytes);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ss(tmem + 64 * ab, smem_desc_sw128(a + kk * 32, 16, 1024), smem_desc_sw128(q + kk * 32, 16, 1024), id,
                           kk ? 1u : 0u);
                mma_commit(&empty[st]);
                mma_commit(&acc_full[ab]);
            }
            __syncwarp();
            ++op;
            ++na;
        }
        if (lane == 0) {
            mma_commit(drain);
            mbar_drain_wait(drain, 0);
        }
        __syncwarp();
    } else {
        // ================================================================ epilogue: thread = position
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        const int et = threadIdx.x - 64;          // 0..127
        uint32_t na = 0, nb = 0;
        int cur_b = -1;
        DsaTileWalk wk(p, t_begin);
        for (long long i = t_begin; i < t_end; ++i, wk.next(p)) {
            const int b = wk.b, t = wk.t;
            const int L = wk.L;
            const int pos = 128 * t + r;
            if (128 * t >= L) {
                if (pos < p.Lmax) p.scores[(size_t)b * p.Lmax + pos] = -INFINITY;
                continue;
            }
            if (b != cur_b) {
                // the sequence's head weights, in the other of two buffers
                float* wb = wsm + (nb & 1) * kDsaMaxHI;
                if (et < p.HI) wb[et] = __ldg(p.w + (size_t)b * p.HI + et);
                asm volatile("bar.sync 1, 128;" ::: "memory");
                ++nb;
                cur_b = b;
            }
            const float* wb = wsm + ((nb - 1) & 1) * kDsaMaxHI;
            const uint32_t ab = na & 1;
            if (!dsa_group_wait128(&acc_full[ab], (na >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            float s = 0.f;
            for (int c0 = 0; c0 < p.HI; c0 += 16) {
                float v[16];
                tmem_ld16(tmem + lane_off + 64 * ab + c0, v);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) s = fmaf(wb[c0 + j], fmaxf(v[j], 0.f), s);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[ab]);
            ++na;
            if (pos < p.Lmax) p.scores[(size_t)b * p.Lmax + pos] = pos < L ? s : -INFINITY;
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

// ------------------------------------------------------------------------------------- top-k

constexpr int kTopkThreads = 1024;

struct DsaTopkParams {
    const float* scores;     // [B, Lmax]
    const int* seqlens;
    int* idx;                // [B, k]
    int B, Lmax, k;
};

// Order-preserving integer image of an fp32 score: larger scores give larger keys, equal
// scores equal keys (-0 is taken as +0, as the two compare equal).
__device__ __forceinline__ uint32_t dsa_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive scan of one int per thread (1024 threads); returns the exclusive prefix
// and the block total through *total.
__device__ __forceinline__ int dsa_block_scan(int v, int* wsum, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += n;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = wsum[lane];
        int y = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, y, off);
            if (lane >= off) y += n;
        }
        wsum[lane] = y - w;                 // exclusive prefix of the warp totals
        if (lane == 31) wsum[32] = y;
    }
    __syncthreads();
    const int r = wsum[warp] + x - v;
    *total = wsum[32];
    __syncthreads();
    return r;
}

constexpr int kTopkCluster = 4;            // CTAs per sequence, each over a quarter of the positions

__device__ __forceinline__ void dsa_cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t dsa_mapa(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
__device__ __forceinline__ int dsa_ld_cluster(uint32_t a) {
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ void dsa_st_cluster(uint32_t a, int v) {
    asm volatile("st.shared::cluster.s32 [%0], %1;" :: "r"(a), "r"(v) : "memory");
}

// A cluster of kTopkCluster CTAs per sequence (two CTAs per SM, so that 64 sequences run in one
// wave): each builds the digit histograms of its quarter of the positions, rank 0 adds the four
// through distributed shared memory and picks the digit, each CTA counts its keys above the
// digit from its own histogram, and in the last pass each CTA writes the kept positions of its
// quarter after those of the ranks before it.
__global__ void __launch_bounds__(kTopkThreads, 2) dsa_topk_kernel(const DsaTopkParams p) {
    __shared__ int hist[2048];
    __shared__ int wsum[33];
    __shared__ int sel[2];                  // [0] digit chosen, [1] remaining after the pass
    __shared__ int counts[2 * kTopkCluster];   // rank 0: each rank's larger / equal key counts
    uint32_t rank;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
    const int b = blockIdx.x / kTopkCluster;
    int L = __ldg(p.seqlens + b);
    L = L < 0 ? 0 : (L > p.Lmax ? p.Lmax : L);
    const float* sc = p.scores + (size_t)b * p.Lmax;
    int* out = p.idx + (size_t)b * p.k;
    const int kk = min(p.k, L);
    const int tid = threadIdx.x, lane = tid & 31;
    // this CTA's quarter of the positions (a multiple of 4 long, for 16-byte loads)
    const int qsize = (((L + kTopkCluster - 1) / kTopkCluster) + 3) & ~3;
    const int q0 = min(L, (int)rank * qsize), q1 = min(L, q0 + qsize);
    uint32_t prefix = 0, pmask = 0;
    int remaining = kk;                     // how many of the largest keys still to place
    int n_gt_q = 0, n_eq_q = 0;             // this quarter's keys above / equal to the threshold
    const bool vec = ((reinterpret_cast<uintptr_t>(sc) & 15u) == 0);
    auto load4 = [&](int s, float* f) {
        if (vec && s + 3 < q1) {
            const float4 x = __ldg(reinterpret_cast<const float4*>(sc + s));
            f[0] = x.x; f[1] = x.y; f[2] = x.z; f[3] = x.w;
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) f[e] = s + e < q1 ? __ldg(sc + s + e) : -INFINITY;
        }
    };
    if (kk < L) {
        // three digit passes, most significant first: 11, 11 and 10 bits
        for (int pass = 0; pass < 3; ++pass) {
            const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
            const int nbins = pass == 2 ? 1024 : 2048;
            for (int i = tid; i < 2048; i += kTopkThreads) hist[i] = 0;
            __syncthreads();
            for (int base = q0; base < q1; base += 4 * kTopkThreads) {
                const int s = base + 4 * tid;
                float f[4];
                load4(s, f);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t key = dsa_key(f[e]);
                    const bool in = s + e < q1 && (key & pmask) == prefix;
                    const uint32_t bin = (key >> shift) & (uint32_t)(nbins - 1);
                    // warp-aggregated increments: lanes with the same bin add once
                    const uint32_t act = __ballot_sync(0xffffffffu, in);
                    if (in) {
                        const uint32_t peers = __match_any_sync(act, bin);
                        if ((__ffs(peers) - 1) == lane) atomicAdd(&hist[bin], __popc(peers));
                    }
                }
            }
            dsa_cluster_sync();             // every quarter's histogram is complete
            if (rank == 0) {
                // the digit holding the remaining-th largest key: suffix sums over the bins of the
                // four histograms, high to low (thread i takes bins 2i and 2i + 1 from the top)
                const int hi_bin = nbins - 1 - 2 * tid;
                int c0 = 0, c1 = 0;
                for (int r = 0; r < kTopkCluster; ++r) {
                    if (2 * tid < nbins) c0 += dsa_ld_cluster(dsa_mapa(&hist[hi_bin], r));
                    if (2 * tid + 1 < nbins) c1 += dsa_ld_cluster(dsa_mapa(&hist[hi_bin - 1], r));
                }
                int tot;
                const int before = dsa_block_scan(c0 + c1, wsum, &tot);     // keys in higher bins
                int dig = -1, rem = 0;
                if (2 * tid < nbins) {
                    if (before < remaining && before + c0 >= remaining) {
                        dig = hi_bin;
                        rem = remaining - before;
                    } else if (2 * tid + 1 < nbins && before + c0 < remaining && before + c0 + c1 >= remaining) {
                        dig = hi_bin - 1;
                        rem = remaining - before - c0;
                    }
                }
                if (dig >= 0)
                    for (int r = 0; r < kTopkCluster; ++r) {
                        dsa_st_cluster(dsa_mapa(&sel[0], r), dig);
                        dsa_st_cluster(dsa_mapa(&sel[1], r), rem);
                    }
            }
            dsa_cluster_sync();             // the digit is known everywhere; rank 0 is done reading
            prefix |= (uint32_t)sel[0] << shift;
            pmask |= (uint32_t)(nbins - 1) << shift;
            remaining = sel[1];
            // this quarter's keys in bins above the chosen digit are all kept: their count, from its
            // own histogram (the scan's barriers end the reads before the next pass clears it)
            {
                int c = 0;
                for (int bin = sel[0] + 1 + tid; bin < nbins; bin += kTopkThreads) c += hist[bin];
                if (pass == 2) n_eq_q = hist[sel[0]];
                int t;
                dsa_block_scan(c, wsum, &t);
                n_gt_q += t;
            }
        }
    }
    // keep every key above the threshold key `prefix` and the first `remaining` keys equal to it,
    // in position order.  With all positions kept the passes are skipped (prefix = 0, remaining =
    // kk = L): every key is at least 0, so every position is kept.  Each quarter's output starts
    // after the kept positions of the quarters before it, from the ranks' counts.
    // with every position kept (no passes), all count as above the threshold
    int tot = kk < L ? n_gt_q : q1 - q0;
    const int tot_eq_q = kk < L ? n_eq_q : 0;
    if (tid == 0) {
        dsa_st_cluster(dsa_mapa(&counts[2 * rank], 0), tot);
        dsa_st_cluster(dsa_mapa(&counts[2 * rank + 1], 0), tot_eq_q);
    }
    dsa_cluster_sync();
    int gt_pre = 0, eq_pre = 0;
    for (uint32_t r = 0; r < rank; ++r) {
        gt_pre += dsa_ld_cluster(dsa_mapa(&counts[2 * r], 0));
        eq_pre += dsa_ld_cluster(dsa_mapa(&counts[2 * r + 1], 0));
    }
    int o_base = gt_pre + max(0, min(eq_pre, remaining)), eq_seen = eq_pre;
    for (int base = q0; base < q1; base += 4 * kTopkThreads) {
        const int s = base + 4 * tid;
        float f[4];
        load4(s, f);
        uint32_t key[4];
        int ng = 0, ne = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            key[e] = dsa_key(f[e]);
            const bool live = s + e < q1;
            ng += live && key[e] > prefix;
            ne += live && key[e] == prefix;
        }
        const int pre = dsa_block_scan(ng + (ne << 16), wsum, &tot);
        const int gt_before = pre & 0xffff;
        int eq_before = eq_seen + (pre >> 16);
        int o = o_base + gt_before + max(0, min(eq_before - eq_seen, remaining - eq_seen));
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (s + e >= q1) break;
            if (key[e] > prefix) {
                out[o++] = s + e;
            } else if (key[e] == prefix) {
                if (eq_before < remaining) out[o++] = s + e;
                ++eq_before;
            }
        }
        const int tot_gt = tot & 0xffff, tot_eq = tot >> 16;
        o_base += tot_gt + max(0, min(tot_eq, remaining - eq_seen));
        eq_seen += tot_eq;
    }
    if (rank == 0)
        for (int i = kk + tid; i < p.k; i += kTopkThreads) out[i] = -1;
    dsa_cluster_sync();                     // rank 0's counts stay readable until every rank is done
}

// ------------------------------------------------------------------------------------- attention

constexpr int kAttThreads = 288;           // MMA issuer, 4 softmax warps, 4 gather warps
constexpr uint32_t kAttSlab = 128 * 128;   // 128 rows x 64 channels bf16
constexpr uint32_t kAttQSlab = 64 * 128;   // 64 heads x 64 channels
constexpr uint32_t kAttSmQ = 0;                                  // 4 x 8 KB
constexpr uint32_t kAttSmK = kAttSmQ + 4 * kAttQSlab;            // 4 x 16 KB
constexpr uint32_t kAttSmV = kAttSmK + 4 * kAttSlab;             // 4 x 16 KB
constexpr uint32_t kAttSmP = kAttSmV + 4 * kAttSlab;             // 128 keys x 64 heads bf16
constexpr uint32_t kAttSmRed = kAttSmP + kAttSlab;               // float [4][64]
constexpr uint32_t kAttSmM = kAttSmRed + 4 * 64 * 4;             // float [64] reference max
constexpr uint32_t kAttSmA = kAttSmM + 64 * 4;                   // float [64] rescale factors
constexpr uint32_t kAttSmL = kAttSmA + 64 * 4;                   // float4 [16][128] running sums
constexpr uint32_t kAttSmBar = kAttSmL + 16 * 128 * 16;
constexpr uint32_t kAttSmem = kAttSmBar + 16 * 8 + 32;
static_assert(kAttSmem <= 232448, "attention shared memory exceeds the per-block limit");
constexpr float kAttRescale = 8.0f;        // move the reference max only when exceeded by 2^8

struct DsaAttendParams {
    const __nv_bfloat16* k;  // [B, Lmax, 256]
    const __nv_bfloat16* v;
    const int* idx;          // [B, kmax] ascending, -1 padding
    const int* seqlens;
    float* out;              // [B, Hq, 256]
    int B, Hq, Lmax, kmax;
    int rows;                // rows of the key / value maps (B * Lmax): a row index past every row
    float scale_log2;
};

// Four rows of a 2-D map (one row high box of 64 bf16 channels, 128-byte swizzle) gathered into
// four consecutive 128-byte rows of a swizzled slab; completion counted in bytes on `bar`.  A row
// index past the map's rows reads zeros.
__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* m, uint64_t* bar, int x, int r0, int r1,
                                            int r2, int r3) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cta.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];"
        :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)),
           "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
        : "memory");
}

// Column reduction of 32 values per lane across a warp: returns, in lane c, the max (or sum)
// over the 32 lanes of column c (a butterfly that halves the columns kept at each step).
template <bool kMax>
__device__ __forceinline__ float dsa_colred32(float* t, int lane) {
#pragma unroll
    for (int x = 16; x >= 1; x >>= 1) {
        const bool hi = (lane & x) != 0;
#pragma unroll
        for (int i = 0; i < x; ++i) {
            const float send = hi ? t[i] : t[i + x];
            const float keep = hi ? t[i + x] : t[i];
            const float o = __shfl_xor_sync(0xffffffffu, send, x);
            t[i] = kMax ? fmaxf(keep, o) : keep + o;
        }
    }
    return t[0];
}

// The position of row 32 w + lane of kept-position tile jj (-1 past the tile count or the kept count).
__device__ __forceinline__ int dsa_tile_pos(const int* idx_b, int jj, int count, int w, int lane) {
    const int row = 128 * jj + 32 * w + lane;
    return row < count ? __ldg(idx_b + row) : -1;
}

// Rows 32 w .. 32 w + 31 of a 128-row tile of gathered 512-byte rows (lane l holds the position
// `mine` of row 32 w + l, in the sequence whose first map row is row0) into four 128-byte-swizzled
// slabs of 64 channels: lane l issues one gather4 of rows 32 w + 4 (l >> 2) .. + 3 for slab l & 3.
// Positions -1 and positions past Lmax (reported) read zeros (row index `oob`, past the map).
// The warp's 16 KB are announced on `bar` before any copy is issued.
__device__ __forceinline__ void dsa_gather_tile(uint8_t* dst, const CUtensorMap* m, uint64_t* bar, int row0,
                                                int mine, int Lmax, int oob, int w, int lane) {
    if (__any_sync(0xffffffffu, mine >= Lmax) && lane == 0) record_error(HCA_ERR_DEVICE_INPUT);
    const int row = (mine >= 0 && mine < Lmax) ? row0 + mine : oob;
    if (lane == 0) mbar_arrive_expect_tx(bar, 32 * 4 * 128);
    __syncwarp();
    const int g = lane >> 2, slab = lane & 3;
    const int r0 = __shfl_sync(0xffffffffu, row, 4 * g), r1 = __shfl_sync(0xffffffffu, row, 4 * g + 1);
    const int r2 = __shfl_sync(0xffffffffu, row, 4 * g + 2), r3 = __shfl_sync(0xffffffffu, row, 4 * g + 3);
    tma_gather4(dst + slab * kAttSlab + (32 * w + 4 * g) * 128, m, bar, 64 * slab, r0, r1, r2, r3);
}

__global__ void __launch_bounds__(kAttThreads, 1)
dsa_attend_kernel(const DsaAttendParams p, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
    extern __shared__ __align__(1024) uint8_t dsmem[];
    if (smem_u32(dsmem) & 1023u) {
        if (threadIdx.x == 0) record_error(HCA_ERR_INTERNAL);
        return;
    }
    uint8_t* sm = dsmem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kAttSmBar);
    uint64_t* q_full = bars + 0;
    uint64_t* k_full = bars + 1;        // 4 worker warps' gathers: the tile's key rows are in place
    uint64_t* s_full = bars + 2;        // S^T of the tile is in tensor memory (commit)
    uint64_t* s_read = bars + 3;        // 4 worker warps: S^T read
    uint64_t* p_full = bars + 4;        // 4 worker warps: P^T and the value rows are in place
    uint64_t* pv_done = bars + 5;       // O^T += V^T P^T done (commit)
    uint64_t* drain = bars + 6;
    uint64_t* v_full = bars + 7;        // 4 worker warps' gathers: the tile's value rows are in place
    int* misc = reinterpret_cast<int*>(sm + kAttSmBar + 16 * 8);
    volatile int* abort_flag = misc;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 1);
    float* red = reinterpret_cast<float*>(sm + kAttSmRed);
    float* mref = reinterpret_cast<float*>(sm + kAttSmM);
    float* alpha = reinterpret_cast<float*>(sm + kAttSmA);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // a cluster of two CTAs per sequence: rank 0 takes the first half of the kept tiles, rank 1
    // the rest; at the end they exchange partials and each merges and writes half the channels
    const int b = blockIdx.x >> 1;
    uint32_t rank;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
    int L = __ldg(p.seqlens + b);
    L = L < 0 ? 0 : (L > p.Lmax ? p.Lmax : L);
    const int count = min(p.kmax, L);
    const int nt_all = (count + 127) / 128;
    const int nt_first = (nt_all + 1) / 2;
    const int jt0 = rank ? nt_first : 0;                  // this CTA's first tile of the sequence
    const int nt = rank ? nt_all - nt_first : nt_first;   // and its number of tiles
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        mbar_init(q_full, 1);
        mbar_init(k_full, 4);
        mbar_init(s_full, 1);
        mbar_init(s_read, 4);
        mbar_init(p_full, 4);
        mbar_init(pv_done, 1);
        mbar_init(drain, 1);
        mbar_init(v_full, 4);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = 0, tO = 64;     // S^T: 64 columns; O^T: two chunks of 128 channels x 64 heads
    const int* idx_b = p.idx + (size_t)b * p.kmax;

    if (warp == 0) {
        // ================================================================ MMA issuer (+ query load)
        if (lane == 0 && nt > 0) {
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            mbar_arrive_expect_tx(q_full, 4 * kAttQSlab);
            for (int s = 0; s < 4; ++s) tma_load_4d(sm + kAttSmQ + s * kAttQSlab, &tm_q, q_full, 64 * s, 0, b, 0);
        }
        const uint32_t id_s = idesc_bf16(128, kDsaHeads, 0, 0);
        const uint32_t id_o = idesc_bf16(128, kDsaHeads, 1, 1);
        bool ok = nt == 0 || warp_wait(q_full, 0, abort_flag);
        for (int j = 0; ok && j < nt; ++j) {
            if (!warp_wait(k_full, j & 1, abort_flag)) { ok = false; break; }
            if (j > 0 && !warp_wait(s_read, (j - 1) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t kb = smem_u32(sm + kAttSmK), qb = smem_u32(sm + kAttSmQ);
#pragma unroll
                for (int s = 0; s < 4; ++s)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ss(tmem + tS, smem_desc_sw128(kb + s * kAttSlab + kk * 32, 16, 1024),
                               smem_desc_sw128(qb + s * kAttQSlab + kk * 32, 16, 1024), id_s, (s | kk) ? 1u : 0u);
                mma_commit(s_full);
            }
            __syncwarp();
            if (!warp_wait(p_full, j & 1, abort_flag)) { ok = false; break; }
            if (!warp_wait(v_full, j & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t vb = smem_u32(sm + kAttSmV), pb = smem_u32(sm + kAttSmP);
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss(tmem + tO + 64 * c, smem_desc_sw128(vb + 2 * c * kAttSlab + kk * 2048, kAttSlab, 1024),
                               smem_desc_sw128(pb + kk * 2048, 8192, 1024), id_o, (j | kk) ? 1u : 0u);
                mma_commit(pv_done);
            }
            __syncwarp();
        }
        if (lane == 0) {
            mma_commit(drain);
            mbar_drain_wait(drain, 0);
        }
        __syncwarp();
    } else if (warp >= 5) {
        // ================================================================ gathers
        // warp 5 + w fetches rows 32 w .. 32 w + 31 of every tile: the keys of tile j + 1 as soon
        // as S^T of tile j is in tensor memory, the values of tile j once PV of tile j - 1 is done
        const int w = warp - 5;
        const int row0 = b * p.Lmax;    // the sequence's first row in the key / value maps
        int k_issued = 0, v_issued = 0;
        // each tile's positions are loaded one tile ahead of their key gather (the value gather
        // of the same tile reuses them)
        int cur = nt > 0 ? dsa_tile_pos(idx_b, jt0, count, w, lane) : -1;
        if (nt > 0) {
            dsa_gather_tile(sm + kAttSmK, &tm_k, k_full, row0, cur, p.Lmax, p.rows, w, lane);
            k_issued = 1;
        }
        for (int j = 0; j < nt; ++j) {
            const int nxt = j + 1 < nt ? dsa_tile_pos(idx_b, jt0 + j + 1, count, w, lane) : -1;
            if (j > 0 && !warp_wait(pv_done, (j - 1) & 1, abort_flag)) break;
            dsa_gather_tile(sm + kAttSmV, &tm_v, v_full, row0, cur, p.Lmax, p.rows, w, lane);
            ++v_issued;
            if (j + 1 < nt) {
                if (!warp_wait(s_full, j & 1, abort_flag)) break;
                dsa_gather_tile(sm + kAttSmK, &tm_k, k_full, row0, nxt, p.Lmax, p.rows, w, lane);
                ++k_issued;
            }
            cur = nxt;
        }
        // gathers still in flight (after an abort) land before the buffers are reused or released
        if (lane == 0) {
            if (k_issued) mbar_drain_wait(k_full, (k_issued - 1) & 1);
            if (v_issued) mbar_drain_wait(v_full, (v_issued - 1) & 1);
        }
        __syncwarp();
    } else {
        // ================================================================ softmax, epilogue
        // a warp reaches only the TMEM lane quarter (warp id mod 4): rows / lanes 32 w .. 32 w + 31
        const int w = warp & 3;
        const int r = 32 * w + lane;
        const uint32_t lane_off = (uint32_t)(32 * w) << 16;
        // this thread's running softmax sums of heads 4 i .. 4 i + 3 at lsum[128 i + r] (shared
        // memory, consecutive threads on consecutive 16-byte words)
        float4* lsum = reinterpret_cast<float4*>(sm + kAttSmL);
#pragma unroll
        for (int i = 0; i < 16; ++i) lsum[128 * i + r] = make_float4(0.f, 0.f, 0.f, 0.f);
        bool ok = true;
        for (int j = 0; ok && j < nt; ++j) {
            const int nvalid = count - 128 * (jt0 + j);
            if (!dsa_group_wait128(s_full, j & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            float z[64];
#pragma unroll
            for (int c = 0; c < 64; c += 16) tmem_ld16(tmem + lane_off + tS + c, z + c);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_read);
            const bool valid = r < nvalid;
#pragma unroll
            for (int h = 0; h < 64; ++h) z[h] = valid ? z[h] * p.scale_log2 : -INFINITY;
            // tile max per head over the 128 rows, then the reference max (moved lazily)
            {
                float t[32];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) t[i] = z[32 * half + i];
                    red[w * 64 + 32 * half + lane] = dsa_colred32<true>(t, lane);
                }
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (threadIdx.x >= 32 && threadIdx.x < 96) {
                const int h = threadIdx.x - 32;
                const float tm = fmaxf(fmaxf(red[h], red[64 + h]), fmaxf(red[128 + h], red[192 + h]));
                const float mo = j == 0 ? -INFINITY : mref[h];
                if (j == 0 || tm > mo + kAttRescale) {
                    alpha[h] = j == 0 ? 1.f : ex2(mo - tm);
                    mref[h] = tm;
                } else {
                    alpha[h] = 1.f;
                }
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            // PV of the previous tile done: O^T is stable and the P buffer free
            if (j > 0 && !dsa_group_wait128(pv_done, (j - 1) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            bool any = false;
            if (j > 0)
#pragma unroll
                for (int h = 0; h < 64; ++h) any |= alpha[h] != 1.f;
            if (any) {
                // O^T rows (channels 128 c + r) times alpha per head column; PV of the last tile is done
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float4 l = lsum[128 * i + r];
                    l.x *= alpha[4 * i]; l.y *= alpha[4 * i + 1]; l.z *= alpha[4 * i + 2]; l.w *= alpha[4 * i + 3];
                    lsum[128 * i + r] = l;
                }
#pragma unroll 1
                for (int c = 0; c < 2; ++c)
#pragma unroll 1
                    for (int c16 = 0; c16 < 64; c16 += 16) {
                        float o[16];
                        uint32_t wv[16];
                        const uint32_t ta = tmem + lane_off + tO + 64 * c + c16;
                        tmem_ld16(ta, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i) wv[i] = __float_as_uint(o[i] * alpha[c16 + i]);
                        tmem_st16(ta, wv);
                    }
                tmem_wait_st();
                tc_fence_before();
            }
            // probabilities: P^T row r (64 heads) in bf16, and this thread's share of the sums of
            // the same rounded values (numerator and normaliser use identical weights)
            uint32_t pk[32];
#pragma unroll
            for (int h = 0; h < 64; h += 2)
                pk[h >> 1] = pack_bf16x2(ex2(z[h] - mref[h]), ex2(z[h + 1] - mref[h + 1]));
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float4 l = lsum[128 * i + r];
                l.x += bf16lo(pk[2 * i]); l.y += bf16hi(pk[2 * i]);
                l.z += bf16lo(pk[2 * i + 1]); l.w += bf16hi(pk[2 * i + 1]);
                lsum[128 * i + r] = l;
            }
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4*>(sm + kAttSmP + dsa_sw(r, c)) =
                    make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            // P^T is written (the MMA issuer also waits for the value rows)
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        // the last PV is done before O^T is read
        if (ok && nt > 0 && !dsa_group_wait128(pv_done, (nt - 1) & 1, abort_flag)) ok = false;
        tc_fence_after();
        // ---- this CTA's softmax sums per head (column sums, then the 4 warps) and its max
        {
            float t[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 l = lsum[128 * (8 * half + i) + r];
                    t[4 * i] = l.x; t[4 * i + 1] = l.y; t[4 * i + 2] = l.z; t[4 * i + 3] = l.w;
                }
                red[w * 64 + 32 * half + lane] = dsa_colred32<false>(t, lane);
            }
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (threadIdx.x >= 32 && threadIdx.x < 96) {
            const int h = threadIdx.x - 32;
            alpha[h] = nt > 0 ? (red[h] + red[64 + h]) + (red[128 + h] + red[192 + h]) : 0.f;   // l
            if (nt == 0) mref[h] = -INFINITY;
        }
        if (threadIdx.x == 32) misc[2] = ok ? 1 : 0;
        tc_fence_before();
    }
    // ---- merge the two halves: out = (O0 2^(m0-M) + O1 2^(m1-M)) / (l0 2^(m0-M) + l1 2^(m1-M)).
    // Rank r writes the output channels 128 r .. 128 r + 127: each rank sends the other its
    // (max, sum, ok) and its O^T rows of the other's channel half, then both merge the same way.
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // neither rank reads its key / value buffers any more (its MMAs are drained): the peer may
    // write there
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    // the peer's O^T rows of this rank's channel half [128 ch][64 heads], each 256-byte row's
    // 16-byte chunks XOR-swizzled by the row's low four bits, so that 32 threads on 32
    // consecutive rows touch all banks; the peer's max [64], sum [64] and ok flag
    float* ox = reinterpret_cast<float*>(sm + kAttSmK);
    float* mlx = reinterpret_cast<float*>(sm + kAttSmV);
    if (warp >= 1 && warp <= 4) {
        const int w = warp & 3;
        const int r = 32 * w + lane;
        const uint32_t lane_off = (uint32_t)(32 * w) << 16;
        const uint32_t peer = rank ^ 1u;
        uint32_t ro, rml;
        asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ro) : "r"(smem_u32(ox)), "r"(peer));
        asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rml) : "r"(smem_u32(mlx)), "r"(peer));
        const uint32_t dst = ro + (uint32_t)(r * 256);
#pragma unroll 1
        for (int c16 = 0; c16 < 64; c16 += 16) {
            float o[16];
            if (nt > 0) {
                tmem_ld16(tmem + lane_off + tO + 64 * peer + c16, o);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) o[i] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < 16; i += 4)
                asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};"
                             :: "r"(dst + 16 * (((c16 + i) >> 2) ^ (r & 15))), "f"(o[i]), "f"(o[i + 1]),
                                "f"(o[i + 2]), "f"(o[i + 3]) : "memory");
        }
        if (threadIdx.x >= 32 && threadIdx.x < 96) {
            const int h = threadIdx.x - 32;
            asm volatile("st.shared::cluster.f32 [%0], %1;" :: "r"(rml + 4 * h), "f"(mref[h]) : "memory");
            asm volatile("st.shared::cluster.f32 [%0], %1;" :: "r"(rml + 256 + 4 * h), "f"(alpha[h]) : "memory");
        }
        if (threadIdx.x == 32)
            asm volatile("st.shared::cluster.f32 [%0], %1;" :: "r"(rml + 512), "f"(misc[2] ? 1.f : 0.f) : "memory");
        tc_fence_before();
    }
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    if (warp >= 1 && warp <= 4) {
        const int w = warp & 3;
        const int r = 32 * w + lane;
        const uint32_t lane_off = (uint32_t)(32 * w) << 16;
        tc_fence_after();
        if (threadIdx.x >= 32 && threadIdx.x < 96) {
            const int h = threadIdx.x - 32;
            // rank 0's and rank 1's (max, sum), whichever this rank is
            const float m0 = rank ? mlx[h] : mref[h], l0 = rank ? mlx[64 + h] : alpha[h];
            const float m1 = rank ? mref[h] : mlx[h], l1 = rank ? alpha[h] : mlx[64 + h];
            const float M = fmaxf(m0, m1);
            const float e0 = ex2(m0 - M), e1 = m1 == -INFINITY ? 0.f : ex2(m1 - M);
            const float inv = 1.f / (l0 * e0 + l1 * e1);
            const bool good = misc[2] && mlx[128] != 0.f;
            red[h] = good ? e0 * inv : NAN;          // weight of rank 0's O^T
            red[64 + h] = good ? e1 * inv : NAN;     // weight of rank 1's
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        float* ob = p.out + (size_t)b * p.Hq * kDsaD + 128 * rank + r;
#pragma unroll 1
        for (int c16 = 0; c16 < 64; c16 += 16) {
            float o[16];
            if (nt > 0) {
                tmem_ld16(tmem + lane_off + tO + 64 * rank + c16, o);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) o[i] = 0.f;
            }
            float x[16];
#pragma unroll
            for (int i = 0; i < 16; i += 4) {
                const float4 t = *reinterpret_cast<const float4*>(ox + r * 64 + 4 * (((c16 + i) >> 2) ^ (r & 15)));
                x[i] = t.x; x[i + 1] = t.y; x[i + 2] = t.z; x[i + 3] = t.w;
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int h = c16 + i;
                const float o0 = rank ? x[i] : o[i], o1 = rank ? o[i] : x[i];
                if (h < p.Hq) ob[(size_t)h * kDsaD] = fmaf(o0, red[h], o1 * red[64 + h]);
            }
        }
        tc_fence_before();
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

}  // namespace hca
