// decode.cuh -- split-KV HCA decode on tcgen05 tensor cores (sm_100a).
//
// One new query per sequence attends, in one softmax, to its n_c visible compressed
// entries and to its raw window of the last W tokens (official blog "ERNIE 5.5 Flash
// Base . ERNIE", section 2.1; Zhidx article, section "1. Latent-Gated Sparse
// Attention").  With 64 query heads sharing one KV head, every cached byte feeds 64
// heads, so the dot products run on the tensor cores and the kernel is bound by HBM.
//
// Work decomposition.  A unit is one (sequence, KV head) pair; its keys are cut into
// tiles of 128 (compressed tiles first, then window tiles).  All tiles of the batch are
// laid end to end and cut into one contiguous range per CTA (one CTA per SM), so ragged
// batches balance to within one tile.  A CTA may cover the tail of one unit and the
// head of the next; for each (CTA, unit) piece it writes a partial record (running max
// m, sum l, unnormalised O) into the workspace, and the combine kernel merges the
// records of each unit with a log-sum-exp and applies the optional output gate.
//
// Per tile, inside a CTA (warp-specialised):
//   warp 0 (1 thread)  TMA: K and V tiles as 16 KB slabs (128 keys x 64 channels, 128-byte
//                      swizzle) through ONE ring of 8 slots (slot s always holds channel
//                      slab s), in a fixed order in which K runs up to A tiles ahead of V
//                      (A = 4 S buffers, 2 with QK normalisation): K0 .. K(A-1), V0, KA,
//                      V1, K(A+1), ...  While the first tile's softmax runs, the next tiles'
//                      K streams at full rate into the whole ring instead of half of it;
//                      the query rows of each piece;
//   warp 1 (1 thread)  tcgen05.mma  S^T[128 keys x 64 heads] = K . Q^T into TMEM (and, with
//                      QK normalisation, diag(K K^T) for the key norms);
//   warp 2 (1 thread)  tcgen05.mma  O^T[512 ch x 64 heads] += V^T . P^T (TMEM, 4 x 128);
//   warps 3-10         softmax: thread = (key row, 32 of the 64 heads), two warps per TMEM
//                      lane quarter; per-head running max with lazy rescaling (only when a
//                      logit exceeds the max by 2^8), P^T in bf16 to shared memory (two
//                      buffers); each thread keeps its rows' running sums in registers, so the
//                      sums are reduced across threads once per piece, in the epilogue that
//                      writes the record.
// QK normalisation and paged caches are compile-time variants: the common path carries none of
// their code (instruction fetch, not arithmetic, bounds the softmax of a launch's first tile).
// Two MMA issuers keep QK^T of the next tiles from queueing behind PV of this one.
// Every mbarrier wait is bounded (see common.cuh).
#pragma once

#include "common.cuh"

namespace hca {

constexpr int kDecD = 512;                 // head dim (d == dv)
constexpr int kDecSlabs = kDecD / 64;      // 64-channel slabs per key row
constexpr int kDecTile = 128;              // keys per tile (MMA M of S^T)
constexpr int kDecHeads = 64;              // MMA N: query heads of one KV group (padded)
constexpr int kDecRing = 8;                // slab slots shared by K and V: slot s = channel slab s
constexpr int kDecLook = 4;                // S buffers: K tiles ahead of V (2 with QK normalisation)
constexpr int kDecLookNorm = 2;
constexpr int kDecPBufs = 2;               // P^T buffers
constexpr int kDecThreads = 352;           // 11 warps: TMA, QK^T MMA, PV MMA, 8 softmax
constexpr int kDecSoftWarp0 = 3;           // first softmax warp
constexpr int kDecSoftWarps = 8;
constexpr uint32_t kSlabBytes = 128 * 128;                 // 128 rows x 128 B
constexpr uint32_t kDecQBytes = kDecHeads * kDecD * 2;     // 64 KB
constexpr uint32_t kDecPBytes = kDecTile * kDecHeads * 2;  // 16 KB
constexpr float kRescaleThreshold = 8.0f;                  // log2 units

// TMEM columns
constexpr uint32_t kTmS = 0;      // S^T buffers 0, 1 (64 columns each)
constexpr uint32_t kTmO = 128;    // 4 x 64  O^T chunks (128 channels each)
constexpr uint32_t kTmS2 = 384;   // S^T buffers 2, 3 -- or, with QK normalisation,
constexpr uint32_t kTmKK = 384;   // 128     K K^T

__host__ __device__ constexpr uint32_t dec_s_col(int b) { return b < 2 ? kTmS + 64u * b : kTmS2 + 64u * (b - 2); }

// shared-memory layout (offsets from a 1024-aligned base)
constexpr uint32_t kSmQ = 0;
constexpr uint32_t kSmP = kSmQ + kDecQBytes;
constexpr uint32_t kSmRing = kSmP + kDecPBufs * kDecPBytes;
constexpr uint32_t kSmBar = kSmRing + kDecRing * kSlabBytes;
constexpr int kNumBars = 4 * kDecRing + 2 + 2 * kDecLook + 2 * kDecPBufs + 3;
constexpr uint32_t kSmRed = (kSmBar + kNumBars * 8 + 127) & ~127u;   // float[4][64] (read as float4)
constexpr uint32_t kSmFin = kSmRed + 4 * 64 * 4;            // float[64] reduction result
constexpr uint32_t kSmMax = kSmFin + 64 * 4;                // float[64] running max per head
constexpr uint32_t kSmAlpha = kSmMax + 64 * 4;              // float[64] rescale factors
constexpr uint32_t kSmSum = kSmAlpha + 64 * 4;              // float[64] running sum per head
constexpr uint32_t kSmMisc = kSmSum + 64 * 4;               // ints
constexpr uint32_t kDecSmemBytes = kSmMisc + 64;            // the dynamic base is checked to be 1024-aligned
static_assert(kDecSmemBytes <= 232448, "decode shared memory exceeds the 227 KB per-block limit");
static_assert(kSmRed % 16 == 0 && kSmFin % 16 == 0 && kSmMax % 16 == 0 && kSmAlpha % 16 == 0 &&
              kSmSum % 16 == 0 && kSmMisc % 16 == 0, "vector-accessed shared arrays must be 16-byte aligned");
static_assert(kSmP % 1024 == 0 && kSmRing % 1024 == 0, "swizzled operand tiles must be 1024-byte aligned");
static_assert(kDecRing == kDecSlabs, "one ring slot per channel slab: a tile op fills the whole ring");

struct DecodeParams {
    const __nv_bfloat16* q;      // [B, Hq, 512]
    const int* seqlens;          // [B]
    const int* page_table;       // [B, max_pages] or null
    const float* gq;             // [512] or null
    const float* gk;
    const __nv_bfloat16* gate;   // [B, Hq, 512] or null
    float* out;                  // [B, Hq, 512]
    long long* total;            // workspace header: total tiles of the batch
    int* meta;                   // [U][2]: first and last CTA holding a piece of unit u
    float* rec_m;                // [R][64]  running max (log2 units)
    float* rec_l;                // [R][64]
    float* rec_o;                // [R][64][512]
    const float* vha_u;          // [Hq, vha_r] Virtual Head Attention factors, or null
    const float* vha_v;
    int vha_r;
    int B, Hq, Hkv, G, blk, W, Nmax, page_size, max_pages, num_pages, flags, nsplit;
    float scale_log2, eps;
};

struct UnitTiles {
    int b, g, nc, nw, nct, nwt, s0;
};

// Visible entries and tiles of unit u.  Out-of-range lengths are clamped and reported.
__device__ __forceinline__ UnitTiles unit_tiles(const DecodeParams& p, int u, bool report) {
    UnitTiles t;
    t.b = u / p.Hkv;
    t.g = u - t.b * p.Hkv;
    int L = __ldg(p.seqlens + t.b);
    if (L < 1) {
        if (report) record_error(HCA_ERR_DEVICE_INPUT);
        L = 1;
    }
    const long long a = (long long)L - p.W;          // (t - W + 1) with t = L - 1
    long long nc = a > 0 ? a / p.blk : 0;
    const long long cap = (p.flags & HCA_PAGED) ? (long long)p.max_pages * p.page_size : (long long)p.Nmax;
    if (nc > cap) {
        if (report) record_error(HCA_ERR_DEVICE_INPUT);
        nc = cap;
    }
    t.nc = (int)nc;
    t.nw = L < p.W ? L : p.W;
    t.nct = (t.nc + kDecTile - 1) / kDecTile;
    t.nwt = (t.nw + kDecTile - 1) / kDecTile;
    // oldest-first window: the nw valid slots are the last ones; ring (slot = position % W):
    // before the ring wraps, positions 0 .. L-1 sit in slots 0 .. L-1
    t.s0 = (p.flags & HCA_WINDOW_RING) ? 0 : p.W - t.nw;
    return t;
}

// Block-wide (all threads) inclusive scan of one int per thread.
__device__ __forceinline__ int block_scan_incl(int v, int* warp_tot, int* total_out) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += n;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    int pre = 0, tot = 0;
    for (int w = 0; w < kDecThreads / 32; ++w) {
        if (w < warp) pre += warp_tot[w];
        tot += warp_tot[w];
    }
    __syncthreads();
    *total_out = tot;
    return v + pre;
}

// Named barrier among the 256 softmax threads.
__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ bool softmax_any(bool pred) {
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
                 "barrier.red.or.pred q, 2, 256, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r) : "r"((uint32_t)pred) : "memory");
    return r != 0;
}

// Wait by all 256 softmax threads with one verdict for the group (barrier.red.and), so
// the eight warps either all go on or all unwind -- their named barriers never strand a
// warp.
__device__ __forceinline__ bool group_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
    const bool ok = mbar_wait(bar, parity, abort);
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
                 "barrier.red.and.pred q, 3, 256, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r) : "r"((uint32_t)ok) : "memory");
    return r != 0;
}

// Warp reduce-scatter of a 32-vector held by every lane: lane l ends with the reduction (max
// or sum) of element l over the 32 lanes.  31 shuffles: at each step a lane keeps one half of
// its remaining elements and trades the other half with its partner.
template <bool kMax>
__device__ __forceinline__ float colreduce32(const float (&v)[32], int lane) {
    float t[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const bool hi = lane & 16;
        const float send = hi ? v[i] : v[i + 16];
        const float keep = hi ? v[i + 16] : v[i];
        const float o = __shfl_xor_sync(0xffffffffu, send, 16);
        t[i] = kMax ? fmaxf(keep, o) : keep + o;
    }
#pragma unroll
    for (int w = 16; w >= 2; w >>= 1) {
        const int hf = w / 2, x = w / 2;
        const bool hi = lane & x;
#pragma unroll
        for (int i = 0; i < hf; ++i) {
            const float send = hi ? t[i] : t[i + hf];
            const float keep = hi ? t[i + hf] : t[i];
            const float o = __shfl_xor_sync(0xffffffffu, send, x);
            t[i] = kMax ? fmaxf(keep, o) : keep + o;
        }
    }
    return t[0];
}

// Byte offset of 16-byte chunk `c` of row `r` in a 128-byte-swizzled slab.
__device__ __forceinline__ uint32_t sw128(uint32_t r, uint32_t c) {
    return r * 128u + (((c ^ r) & 7u) << 4);
}

// This CTA's tiles, in order: (unit u, tile index) pairs of the range [ts, te).
struct TileIter {
    const DecodeParams* p;
    long long te, pu;
    UnitTiles t;
    int u, ntiles, tb, tend, tile, item;
    bool done;

    __device__ void load_unit(long long from) {
        t = unit_tiles(*p, u, false);
        ntiles = t.nct + t.nwt;
        tb = (int)((from > pu ? from : pu) - pu);
        tend = (int)((te < pu + ntiles ? te : pu + ntiles) - pu);
        tile = tb;
    }
    __device__ void init(const DecodeParams* pp, int u0, long long p0, long long ts, long long te_) {
        p = pp;
        te = te_;
        u = u0;
        pu = p0;
        item = 0;
        done = u0 < 0 || ts >= te_;
        if (!done) load_unit(ts);
    }
    __device__ bool first() const { return tile == tb; }
    __device__ bool last() const { return tile == tend - 1; }
    __device__ bool comp() const { return tile < t.nct; }
    // keys of the current tile that belong to the sequence
    __device__ int nvalid() const {
        return comp() ? min(kDecTile, t.nc - tile * kDecTile)
                      : min(kDecTile, t.nw - (tile - t.nct) * kDecTile);     // slots s0 .. s0 + nw - 1
    }
    __device__ void next() {
        if (++tile < tend) return;
        ++item;
        pu += ntiles;
        ++u;
        if (pu >= te) {
            done = true;
            return;
        }
        load_unit(pu);
    }
};

__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

template <bool NORM, bool PAGED>
__global__ void __launch_bounds__(kDecThreads, 1)
decode_split_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_kw, const __grid_constant__ CUtensorMap tm_vw) {
    extern __shared__ __align__(1024) uint8_t dsmem[];
    // the swizzled operand tiles need a 1024-byte aligned base; there is no room for slack
    if (smem_u32(dsmem) & 1023u) {
        if (threadIdx.x == 0) record_error(HCA_ERR_INTERNAL);
        return;
    }
    uint8_t* sm = dsmem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kSmBar);
    // A slot's landed / consumed barriers come in a K and a V copy: each consumer then sees only
    // its own ops, in order, so a phase-parity wait is never two phases ahead of the barrier.
    uint64_t* full_k = bars;                       // [kDecRing] K slab landed
    uint64_t* full_v = full_k + kDecRing;          // [kDecRing] V slab landed
    uint64_t* empty_k = full_v + kDecRing;         // [kDecRing] K slab consumed (QK^T issued and done)
    uint64_t* empty_v = empty_k + kDecRing;        // [kDecRing] V slab consumed (PV issued and done)
    uint64_t* q_full = empty_v + kDecRing;
    uint64_t* q_empty = q_full + 1;
    uint64_t* s_full = q_full + 2;                 // [kDecLook]
    uint64_t* s_empty = s_full + kDecLook;         // [kDecLook]
    uint64_t* p_full = s_empty + kDecLook;         // [kDecPBufs]
    uint64_t* p_empty = p_full + kDecPBufs;        // [kDecPBufs]
    uint64_t* o_full = p_empty + kDecPBufs;
    uint64_t* o_empty = o_full + 1;
    uint64_t* q_tma = o_full + 2;                  // query slabs landed (TMA)
    float* red = reinterpret_cast<float*>(sm + kSmRed);
    float* fin = reinterpret_cast<float*>(sm + kSmFin);
    float* m_s = reinterpret_cast<float*>(sm + kSmMax);
    float* al_s = reinterpret_cast<float*>(sm + kSmAlpha);
    float* l_s = reinterpret_cast<float*>(sm + kSmSum);
    int* misc = reinterpret_cast<int*>(sm + kSmMisc);
    volatile int* abort_flag = misc + 0;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 1);
    int* sched = misc + 2;          // [0] = first unit, [2..8] scan scratch

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr bool norm = NORM;
    constexpr bool paged = PAGED;
    const int U = p.B * p.Hkv;
    const int cta = blockIdx.x;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int i = 0; i < kDecRing; ++i) {
            mbar_init(&full_k[i], 1);
            mbar_init(&full_v[i], 1);
            mbar_init(&empty_k[i], 1);
            mbar_init(&empty_v[i], 1);
        }
        mbar_init(q_full, kDecSoftWarps);
        mbar_init(q_empty, 1);
        for (int i = 0; i < kDecLook; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_empty[i], kDecSoftWarps);
        }
        for (int i = 0; i < kDecPBufs; ++i) {
            mbar_init(&p_full[i], kDecSoftWarps);
            mbar_init(&p_empty[i], 1);
        }
        mbar_init(o_full, 1);
        mbar_init(o_empty, kDecSoftWarps);
        mbar_init(q_tma, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, 512);
    if (threadIdx.x == 32) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_kw);
        prefetch_tmap(&tm_vw);
    }

    // ---- this CTA's tile range [ts, te) of the batch, and the unit holding tile ts.
    // With at most one unit per thread, each thread reads its unit's length once.
    const bool small_batch = U <= kDecThreads;
    int my_n = 0;
    if (small_batch && threadIdx.x < U) {
        UnitTiles t = unit_tiles(p, threadIdx.x, true);
        my_n = t.nct + t.nwt;
    }
    long long total = 0;
    if (small_batch) {
        total = my_n;
    } else {
        for (int u = threadIdx.x; u < U; u += kDecThreads) {
            UnitTiles t = unit_tiles(p, u, true);
            total += t.nct + t.nwt;
        }
    }
    {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) total += __shfl_xor_sync(0xffffffffu, total, off);
        long long* wt = reinterpret_cast<long long*>(red);
        if (lane == 0) wt[warp] = total;
        __syncthreads();
        total = 0;
        for (int w = 0; w < kDecThreads / 32; ++w) total += wt[w];
        __syncthreads();
    }
    // Two ways to cut the batch's tiles into one range per CTA (tpc = ceil(total / nsplit)):
    //  - unit-aligned, when the batch has no more units than CTAs: unit u gets
    //    k_u = clamp(max(floor(tiles_u * nsplit / total), ceil(tiles_u / T)), 1, tiles_u) CTAs
    //    and its tiles are split evenly among them, for the smallest T in tpc .. tpc + 3 whose
    //    counts fit the grid.  Every CTA then holds exactly one piece (no second query load,
    //    record and pipeline refill inside a CTA) of at most T tiles;
    //  - otherwise (no such T: a ragged batch whose long units cannot be cut finely enough)
    //    equal ranges of tpc tiles (the last CTAs may get fewer or none); a range may hold the
    //    tail of one unit and the head of the next.
    const long long tpc = (total + p.nsplit - 1) / p.nsplit;
    long long* sched64 = reinterpret_cast<long long*>(red + 64);   // [0] ts, [1] te, [2] p_first
    // the four candidate counts are summed in one reduction, as 16-bit fields of a 64-bit
    // word: k_u <= nsplit * tiles_u / total + 1, so each sum is at most nsplit + U < 2^16
    unsigned long long* wsum = reinterpret_cast<unsigned long long*>(red);   // [warp]
    int my_k = 0;
    bool aligned = false;
    if (small_batch && U <= p.nsplit && p.nsplit < 0x8000 && total > 0 && total <= 0x3fffffffll) {
        const unsigned n32 = (unsigned)my_n;
        const unsigned fl = threadIdx.x < U ? (unsigned)((long long)my_n * p.nsplit / total) : 0u;
        unsigned long long packed = 0;
        if (threadIdx.x < U)
#pragma unroll 1
            for (unsigned w = 0; w < 4; ++w) {
                const unsigned T = (unsigned)tpc + w;
                packed |= (unsigned long long)max(1u, min(n32, max(fl, (n32 + T - 1u) / T))) << (16 * w);
            }
        unsigned long long sum = packed;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane == 0) wsum[warp] = sum;
        __syncthreads();
        sum = 0;
        for (int v = 0; v < kDecThreads / 32; ++v) sum += wsum[v];
        __syncthreads();
        for (int w = 3; w >= 0; --w)
            if ((int)((sum >> (16 * w)) & 0xffffu) <= p.nsplit) {
                aligned = true;
                my_k = (int)((packed >> (16 * w)) & 0xffffu);
            }
    }
    if (threadIdx.x == 0) {
        sched[0] = -1;
        sched64[0] = aligned ? 0 : min(total, tpc * cta);
        sched64[1] = aligned ? 0 : min(total, tpc * (cta + 1));
    }
    __syncthreads();
    if (aligned) {
        // the unit whose block of CTAs holds this CTA (block-wide scans over units, one
        // unit per thread)
        int tot_t, tot_c;
        const int incl_t = block_scan_incl(my_n, sched + 2, &tot_t);
        const int incl_c = block_scan_incl(my_k, sched + 2, &tot_c);
        const long long pu = incl_t - my_n;
        const int cu = incl_c - my_k;
        if (threadIdx.x < U && cu <= cta && cta < cu + my_k) {
            const int i = cta - cu;
            sched[0] = threadIdx.x;
            sched64[2] = pu;
            sched64[0] = pu + (long long)my_n * i / my_k;
            sched64[1] = pu + (long long)my_n * (i + 1) / my_k;
        }
        __syncthreads();
    } else {
        // the unit holding tile ts (block-wide scan over units)
        const long long ts0 = sched64[0];
        long long base = 0;
        for (int c0 = 0; c0 < U; c0 += kDecThreads) {
            const int u = c0 + threadIdx.x;
            int n = 0;
            if (small_batch) {
                n = my_n;
            } else if (u < U) {
                UnitTiles t = unit_tiles(p, u, false);
                n = t.nct + t.nwt;
            }
            int tot;
            const int incl = block_scan_incl(n, sched + 2, &tot);
            const long long pu = base + incl - n;
            if (u < U && pu <= ts0 && ts0 < pu + n) {
                sched[0] = u;
                sched64[2] = pu;
            }
            base += tot;
        }
        __syncthreads();
    }
    const long long ts = sched64[0];
    const long long te = sched64[1];
    if (cta == 0 && threadIdx.x == 0) *p.total = total;
    const int u_first = sched[0];
    const long long p_first = sched64[2];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const bool have_work = (ts < te) && u_first >= 0;

    // K tiles in flight ahead of V (the S buffers the softmax has not read yet)
    const int look = norm ? kDecLookNorm : kDecLook;
    if (have_work && warp == 0) {
        // ===================================================== TMA producer (one thread)
        if (lane == 0) {
            TileIter ki, vi;
            ki.init(&p, u_first, p_first, ts, te);
            vi.init(&p, u_first, p_first, ts, te);
            int kn = 0, vn = 0, qitem = 0;
            int last = -1;      // kind of the previous op (every op fills all slots): 0 K, 1 V
            // test switch (hca_debug_set_drop_slab): the first K slab is never requested
            bool drop = *reinterpret_cast<volatile int*>(&g_debug_drop_slab) != 0;
            // Page ids of the two 64-entry halves of the current compressed K (V) tile, read
            // from the page table once per tile, as soon as the iterator reaches the tile (the
            // previous op's slabs are still in flight, so the load's latency hides behind
            // them).  A page id outside the pool is reported and clamped into it, so every
            // load stays inside the pool.
            int kpg[2] = {0, 0}, vpg[2] = {0, 0};
            auto pages_of = [&](const TileIter& it, int* pg) {
                if (!paged || it.done || !it.comp()) return;
                const int j0 = it.tile * kDecTile;
                const int* row = p.page_table + (size_t)it.t.b * p.max_pages;
                pg[0] = __ldg(row + j0 / p.page_size);
                pg[1] = j0 + 64 < it.t.nc ? __ldg(row + (j0 + 64) / p.page_size) : pg[0];
                if (min(pg[0], pg[1]) < 0 || max(pg[0], pg[1]) >= p.num_pages) {
                    record_error(HCA_ERR_DEVICE_INPUT);
                    pg[0] = min(max(pg[0], 0), p.num_pages - 1);
                    pg[1] = min(max(pg[1], 0), p.num_pages - 1);
                }
            };
            pages_of(ki, kpg);
            pages_of(vi, vpg);
            // One slab of the current tile of iterator `it` (K or V) into slot `s`.
            auto issue = [&](const TileIter& it, const int* pg, int s, bool is_v) {
                uint8_t* dst = sm + kSmRing + s * kSlabBytes;
                uint64_t* bar = is_v ? &full_v[s] : &full_k[s];
                const CUtensorMap* m = it.comp() ? (is_v ? &tm_v : &tm_k) : (is_v ? &tm_vw : &tm_kw);
                if (it.comp() && paged) {
                    const int j0 = it.tile * kDecTile;
                    const bool h1 = j0 + 64 < it.t.nc;
                    mbar_arrive_expect_tx(bar, h1 ? 2 * 8192 : 8192);
                    for (int h = 0; h < (h1 ? 2 : 1); ++h)
                        tma_load_4d(dst + h * 8192, m, bar, 64 * s, it.t.g, (j0 + 64 * h) % p.page_size, pg[h]);
                } else {
                    mbar_arrive_expect_tx(bar, kSlabBytes);
                    const int row = it.comp() ? it.tile * kDecTile : it.t.s0 + (it.tile - it.t.nct) * kDecTile;
                    tma_load_4d(dst, m, bar, 64 * s, it.t.g, row, it.t.b);
                }
            };
            while (!ki.done || !vi.done) {
                // K runs up to `look` tiles ahead of V, but a piece's first K waits until every
                // V of the previous piece is out
                const bool do_k = !ki.done && kn < vn + look && (!ki.first() || vn == kn);
                if (do_k && ki.first()) {
                    // the piece's 64 query rows (heads g*G ..), eight 8 KB slabs, once the
                    // previous piece's QK^T no longer reads them
                    if (!mbar_wait(q_empty, (qitem & 1) ^ 1, abort_flag)) break;
                    mbar_arrive_expect_tx(q_tma, kDecQBytes);
                    for (int s = 0; s < kDecSlabs; ++s)
                        tma_load_4d(sm + kSmQ + s * 8192, &tm_q, q_tma, 64 * s, ki.t.g * p.G, ki.t.b, 0);
                    ++qitem;
                }
                bool ok = true;
                for (int s = 0; s < kDecSlabs; ++s) {
                    // the slot is free once the previous op in it (every op fills all slots) has
                    // been consumed; all ops before that one were consumed before it was issued
                    if (last >= 0 && !mbar_wait(last ? &empty_v[s] : &empty_k[s],
                                                (uint32_t)((last ? vn : kn) - 1) & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (drop) {
                        drop = false;
                        continue;
                    }
                    if (do_k) issue(ki, kpg, s, false);
                    else issue(vi, vpg, s, true);
                }
                if (!ok) break;
                last = do_k ? 0 : 1;
                if (do_k) {
                    ki.next();
                    pages_of(ki, kpg);
                    ++kn;
                } else {
                    vi.next();
                    pages_of(vi, vpg);
                    ++vn;
                }
            }
        }
    } else if (have_work && warp == 1) {
        // ===================================================== QK^T issuer (warp waits, lane 0 issues)
        const uint32_t id_s = idesc_bf16(128, kDecHeads, 0, 0);
        const uint32_t id_kk = idesc_bf16(128, 128, 0, 0);
        const uint32_t q_base = smem_u32(sm + kSmQ);
        TileIter it;
        it.init(&p, u_first, p_first, ts, te);
        int n = 0;
        while (!it.done) {
            const int sb = n % look;
            const uint32_t sph = (uint32_t)(n / look) & 1u;
            if (it.first() && !warp_wait(q_full, it.item & 1, abort_flag)) break;
            if (!warp_wait(&s_empty[sb], sph ^ 1u, abort_flag)) break;
            // the K K^T accumulator has one buffer: wait until tile n-1's softmax has read it
            if (norm && n > 0 &&
                !warp_wait(&s_empty[(n - 1) % look], (uint32_t)((n - 1) / look) & 1u, abort_flag))
                break;
            tc_fence_after();
            bool ok = true;
            for (int s = 0; s < kDecSlabs; ++s) {
                if (!warp_wait(&full_k[s], (uint32_t)n & 1u, abort_flag)) { ok = false; break; }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t k_base = smem_u32(sm + kSmRing + s * kSlabBytes);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = smem_desc_sw128(k_base + kk * 32, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(q_base + s * 8192 + kk * 32, 16, 1024);
                        mma_ss(tmem + dec_s_col(sb), ad, bd, id_s, (s | kk) ? 1u : 0u);
                        if (norm) mma_ss(tmem + kTmKK, ad, ad, id_kk, (s | kk) ? 1u : 0u);
                    }
                    mma_commit(&empty_k[s]);
                }
                __syncwarp();
            }
            if (!ok) break;
            if (lane == 0) {
                mma_commit(&s_full[sb]);
                if (it.last()) mma_commit(q_empty);
            }
            __syncwarp();
            ++n;
            it.next();
        }
    } else if (have_work && warp == 2) {
        // ===================================================== PV issuer (warp waits, lane 0 issues)
        const uint32_t id_o = idesc_bf16(128, kDecHeads, 1, 1);
        TileIter it;
        it.init(&p, u_first, p_first, ts, te);
        int n = 0;
        while (!it.done) {
            const int b = n % kDecPBufs;
            if (!warp_wait(&p_full[b], (n / kDecPBufs) & 1, abort_flag)) break;
            if (it.first() && !warp_wait(o_empty, (it.item & 1) ^ 1, abort_flag)) break;
            tc_fence_after();
            const int nvalid = it.nvalid();
            const bool partial = nvalid < kDecTile;
            const uint32_t p_base = smem_u32(sm + kSmP + b * kDecPBytes);
            bool ok = true;
            for (int c = 0; c < 4; ++c) {
                const int st0 = 2 * c, st1 = 2 * c + 1;
                if (!warp_wait(&full_v[st0], (uint32_t)n & 1u, abort_flag) ||
                    !warp_wait(&full_v[st1], (uint32_t)n & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                if (partial) {
                    // rows >= nvalid may hold anything (caller memory past the visible
                    // entries, or ring slots not yet written): zero them so 0-probability keys
                    // contribute exactly 0
                    const int nz = (kDecTile - nvalid) * 8;
                    for (int i = lane; i < 2 * nz; i += 32) {
                        const int sl = i / nz, k = i - sl * nz;
                        const int r = nvalid + (k >> 3);
                        uint8_t* slab = sm + kSmRing + (sl ? st1 : st0) * kSlabBytes;
                        *reinterpret_cast<uint4*>(slab + r * 128 + (k & 7) * 16) = make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t v_base = smem_u32(sm + kSmRing + st0 * kSlabBytes);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint64_t ad = smem_desc_sw128(v_base + kk * 2048, kSlabBytes, 1024);
                        const uint64_t bd = smem_desc_sw128(p_base + kk * 2048, 8192, 1024);
                        mma_ss(tmem + kTmO + 64 * c, ad, bd, id_o, (it.first() && kk == 0) ? 0u : 1u);
                    }
                    mma_commit(&empty_v[st0]);
                    mma_commit(&empty_v[st1]);
                }
                __syncwarp();
            }
            if (!ok) break;
            if (lane == 0) {
                mma_commit(&p_empty[b]);
                if (it.last()) mma_commit(o_full);
            }
            __syncwarp();
            ++n;
            it.next();
        }
    } else if (have_work && warp >= kDecSoftWarp0) {
        // ===================================================== softmax / epilogue (8 warps)
        // Two warps per TMEM lane quarter; each owns 32 of the 64 heads of the quarter's 32 key
        // rows (a thread holds one key row's 32 logits).
        const int q4 = warp & 3;                             // TMEM lane quarter
        const int hh = (warp - kDecSoftWarp0) >> 2;          // head half: heads 32*hh .. 32*hh + 31
        const int h0 = 32 * hh;
        const int r = q4 * 32 + lane;            // key row within the tile / channel within a chunk
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        const int sidx = threadIdx.x - 32 * kDecSoftWarp0;   // 0..255
        TileIter it;
        it.init(&p, u_first, p_first, ts, te);
        int n = 0;
        bool ok = true;
        // this thread's share of the running row sums: sum over its key rows of p, per head
        float lsum[32];
#pragma unroll
        for (int h = 0; h < 32; ++h) lsum[h] = 0.f;
        while (ok && !it.done) {
            const bool first = it.first(), last = it.last();
            if (first) {
                // ---- the piece's queries arrive by TMA; with QK normalisation they are
                // rewritten in place as q' = q / rms(q) * g_q * g_k (bf16), since
                // q_hat . k_hat = (q' . k) / rms(k)
                if (!group_wait(q_tma, it.item & 1, abort_flag)) { ok = false; break; }
                if (NORM) {
                    const int h = sidx >> 2, part = sidx & 3;      // 4 threads per head, 128 channels each
                    float ss = 0.f;
#pragma unroll 1
                    for (int c = 0; c < 128; c += 8) {
                        const int cc = 128 * part + c;
                        const uint4 x = *reinterpret_cast<const uint4*>(sm + kSmQ + (cc >> 6) * 8192 +
                                                                      sw128(h, (cc & 63) >> 3));
                        const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float a = bf16lo(w4[i]), b2 = bf16hi(w4[i]);
                            ss = fmaf(a, a, fmaf(b2, b2, ss));
                        }
                    }
                    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
                    const float inv = rsqrtf(ss * (1.f / kDecD) + p.eps);
#pragma unroll 1
                    for (int c = 0; c < 128; c += 8) {
                        const int cc = 128 * part + c;
                        uint4* ptr =
                            reinterpret_cast<uint4*>(sm + kSmQ + (cc >> 6) * 8192 + sw128(h, (cc & 63) >> 3));
                        const uint4 x = *ptr;
                        uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int ch = cc + 2 * i;
                            const float a = bf16lo(w4[i]) * inv * __ldg(p.gq + ch) * __ldg(p.gk + ch);
                            const float b2 = bf16hi(w4[i]) * inv * __ldg(p.gq + ch + 1) * __ldg(p.gk + ch + 1);
                            w4[i] = pack_bf16x2(a, b2);
                        }
                        *ptr = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(q_full);
            }

            const int sb = n % look;
            const bool valid = r < it.nvalid();
            if (!group_wait(&s_full[sb], (n / look) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            float z[32];
            tmem_ld16(tmem + lane_off + dec_s_col(sb) + h0, z);
            tmem_ld16(tmem + lane_off + dec_s_col(sb) + h0 + 16, z + 16);
            float kscale = p.scale_log2;
            if (NORM) {
                float d[32];
                tmem_ld16(tmem + lane_off + kTmKK + q4 * 32, d);
                tmem_ld16(tmem + lane_off + kTmKK + q4 * 32 + 16, d + 16);
                tmem_wait_ld();
                float diag = 0.f;
#pragma unroll
                for (int j = 0; j < 32; ++j) diag = (j == lane) ? d[j] : diag;
                kscale *= rsqrtf(diag * (1.f / kDecD) + p.eps);
            } else {
                tmem_wait_ld();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty[sb]);
#pragma unroll
            for (int h = 0; h < 32; ++h) z[h] = valid ? z[h] * kscale : -INFINITY;

            // ---- running max (shared m_s[64]): full reduction on the first tile of a
            // piece; afterwards only when some logit exceeds the max by 2^threshold
            bool need;
            if (first) {
                need = true;
            } else {
                bool mine = false;
#pragma unroll
                for (int h = 0; h < 32; h += 4) {
                    const float4 mm = *reinterpret_cast<const float4*>(m_s + h0 + h);
                    mine |= (z[h] > mm.x + kRescaleThreshold) | (z[h + 1] > mm.y + kRescaleThreshold) |
                            (z[h + 2] > mm.z + kRescaleThreshold) | (z[h + 3] > mm.w + kRescaleThreshold);
                }
                need = softmax_any(mine);
            }
            if (need) {
                const float tmax = colreduce32<true>(z, lane);    // max of head h0 + lane over this warp's rows
                red[q4 * 64 + h0 + lane] = tmax;
                softmax_bar();
                if (sidx < 64) {
                    const float mo = first ? -INFINITY : m_s[sidx];
                    const float mn = fmaxf(mo, fmaxf(fmaxf(red[sidx], red[64 + sidx]), fmaxf(red[128 + sidx], red[192 + sidx])));
                    al_s[sidx] = first ? 0.f : ex2(mo - mn);
                    m_s[sidx] = mn;
                }
                softmax_bar();
                if (!first) {
#pragma unroll
                    for (int h = 0; h < 32; ++h) lsum[h] *= al_s[h0 + h];
                    // rescale O^T (this warp's 32 head columns of each chunk) once the previous
                    // PV has landed
                    const int pb = (n - 1) % kDecPBufs;
                    if (!group_wait(&p_empty[pb], ((n - 1) / kDecPBufs) & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
#pragma unroll 1
                        for (int c16 = 0; c16 < 32; c16 += 16) {
                            float o[16];
                            const uint32_t ta = tmem + lane_off + kTmO + 64 * c + h0 + c16;
                            tmem_ld16(ta, o);
                            tmem_wait_ld();
                            uint32_t w[16];
#pragma unroll
                            for (int j = 0; j < 16; ++j) w[j] = __float_as_uint(o[j] * al_s[h0 + c16 + j]);
                            tmem_st16(ta, w);
                        }
                    }
                    tmem_wait_st();
                    tc_fence_before();
                }
            }
            // ---- probabilities (and this thread's row sums)
            uint32_t pk[16];
#pragma unroll
            for (int h = 0; h < 32; h += 4) {
                const float4 mm = *reinterpret_cast<const float4*>(m_s + h0 + h);
                z[h] = ex2(z[h] - mm.x);
                z[h + 1] = ex2(z[h + 1] - mm.y);
                z[h + 2] = ex2(z[h + 2] - mm.z);
                z[h + 3] = ex2(z[h + 3] - mm.w);
                lsum[h] += z[h];
                lsum[h + 1] += z[h + 1];
                lsum[h + 2] += z[h + 2];
                lsum[h + 3] += z[h + 3];
                pk[h >> 1] = pack_bf16x2(z[h], z[h + 1]);
                pk[(h >> 1) + 1] = pack_bf16x2(z[h + 2], z[h + 3]);
            }
            const int pbuf = n % kDecPBufs;
            if (!group_wait(&p_empty[pbuf], ((n / kDecPBufs) & 1) ^ 1, abort_flag)) { ok = false; break; }
            uint8_t* pt = sm + kSmP + pbuf * kDecPBytes;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                *reinterpret_cast<uint4*>(pt + sw128(r, 4 * hh + c)) =
                    make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[pbuf]);

            if (last) {
                // ---- end of this CTA's piece of unit u: the row sums over all key rows, then the
                // record (running max, sum, unnormalised O^T)
                const int u = it.u;
                const int rec = cta + u;
                const float tsum = colreduce32<false>(lsum, lane);
                red[q4 * 64 + h0 + lane] = tsum;
                softmax_bar();
                if (sidx == 0) {
                    if (it.tb == 0) p.meta[2 * u] = cta;
                    if (it.tend == it.ntiles) p.meta[2 * u + 1] = cta;
                }
                if (sidx < 64) {
                    p.rec_m[(size_t)rec * 64 + sidx] = m_s[sidx];
                    p.rec_l[(size_t)rec * 64 + sidx] = (red[sidx] + red[64 + sidx]) + (red[128 + sidx] + red[192 + sidx]);
                }
                softmax_bar();     // red[] is free again before the next piece's first reduction
#pragma unroll
                for (int h = 0; h < 32; ++h) lsum[h] = 0.f;
                if (!group_wait(o_full, it.item & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                float* orec = p.rec_o + (size_t)rec * 64 * kDecD;
                // rolled: the code of a launch's last tile is fetched cold, and a smaller loop
                // costs less fetch than the unrolling saves
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
#pragma unroll 1
                    for (int c16 = 0; c16 < 32; c16 += 16) {
                        float o[16];
                        tmem_ld16(tmem + lane_off + kTmO + 64 * c + h0 + c16, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int h = h0 + c16 + j;
                            if (h < p.G) orec[(size_t)h * kDecD + 128 * c + r] = o[j];
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(o_empty);
            }
            ++n;
            it.next();
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

// Merge the partial records of each unit (log-sum-exp), normalise, apply the gate, and mix the
// heads with Virtual Head Attention when factors are given.
//
// Grid (units, dv / 32), 128 threads: a CTA owns all G heads of one unit for 32 channels, so
// the cross-head VHA mixing happens on chip.  Thread = (head h = tid / 2, 16 channels).  All
// the (m, l, O) values of a chunk of kChunk records are loaded before any is used, so a merge
// of up to kChunk pieces costs one memory round trip after the unit's range is known.  The
// gate logits and the VHA factors are inputs, not products of the split kernel: they are read
// before griddepcontrol.wait, while the split kernel still runs.  The VHA variant keeps the
// factors, the merged outputs and V^T o in dynamic shared memory (combine_vha_smem bytes).
constexpr int kMergeCh = 32;              // channels per combine CTA
constexpr int kDecVhaMaxRank = 32;        // fused VHA rank limit

__host__ __device__ constexpr uint32_t combine_vha_smem(int r) {
    return (uint32_t)(2 * kDecHeads * r + kDecHeads * kMergeCh + r * kMergeCh) * 4u;
}

template <int kChunk, bool kVha>
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeParams p) {
    extern __shared__ float cs[];
    const int u = blockIdx.x;
    const int h = threadIdx.x >> 1;
    const int c16 = 16 * (threadIdx.x & 1);
    const int c = blockIdx.y * kMergeCh + c16;                      // channels c .. c+15
    const int b = u / p.Hkv, g = u - (u / p.Hkv) * p.Hkv;
    const bool live = h < p.G;
    const size_t orow = ((size_t)b * p.Hq + (size_t)g * p.G + (live ? h : 0)) * kDecD + c;
    const bool gated = (p.flags & HCA_OUT_GATE) != 0;
    const int R = p.vha_r;
    float* os = cs;                                   // [64][32] merged, gated outputs (16-byte rows)
    float* ts = os + kDecHeads * kMergeCh;            // [R][32]  V^T o
    float* vs = ts + R * kMergeCh;                    // [G][R]
    float* us = vs + kDecHeads * R;                   // [G][R]
    uint4 graw[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
    if (gated && live) {
        graw[0] = __ldg(reinterpret_cast<const uint4*>(p.gate + orow));
        graw[1] = __ldg(reinterpret_cast<const uint4*>(p.gate + orow) + 1);
    }
    if (kVha) {
        for (int i = threadIdx.x; i < p.G * R; i += 128) {
            vs[i] = __ldg(p.vha_v + i);
            us[i] = __ldg(p.vha_u + i);
        }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (*reinterpret_cast<volatile unsigned int*>(&g_error) == HCA_ERR_TIMEOUT) {
        // a split CTA gave up: its records (and the unit ranges) may be stale, so the outputs are
        // marked invalid rather than merged from whatever the workspace holds
        if (live)
            for (int j = 0; j < 4; ++j)
                *reinterpret_cast<float4*>(p.out + orow + 4 * j) = make_float4(NAN, NAN, NAN, NAN);
        return;
    }
    const int first = __ldg(p.meta + 2 * u), last = __ldg(p.meta + 2 * u + 1);
    if (first < 0 || last < first || last >= p.nsplit) {
        if (threadIdx.x == 0 && blockIdx.y == 0) record_error(HCA_ERR_DEVICE_INPUT);
        return;
    }
    float M = -INFINITY, L = 0.f;
    float acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0.f;
    const int hh = live ? h : 0;
    for (int i0 = first; i0 <= last; i0 += kChunk) {
        float m[kChunk], l[kChunk];
        float4 o[kChunk][4];
#pragma unroll
        for (int k = 0; k < kChunk; ++k) {
            const bool ok = live && i0 + k <= last;   // ranges are contiguous: every CTA in between has a piece
            const size_t rec = (size_t)(i0 + k + u);
            m[k] = ok ? __ldcg(p.rec_m + rec * 64 + hh) : -INFINITY;
            l[k] = ok ? __ldcg(p.rec_l + rec * 64 + hh) : 0.f;
            const float4* op = reinterpret_cast<const float4*>(p.rec_o + (rec * 64 + hh) * kDecD + c);
#pragma unroll
            for (int j = 0; j < 4; ++j) o[k][j] = ok ? __ldcg(op + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float Mn = M;
#pragma unroll
        for (int k = 0; k < kChunk; ++k) Mn = fmaxf(Mn, m[k]);
        if (Mn == -INFINITY) continue;
        const float sc = M == -INFINITY ? 0.f : exp2f(M - Mn);
        L *= sc;
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[j] *= sc;
#pragma unroll
        for (int k = 0; k < kChunk; ++k) {
            const float w = m[k] == -INFINITY ? 0.f : exp2f(m[k] - Mn);
            L = fmaf(w, l[k], L);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                acc[4 * j] = fmaf(w, o[k][j].x, acc[4 * j]);
                acc[4 * j + 1] = fmaf(w, o[k][j].y, acc[4 * j + 1]);
                acc[4 * j + 2] = fmaf(w, o[k][j].z, acc[4 * j + 2]);
                acc[4 * j + 3] = fmaf(w, o[k][j].w, acc[4 * j + 3]);
            }
        }
        M = Mn;
    }
    const float inv = 1.f / L;
    float r[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) r[j] = acc[j] * inv;
    if (gated) {
        const uint32_t gw[8] = {graw[0].x, graw[0].y, graw[0].z, graw[0].w, graw[1].x, graw[1].y, graw[1].z, graw[1].w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            r[2 * j] *= __frcp_rn(1.f + __expf(-bf16lo(gw[j])));
            r[2 * j + 1] *= __frcp_rn(1.f + __expf(-bf16hi(gw[j])));
        }
    }
    if (kVha) {
        // o'[:, ch] = o[:, ch] + U (V^T o[:, ch]) over the G heads of this token.  Thread i of
        // the V^T o step owns rank k = i / 8 and channels 4 (i % 8) .. +3: a warp reads one 128-byte
        // row of os per head (broadcast to its four ranks) and four V values (broadcast).
        if (live) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                *reinterpret_cast<float4*>(os + h * kMergeCh + c16 + 4 * j) =
                    make_float4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
        } else if (h < kDecHeads) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                *reinterpret_cast<float4*>(os + h * kMergeCh + c16 + 4 * j) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        __syncthreads();
        for (int i = threadIdx.x; i < R * (kMergeCh / 4); i += 128) {
            const int k = i >> 3, c4 = (i & 7) * 4;
            float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
            for (int hd = 0; hd < p.G; ++hd) {
                const float vk = vs[hd * R + k];
                const float4 o4 = *reinterpret_cast<const float4*>(os + hd * kMergeCh + c4);
                t.x = fmaf(vk, o4.x, t.x);
                t.y = fmaf(vk, o4.y, t.y);
                t.z = fmaf(vk, o4.z, t.z);
                t.w = fmaf(vk, o4.w, t.w);
            }
            *reinterpret_cast<float4*>(ts + k * kMergeCh + c4) = t;
        }
        __syncthreads();
        if (live) {
            for (int k = 0; k < R; ++k) {
                const float uk = us[h * R + k];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float4 t4 = *reinterpret_cast<const float4*>(ts + k * kMergeCh + c16 + 4 * j);
                    r[4 * j] = fmaf(uk, t4.x, r[4 * j]);
                    r[4 * j + 1] = fmaf(uk, t4.y, r[4 * j + 1]);
                    r[4 * j + 2] = fmaf(uk, t4.z, r[4 * j + 2]);
                    r[4 * j + 3] = fmaf(uk, t4.w, r[4 * j + 3]);
                }
            }
        }
    }
    if (live) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
            *reinterpret_cast<float4*>(p.out + orow + 4 * j) = make_float4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
    }
}

}  // namespace hca
