// backward.cuh -- gradients of the HCA layer (sm_100a): dq, the raw dk / dv (through the window
// and through the pooling) and the pooling weights' dw.
//
// The layer (official blog "ERNIE 5.5 Flash Base . ERNIE", section 2.1): every 128 tokens are
// pooled into one cached entry, Kc[j] = sum_i alpha_i K[blk j + i] with alpha = softmax of the
// block's weights (Vc likewise), and each query attends, in one softmax, to the entries
// j < n_c(t) and to the raw window t-W+1 .. t.  With P the softmax, O the output and dO the
// incoming gradient, the textbook attention backward is
//     D = rowsum(dO * O),  dP = dO V^T,  dS = P * (dP - D),
//     dq = scale dS K,  dkeys = scale dS^T q,  dvals = P^T dO,
// and the pooling hands dKc / dVc back to the raw rows: dK_i += alpha_i dKc, dV_i += alpha_i dVc,
// dw_i = alpha_i (dalpha_i - sum_i' alpha_i' dalpha_i'), dalpha_i = K_i . dKc + V_i . dVc.
// The stored cache is bf16; its rounding has no gradient (the entries are taken as stored).
//
// Work unit: a row tile of 128 (token, head) rows -- tpt = 128 / G tokens times the G query heads
// of one KV head -- against a key tile of 128 keys: entries 128 j .. of the cache, or raw tokens
// 128 kt .. (tiles aligned to multiples of 128, so that both kernels below name the same tiles).
// A 512-dim head makes one key tile's dK and dV accumulators (2 x 128 x 512 fp32) twice the
// tensor memory of an SM, so P and dS are formed once and kept in global memory instead of being
// recomputed per accumulator:
//   bwd_pre_kernel  D for every (token, head) row (one warp per row); clears the accumulators.
//   bwd_dq_kernel   one CTA per row tile.  Phase S: per key tile, S = Q K^T and dP = dO V^T into
//                   one of two tensor-memory buffers (the MMAs of the next tile overlap the
//                   softmax of this one); eight softmax warps form P and dS in bf16 and write the
//                   pair to the tile's record (64 KB, the operand layout of the tensor cores).
//                   Phase A: dq = scale sum_j dS_j K_j, all 512 channels in tensor memory, dS
//                   read back from the records just written (L2).
//   bwd_dkv_kernel  one CTA per (key tile, dV or dK, range of row tiles): dV = sum P^T dO or
//                   dK = scale sum dS^T Q from the records, 512 channels in tensor memory, added
//                   with fp32 atomics into the entries' gradients (workspace) or the raw keys'.
//   bwd_pool_kernel one CTA per (sequence, block): pooling backward into dk, dv and dw.
// The records of a segment of row tiles are written by one dq launch and read by the dk/dv launch
// that follows, which bounds the workspace; the host walks the segments.  Operands stream through
// a ring of six 32 KB slots; the MMA issuer consumes ops in the producer's order.  Every wait is
// bounded (common.cuh).
#pragma once

#include "common.cuh"

namespace hca {

constexpr int kBwdD = 512;
constexpr int kDqThreads = 320;             // producer, MMA issuer, 8 softmax / epilogue warps
constexpr int kKvThreads = 192;             // producer, MMA issuer, 4 epilogue warps
constexpr int kBwdRing = 6;
constexpr uint32_t kBwdSlab = 16384;         // 128 rows x 64 columns bf16, 128-byte swizzle
constexpr uint32_t kBwdSlot = 2 * kBwdSlab;  // two slabs
constexpr uint32_t kBwdRec = 2 * kBwdSlot;   // one (row tile, key tile) record: P, then dS
constexpr uint32_t kBwdSmRing = 0;
constexpr uint32_t kBwdSmStage = kBwdSmRing + kBwdRing * kBwdSlot;   // 4 KB per softmax / epilogue warp
constexpr uint32_t kBwdStageBytes = 4096;
constexpr uint32_t kBwdSmBar = kBwdSmStage + 8 * kBwdStageBytes;
constexpr int kBwdNumBars = 2 * kBwdRing + 12;
constexpr uint32_t kBwdSmMisc = kBwdSmBar + kBwdNumBars * 8;
constexpr uint32_t kBwdSmem = kBwdSmMisc + 16;
static_assert(kBwdSmem <= 232448, "backward shared memory exceeds the per-block limit");
static_assert(kBwdSlot % 1024 == 0, "swizzled operands 1024-aligned");

struct BwdParams {
    const float* lse;             // [B, Hq, T] natural log
    float* drow;                  // [B, T, Hq] D = rowsum(dO * O)
    const void* out;              // [B, T, Hq, 512] fp32 or bf16 (forward output)
    const __nv_bfloat16* dout;    // [B, T, Hq, 512]
    const __nv_bfloat16* k;       // [B, T, Hkv, 512] raw
    const __nv_bfloat16* v;
    const float* w;               // [B, T] or null
    float* dq;                    // [B, T, Hq, 512]
    float* dk;                    // [B, T, Hkv, 512]
    float* dv;
    float* dkc;                   // [B, Nc, Hkv, 512] (workspace)
    float* dvc;
    float* dw;                    // [B, T]
    uint8_t* rec;                 // [B, Hkv, seg, nt_max] records of kBwdRec bytes (workspace)
    int B, T, Hq, Hkv, G, tpt, blk, W, Nc, ntile_t, out_f32;
    int nkc, nkw, nt_max, seg;    // compressed / raw key tiles; record slots per row tile; segment
    int s0, s1;                   // this launch's segment of row tiles
    long long dq_items;           // B * Hkv * (s1 - s0)
    int ch_rows, nch;             // dk/dv: row tiles per chunk of a compressed key tile, chunks
    int kta, nraw;                // dk/dv: first raw key tile touching the segment, their count
    long long kv_items;
    float scale, scale_log2;
};

__device__ __forceinline__ int bwd_visible(int t, int W, int blk) {
    const int a = t - W + 1;
    return a > 0 ? a / blk : 0;
}

// Row tile rt of (b, g): rows (token t0 + r / G, head g G + r % G); its key tiles j < nct are the
// entry tiles, then raw tiles kw0, kw0 + 1, .. (128-aligned) covering the window of every token.
struct BwdRows {
    int t0, tlast, nct, wlo, kw0, nt;
};

__device__ __forceinline__ BwdRows bwd_rows(const BwdParams& p, int rt) {
    BwdRows it;
    it.t0 = rt * p.tpt;
    it.tlast = min(it.t0 + p.tpt, p.T) - 1;
    it.nct = (bwd_visible(it.tlast, p.W, p.blk) + 127) / 128;
    it.wlo = max(0, it.t0 - p.W + 1);
    it.kw0 = it.wlo / 128;
    it.nt = it.nct + it.tlast / 128 - it.kw0 + 1;
    return it;
}

__device__ __forceinline__ uint8_t* bwd_record(const BwdParams& p, int b, int g, int rt, int j) {
    return p.rec + ((((size_t)b * p.Hkv + g) * p.seg + (rt - p.s0)) * p.nt_max + j) * (size_t)kBwdRec;
}

// Named barrier among the softmax / epilogue warps (n threads).
template <int n>
__device__ __forceinline__ void bwd_bar() { asm volatile("bar.sync 1, %0;" :: "n"(n) : "memory"); }

template <int n>
__device__ __forceinline__ bool bwd_group_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
    const bool ok = mbar_wait(bar, parity, abort);
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
                 "barrier.red.and.pred q, 2, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r) : "r"((uint32_t)ok), "n"(n) : "memory");
    return r != 0;
}

// Byte offset of 16-byte chunk c of row r in a 128-byte-swizzled slab.
__device__ __forceinline__ uint32_t bwd_sw(uint32_t r, uint32_t c) { return r * 128u + (((c ^ r) & 7u) << 4); }

// A warp's 32 rows x 128 bytes of a record (rows 32 q .. 32 q + 31 of a slab: 4 KB, contiguous in
// the record), lane = row: written through the warp's staging buffer so that every global store
// instruction covers four whole 128-byte lines (a store per lane and row would touch 32 lines).
// v holds the row's eight 16-byte chunks in column order; the record keeps the slab's swizzle.
__device__ __forceinline__ void bwd_warp_rows_out(uint8_t* stg, uint8_t* dst, const uint32_t* v, int lane) {
#pragma unroll
    for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(stg + bwd_sw(lane, c)) = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i)
        *reinterpret_cast<uint4*>(dst + i * 512 + lane * 16) = *reinterpret_cast<const uint4*>(stg + i * 512 + lane * 16);
    __syncwarp();
}

// 32 consecutive fp32 channels of each of a warp's 32 rows (lane = row, v = its 32 values) to
// row-major global rows, through the staging buffer: lane l then writes 16 bytes of row
// 4 i + l / 8, so each instruction covers four whole 128-byte lines.  row_ptr(i) gives the
// destination of the warp's row i (null: skip the row); kAtomic adds with fp32 vector atomics.
template <bool kAtomic, class RowPtr>
__device__ __forceinline__ void bwd_warp_f32_out(uint8_t* stg, const float* v, int lane, RowPtr row_ptr) {
#pragma unroll
    for (int c = 0; c < 8; ++c)
        *reinterpret_cast<float4*>(stg + bwd_sw(lane, c)) = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
    __syncwarp();
    const int k = lane & 7;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int row = 4 * i + (lane >> 3);
        float* d = row_ptr(row);
        const float4 x = *reinterpret_cast<const float4*>(stg + bwd_sw(row, k));
        if (d) {
            if (kAtomic) atomicAdd(reinterpret_cast<float4*>(d + 4 * k), x);
            else *reinterpret_cast<float4*>(d + 4 * k) = x;
        }
    }
    __syncwarp();
}

// -------------------------------------------------------------------------------- D = rowsum(dO O)

// Also clears what the later kernels accumulate into: dk, dv, the entries' dKc / dVc and dw.
__device__ __forceinline__ void bwd_zero(float* x, long long n) {
    float4* x4 = reinterpret_cast<float4*>(x);
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n / 4; i += (long long)gridDim.x * blockDim.x)
        x4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

__global__ void __launch_bounds__(256) bwd_pre_kernel(const BwdParams p) {
    const long long kv = (long long)p.B * p.T * p.Hkv * kBwdD, kvc = (long long)p.B * p.Nc * p.Hkv * kBwdD;
    bwd_zero(p.dk, kv);
    bwd_zero(p.dv, kv);
    if (kvc) {
        bwd_zero(p.dkc, kvc);
        bwd_zero(p.dvc, kvc);
    }
    if (p.dw)
        for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < (long long)p.B * p.T;
             i += (long long)gridDim.x * blockDim.x)
            p.dw[i] = 0.f;
    const long long rows = (long long)p.B * p.T * p.Hq;
    const int lane = threadIdx.x & 31;
    for (long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); row < rows; row += (long long)gridDim.x * 8) {
        const __nv_bfloat16* dr = p.dout + row * kBwdD;
        float s = 0.f;
        for (int c = 8 * lane; c < kBwdD; c += 256) {
            const uint4 g = __ldg(reinterpret_cast<const uint4*>(dr + c));
            const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
            float o[8];
            if (p.out_f32) {
                const float4* orow = reinterpret_cast<const float4*>(static_cast<const float*>(p.out) + row * kBwdD + c);
                const float4 a = __ldg(orow), b2 = __ldg(orow + 1);
                o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b2.x; o[5] = b2.y; o[6] = b2.z; o[7] = b2.w;
            } else {
                const uint4 ob = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.out) + row * kBwdD + c));
                const uint32_t ow[4] = {ob.x, ob.y, ob.z, ob.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    o[2 * i] = bf16lo(ow[i]);
                    o[2 * i + 1] = bf16hi(ow[i]);
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) s = fmaf(bf16lo(gw[i]), o[2 * i], fmaf(bf16hi(gw[i]), o[2 * i + 1], s));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) p.drow[row] = s;
    }
}

// One K-step (16 rows of the contraction, step kk) of D[:, 0:512] += A B, B being 512 channels held
// as four ops of two 64-channel blocks in ring slots op0 .. op0 + 3: a pair of ops in adjacent
// slots is one N = 256 operand (blocks 16 KB apart), otherwise two N = 128 operands.
__device__ __forceinline__ void bwd_mma_blocks(uint32_t tmem, uint64_t ad, uint32_t ring, uint32_t op0, int kk,
                                               uint32_t id_n128, uint32_t id_n256, uint32_t acc) {
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
        const uint32_t sa = (op0 + 2 * pr) % kBwdRing, sb = (op0 + 2 * pr + 1) % kBwdRing;
        const uint32_t ba = ring + sa * kBwdSlot + kk * 2048, bb = ring + sb * kBwdSlot + kk * 2048;
        if (sb == sa + 1) {
            mma_ss(tmem + 256 * pr, ad, smem_desc_sw128(ba, kBwdSlab, 1024), id_n256, acc);
        } else {
            mma_ss(tmem + 256 * pr, ad, smem_desc_sw128(ba, kBwdSlab, 1024), id_n128, acc);
            mma_ss(tmem + 256 * pr + 128, ad, smem_desc_sw128(bb, kBwdSlab, 1024), id_n128, acc);
        }
    }
}

// -------------------------------------------------------------------------------- dq

// Phase S ops of a key tile: 8 x (Q slab, K slab) for S, then 8 x (dO slab, V slab) for dP.
// Phase A ops of a key tile: its dS (32 KB from the record), then the key tile's 512 channels as
// four ops of two 64-channel blocks, the N = 128 B operands of dq[:, 128 d ..] += dS K.
constexpr int kDqPairs = 16;

__global__ void __launch_bounds__(kDqThreads, 1)
bwd_dq_kernel(const BwdParams p, const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
              const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_vc) {
    extern __shared__ __align__(1024) uint8_t dsmem[];
    if (smem_u32(dsmem) & 1023u) {
        if (threadIdx.x == 0) record_error(HCA_ERR_INTERNAL);
        return;
    }
    uint8_t* sm = dsmem;
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kBwdSmBar);
    uint64_t* empty = full + kBwdRing;
    uint64_t* sdp_full = empty + kBwdRing;      // [2]
    uint64_t* sdp_empty = sdp_full + 2;         // [2]
    uint64_t* rec_ready = sdp_full + 4;
    uint64_t* acc_full = sdp_full + 5;
    uint64_t* acc_empty = sdp_full + 6;
    uint64_t* drain = sdp_full + 7;
    int* misc = reinterpret_cast<int*>(sm + kBwdSmMisc);
    volatile int* abort_flag = misc;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int i = 0; i < kBwdRing; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sdp_full[i], 1);
            mbar_init(&sdp_empty[i], 8);
        }
        mbar_init(rec_ready, 1);
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 8);
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const long long stride = gridDim.x;
    auto decode_item = [&](long long i, int& b, int& g, int& rt) {
        g = (int)(i % p.Hkv);
        const long long r = i / p.Hkv;
        b = (int)(r % p.B);
        rt = p.s1 - 1 - (int)(r / p.B);        // heavy (late) row tiles first
    };

    if (warp == 0) {
        // ================================================================ TMA producer
        if (lane == 0) {
            uint32_t op = 0, nitem = 0;
            bool ok = true;
            auto slot = [&](uint32_t& st) -> uint8_t* {
                st = op % kBwdRing;
                if (!mbar_wait(&empty[st], ((op / kBwdRing) & 1) ^ 1, abort_flag)) return nullptr;
                return sm + kBwdSmRing + st * kBwdSlot;
            };
            for (long long i = blockIdx.x; ok && i < p.dq_items; i += stride, ++nitem) {
                int b, g, rt;
                decode_item(i, b, g, rt);
                const BwdRows it = bwd_rows(p, rt);
                for (int j = 0; ok && j < it.nt; ++j) {
                    const bool comp = j < it.nct;
                    const int row = 128 * (comp ? j : it.kw0 + j - it.nct);
                    for (int o = 0; o < kDqPairs; ++o, ++op) {
                        uint32_t st;
                        uint8_t* base = slot(st);
                        if (!base) { ok = false; break; }
                        const int s = o & 7;
                        mbar_arrive_expect_tx(&full[st], kBwdSlot);
                        tma_load_4d(base, o < 8 ? &tm_q : &tm_do, &full[st], 64 * s, g * p.G, it.t0, b);
                        tma_load_4d(base + kBwdSlab, o < 8 ? (comp ? &tm_kc : &tm_k) : (comp ? &tm_vc : &tm_v),
                                    &full[st], 64 * s, g, row, b);
                    }
                }
                // phase A reads the dS the softmax warps have written for this item
                if (ok && !mbar_wait(rec_ready, nitem & 1, abort_flag)) ok = false;
                for (int j = 0; ok && j < it.nt; ++j) {
                    const bool comp = j < it.nct;
                    const int row = 128 * (comp ? j : it.kw0 + j - it.nct);
                    const CUtensorMap* km = comp ? &tm_kc : &tm_k;
                    for (int o = 0; o < 5; ++o, ++op) {
                        uint32_t st;
                        uint8_t* base = slot(st);
                        if (!base) { ok = false; break; }
                        mbar_arrive_expect_tx(&full[st], kBwdSlot);
                        if (o == 0) {
                            bulk_load(base, bwd_record(p, b, g, rt, j) + kBwdSlot, kBwdSlot, &full[st]);
                        } else {
                            const int c = 128 * (o - 1);
                            tma_load_4d(base, km, &full[st], c, g, row, b);
                            tma_load_4d(base + kBwdSlab, km, &full[st], c + 64, g, row, b);
                        }
                    }
                }
            }
            mbar_drain_ring(full, op, kBwdRing);
        }
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        const uint32_t id_s = idesc_bf16(128, 128, 0, 0);
        const uint32_t id_a = idesc_bf16(128, 128, 0, 1), id_a2 = idesc_bf16(128, 256, 0, 1);
        const uint32_t ring = smem_u32(sm + kBwdSmRing);
        uint32_t op = 0, ns = 0, nitem = 0;
        bool ok = true;
        for (long long i = blockIdx.x; ok && i < p.dq_items; i += stride, ++nitem) {
            int b, g, rt;
            decode_item(i, b, g, rt);
            const BwdRows it = bwd_rows(p, rt);
            // tensor memory is free once the previous item's dq has been read out
            if (!warp_wait(acc_empty, (nitem & 1) ^ 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            for (int j = 0; ok && j < it.nt; ++j, ++ns) {
                const uint32_t buf = ns & 1;
                // the softmax warps have read this buffer's previous tile
                if (!warp_wait(&sdp_empty[buf], ((ns >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                for (int o = 0; o < kDqPairs; ++o, ++op) {
                    const uint32_t st = op % kBwdRing;
                    if (!warp_wait(&full[st], (op / kBwdRing) & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t a = ring + st * kBwdSlot, bb = a + kBwdSlab;
                        const uint32_t d = tmem + 256 * buf + (o < 8 ? 0 : 128);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_ss(d, smem_desc_sw128(a + kk * 32, 16, 1024), smem_desc_sw128(bb + kk * 32, 16, 1024),
                                   id_s, ((o & 7) | kk) ? 1u : 0u);
                        mma_commit(&empty[st]);
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (lane == 0) mma_commit(&sdp_full[buf]);
                __syncwarp();
            }
            if (!ok) break;
            // phase A overwrites both buffers: the softmax warps have read the last two tiles
            for (int m = (int)ns - 1; ok && m >= 0 && m >= (int)ns - 2; --m)
                if (!warp_wait(&sdp_empty[m & 1], (m >> 1) & 1, abort_flag)) ok = false;
            if (!ok) break;
            tc_fence_after();
            for (int j = 0; ok && j < it.nt; ++j) {
                for (int o = 0; o < 5; ++o)
                    if (!warp_wait(&full[(op + o) % kBwdRing], ((op + o) / kBwdRing) & 1, abort_flag)) ok = false;
                if (!ok) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t ds = ring + (op % kBwdRing) * kBwdSlot;
#pragma unroll 1
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint64_t ad = smem_desc_sw128(ds + (kk >> 2) * kBwdSlab + (kk & 3) * 32, 16, 1024);
                        bwd_mma_blocks(tmem, ad, ring, op + 1, kk, id_a, id_a2, (j | kk) ? 1u : 0u);
                    }
                    for (int o = 0; o < 5; ++o) mma_commit(&empty[(op + o) % kBwdRing]);
                    if (j == it.nt - 1) mma_commit(acc_full);
                }
                __syncwarp();
                op += 5;
            }
        }
        // every MMA has completed before the CTA releases its shared and tensor memory
        if (lane == 0) {
            mma_commit(drain);
            mbar_drain_wait(drain, 0);
        }
        __syncwarp();
    } else {
        // ================================================================ P, dS and the epilogue
        const int q4 = warp & 3;                  // tensor-memory lane quarter
        const int hc = (warp - 2) >> 2;           // column half
        const int r = q4 * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        uint8_t* stg = sm + kBwdSmStage + (warp - 2) * kBwdStageBytes;
        uint32_t ns = 0, nitem = 0;
        bool ok = true;
        for (long long i = blockIdx.x; ok && i < p.dq_items; i += stride, ++nitem) {
            int b, g, rt;
            decode_item(i, b, g, rt);
            const BwdRows it = bwd_rows(p, rt);
            const int tok = it.t0 + r / p.G;
            const bool live = tok < p.T;
            const int t = live ? tok : p.T - 1;
            const int head = g * p.G + r % p.G;
            const float lse2 = live ? __ldg(p.lse + ((size_t)b * p.Hq + head) * p.T + t) * 1.4426950408889634f : 0.f;
            const float Dr = live ? __ldg(p.drow + ((size_t)b * p.T + t) * p.Hq + head) : 0.f;
            const int nc_t = bwd_visible(t, p.W, p.blk);
            for (int j = 0; ok && j < it.nt; ++j, ++ns) {
                const uint32_t buf = ns & 1;
                if (!bwd_group_wait<256>(&sdp_full[buf], (ns >> 1) & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                int lo, hi;   // valid key columns of this row in the tile
                if (j < it.nct) {
                    lo = 0;
                    hi = min(128, nc_t - 128 * j);
                } else {
                    const int u0 = 128 * (it.kw0 + j - it.nct);
                    lo = max(0, t - p.W + 1 - u0);
                    hi = min(128, t - u0 + 1);
                }
                if (!live) hi = lo;
                // this warp's 32 rows of slab hc: 4 KB, contiguous in the record
                uint8_t* rp = bwd_record(p, b, g, rt, j) + hc * kBwdSlab + q4 * 32 * 128;
                // P goes straight into the staging buffer (the row's chunks at their swizzled
                // places), dS stays in registers until P is out
                uint32_t pd[32];
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int c0 = 64 * hc + 32 * h2;
                    float sv[32], dpv[32];
                    const uint32_t tb = tmem + lane_off + 256 * buf + c0;
                    tmem_ld16(tb, sv);
                    tmem_ld16(tb + 16, sv + 16);
                    tmem_ld16(tb + 128, dpv);
                    tmem_ld16(tb + 144, dpv + 16);
                    tmem_wait_ld();
                    uint32_t pp[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const int c = c0 + e;
                        const float p0 = (c >= lo && c < hi) ? ex2(fmaf(sv[e], p.scale_log2, -lse2)) : 0.f;
                        const float p1 = (c + 1 >= lo && c + 1 < hi) ? ex2(fmaf(sv[e + 1], p.scale_log2, -lse2)) : 0.f;
                        pp[e >> 1] = pack_bf16x2(p0, p1);
                        pd[16 * h2 + (e >> 1)] = pack_bf16x2(p0 * (dpv[e] - Dr), p1 * (dpv[e + 1] - Dr));
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<uint4*>(stg + bwd_sw(lane, 4 * h2 + q)) =
                            make_uint4(pp[4 * q], pp[4 * q + 1], pp[4 * q + 2], pp[4 * q + 3]);
                }
                // S and dP are read: the MMAs of the tile after next may use the buffer
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sdp_empty[buf]);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    *reinterpret_cast<uint4*>(rp + i * 512 + lane * 16) = *reinterpret_cast<const uint4*>(stg + i * 512 + lane * 16);
                __syncwarp();
                bwd_warp_rows_out(stg, rp + kBwdSlot, pd, lane);
            }
            if (!ok) break;
            // the records are complete: hand them to the async proxy (the producer's bulk loads)
            fence_proxy_async_global();
            bwd_bar<256>();
            if (threadIdx.x == 64) mbar_arrive(rec_ready);
            // ---- dq = scale * accumulator, channels 256 hc ..
            if (!bwd_group_wait<256>(acc_full, nitem & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
#pragma unroll 1
            for (int c0 = 0; c0 < 256; c0 += 32) {
                float a[32];
                tmem_ld16(tmem + lane_off + 256 * hc + c0, a);
                tmem_ld16(tmem + lane_off + 256 * hc + c0 + 16, a + 16);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) a[e] *= p.scale;
                const int ch = 256 * hc + c0;
                bwd_warp_f32_out<false>(stg, a, lane, [&](int row) -> float* {
                    const int rr = q4 * 32 + row;
                    const int tk = it.t0 + rr / p.G;
                    if (tk >= p.T) return nullptr;
                    return p.dq + (((size_t)b * p.T + tk) * p.Hq + g * p.G + rr % p.G) * kBwdD + ch;
                });
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// -------------------------------------------------------------------------------- dk, dv

// Item of a dk/dv launch: key tile kt (entries 128 kt .. when comp, else raw tokens 128 kt ..),
// which = 0 for dV (from P and dO) or 1 for dK (from dS and Q), over row tiles [rt_lo, rt_hi).
// Per (b, g): the entry tiles' items first, ordered (chunk of ch_rows row tiles, kt, which) so
// that the CTAs running at once share those rows of Q and dO in L2; then the raw tiles' (kt, which).
struct BwdKeys {
    int b, g, kt, comp, which, k0, nk, rt_lo, rt_hi;
};

__device__ __forceinline__ bool bwd_keys(const BwdParams& p, long long i, BwdKeys& kk) {
    const long long per_c = 2LL * p.nkc * p.nch, per_bg = per_c + 2LL * p.nraw;
    const long long bg = i / per_bg;
    long long rem = i - bg * per_bg;
    kk.b = (int)(bg / p.Hkv);
    kk.g = (int)(bg % p.Hkv);
    kk.which = (int)(rem & 1);
    int lo, hi;
    if (rem < per_c) {
        kk.comp = 1;
        rem >>= 1;
        kk.kt = (int)(rem % p.nkc);
        const int c = (int)(rem / p.nkc);
        kk.k0 = 128 * kk.kt;
        kk.nk = min(128, p.Nc - kk.k0);
        // the first token that sees entry k0: n_c(t) > k0  <=>  t >= blk (k0 + 1) + W - 1
        const long long tmin = (long long)p.blk * (kk.k0 + 1) + p.W - 1;
        lo = tmin >= p.T ? p.ntile_t : (int)(tmin / p.tpt);
        hi = p.ntile_t;
        lo = max(lo, p.s0 + c * p.ch_rows);
        hi = min(hi, min(p.s1, p.s0 + (c + 1) * p.ch_rows));
    } else {
        kk.comp = 0;
        kk.kt = p.kta + (int)((rem - per_c) >> 1);
        if (kk.kt >= p.nkw) return false;
        kk.k0 = 128 * kk.kt;
        kk.nk = min(128, p.T - kk.k0);
        const int tmax = min(p.T - 1, kk.k0 + kk.nk - 1 + p.W - 1);
        lo = max(kk.k0 / p.tpt, p.s0);
        hi = min(tmax / p.tpt + 1, p.s1);
    }
    kk.rt_lo = lo;
    kk.rt_hi = hi;
    return lo < hi && kk.nk > 0;
}

// Record slot of key tile kt in row tile rt (the dq kernel's order).
__device__ __forceinline__ int bwd_slot(const BwdParams& p, const BwdKeys& kk, int rt) {
    if (kk.comp) return kk.kt;
    const BwdRows it = bwd_rows(p, rt);
    return it.nct + kk.kt - it.kw0;
}

__global__ void __launch_bounds__(kKvThreads, 1)
bwd_dkv_kernel(const BwdParams p, const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do) {
    extern __shared__ __align__(1024) uint8_t dsmem[];
    if (smem_u32(dsmem) & 1023u) {
        if (threadIdx.x == 0) record_error(HCA_ERR_INTERNAL);
        return;
    }
    uint8_t* sm = dsmem;
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kBwdSmBar);
    uint64_t* empty = full + kBwdRing;
    uint64_t* acc_full = empty + kBwdRing;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* drain = acc_full + 2;
    int* misc = reinterpret_cast<int*>(sm + kBwdSmMisc);
    volatile int* abort_flag = misc;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int i = 0; i < kBwdRing; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 4);
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const long long stride = gridDim.x;

    if (warp == 0) {
        // ops of one row tile: the record's P (dV) or dS (dK), then dO (dV) or Q (dK) rows as four
        // ops of two 64-channel blocks
        if (lane == 0) {
            uint32_t op = 0;
            bool ok = true;
            for (long long i = blockIdx.x; ok && i < p.kv_items; i += stride) {
                BwdKeys kk;
                if (!bwd_keys(p, i, kk)) continue;
                const CUtensorMap* m = kk.which ? &tm_q : &tm_do;
                for (int rt = kk.rt_lo; ok && rt < kk.rt_hi; ++rt) {
                    const uint8_t* rec = bwd_record(p, kk.b, kk.g, rt, bwd_slot(p, kk, rt)) + kk.which * kBwdSlot;
                    for (int o = 0; o < 5; ++o, ++op) {
                        const uint32_t st = op % kBwdRing;
                        if (!mbar_wait(&empty[st], ((op / kBwdRing) & 1) ^ 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        uint8_t* base = sm + kBwdSmRing + st * kBwdSlot;
                        mbar_arrive_expect_tx(&full[st], kBwdSlot);
                        if (o == 0) {
                            bulk_load(base, rec, kBwdSlot, &full[st]);
                        } else {
                            const int c = 128 * (o - 1);
                            tma_load_4d(base, m, &full[st], c, kk.g * p.G, rt * p.tpt, kk.b);
                            tma_load_4d(base + kBwdSlab, m, &full[st], c + 64, kk.g * p.G, rt * p.tpt, kk.b);
                        }
                    }
                }
            }
            mbar_drain_ring(full, op, kBwdRing);
        }
    } else if (warp == 1) {
        // D[key, channel] += sum over the tile's 128 query rows of X[row, key] Y[row, channel]:
        // A = the record's tile read MN-major (keys contiguous), B = dO / Q MN-major
        const uint32_t id_a = idesc_bf16(128, 128, 1, 1), id_a2 = idesc_bf16(128, 256, 1, 1);
        const uint32_t ring = smem_u32(sm + kBwdSmRing);
        uint32_t op = 0, nitem = 0;
        bool ok = true;
        for (long long i = blockIdx.x; ok && i < p.kv_items; i += stride) {
            BwdKeys kk;
            if (!bwd_keys(p, i, kk)) continue;
            if (!warp_wait(acc_empty, (nitem & 1) ^ 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            for (int rt = kk.rt_lo; ok && rt < kk.rt_hi; ++rt) {
                for (int o = 0; o < 5; ++o)
                    if (!warp_wait(&full[(op + o) % kBwdRing], ((op + o) / kBwdRing) & 1, abort_flag)) ok = false;
                if (!ok) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t x = ring + (op % kBwdRing) * kBwdSlot;
                    const bool first = rt == kk.rt_lo;
#pragma unroll 1
                    for (int q = 0; q < 8; ++q)
                        bwd_mma_blocks(tmem, smem_desc_sw128(x + q * 2048, kBwdSlab, 1024), ring, op + 1, q, id_a, id_a2,
                                       (first && q == 0) ? 0u : 1u);
                    for (int o = 0; o < 5; ++o) mma_commit(&empty[(op + o) % kBwdRing]);
                    if (rt == kk.rt_hi - 1) mma_commit(acc_full);
                }
                __syncwarp();
                op += 5;
            }
            ++nitem;
        }
        if (lane == 0) {
            mma_commit(drain);
            mbar_drain_wait(drain, 0);
        }
        __syncwarp();
    } else {
        // ================================================================ epilogue: one key row per thread
        const int q4 = warp & 3;
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        uint8_t* stg = sm + kBwdSmStage + (warp - 2) * kBwdStageBytes;
        uint32_t nitem = 0;
        for (long long i = blockIdx.x; i < p.kv_items; i += stride) {
            BwdKeys kk;
            if (!bwd_keys(p, i, kk)) continue;
            if (!bwd_group_wait<128>(acc_full, nitem & 1, abort_flag)) break;
            tc_fence_after();
            const float mul = kk.which ? p.scale : 1.f;
            float* base = kk.comp ? (kk.which ? p.dkc : p.dvc) : (kk.which ? p.dk : p.dv);
            const size_t rows = kk.comp ? (size_t)p.Nc : (size_t)p.T;
#pragma unroll 1
            for (int c0 = 0; c0 < kBwdD; c0 += 32) {
                float a[32];
                tmem_ld16(tmem + lane_off + c0, a);
                tmem_ld16(tmem + lane_off + c0 + 16, a + 16);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) a[e] *= mul;
                bwd_warp_f32_out<true>(stg, a, lane, [&](int row) -> float* {
                    const int key = q4 * 32 + row;
                    if (key >= kk.nk) return nullptr;
                    return base + (((size_t)kk.b * rows + kk.k0 + key) * p.Hkv + kk.g) * kBwdD + c0;
                });
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
            ++nitem;
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// -------------------------------------------------------------------------------- pooling backward

// One CTA per (sequence, block): alpha = softmax of the block's weights; the raw rows receive
// alpha_i dKc, alpha_i dVc (added to the window path's gradients already there) and
// dw_i = alpha_i (dalpha_i - sum alpha dalpha), dalpha_i = sum over KV heads of K_i.dKc + V_i.dVc.
constexpr int kPoolThreads = 256;

__global__ void __launch_bounds__(kPoolThreads) bwd_pool_kernel(const BwdParams p) {
    __shared__ float alpha[128], dal[128], red[8];
    const int b = blockIdx.x / p.Nc, j = blockIdx.x - (blockIdx.x / p.Nc) * p.Nc;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t pos0 = (size_t)b * p.T + (size_t)p.blk * j;
    if (warp == 0) {
        float wv[4], m = -INFINITY;
        for (int u = 0; u < 4; ++u) {
            const int i = lane + 32 * u;
            wv[u] = i < p.blk ? (p.w ? __ldg(p.w + pos0 + i) : 0.f) : -INFINITY;
            m = fmaxf(m, wv[u]);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        float s = 0.f;
        for (int u = 0; u < 4; ++u) {
            wv[u] = (lane + 32 * u) < p.blk ? __expf(wv[u] - m) : 0.f;
            s += wv[u];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        for (int u = 0; u < 4; ++u) alpha[lane + 32 * u] = wv[u] / s;
    }
    __syncthreads();
    // dalpha_i: one warp per row at a time, lanes over channels
    for (int i = warp; i < p.blk; i += kPoolThreads / 32) {
        float acc = 0.f;
        for (int g = 0; g < p.Hkv; ++g) {
            const __nv_bfloat16* kr = p.k + ((pos0 + i) * p.Hkv + g) * kBwdD;
            const __nv_bfloat16* vr = p.v + ((pos0 + i) * p.Hkv + g) * kBwdD;
            const float* gk = p.dkc + (((size_t)b * p.Nc + j) * p.Hkv + g) * kBwdD;
            const float* gv = p.dvc + (((size_t)b * p.Nc + j) * p.Hkv + g) * kBwdD;
            for (int c = 2 * lane; c < kBwdD; c += 64) {
                const uint32_t kw = *reinterpret_cast<const uint32_t*>(kr + c);
                const uint32_t vw = *reinterpret_cast<const uint32_t*>(vr + c);
                const float2 a = *reinterpret_cast<const float2*>(gk + c);
                const float2 d = *reinterpret_cast<const float2*>(gv + c);
                acc = fmaf(bf16lo(kw), a.x, fmaf(bf16hi(kw), a.y, acc));
                acc = fmaf(bf16lo(vw), d.x, fmaf(bf16hi(vw), d.y, acc));
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) dal[i] = acc;
    }
    __syncthreads();
    // sum alpha dalpha, then dw
    float part = 0.f;
    for (int i = threadIdx.x; i < p.blk; i += kPoolThreads) part += alpha[i] * dal[i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    if (lane == 0) red[warp] = part;
    __syncthreads();
    float tot = 0.f;
    for (int wi = 0; wi < kPoolThreads / 32; ++wi) tot += red[wi];
    if (p.dw)
        for (int i = threadIdx.x; i < p.blk; i += kPoolThreads) p.dw[pos0 + i] = alpha[i] * (dal[i] - tot);
    // dk, dv of the block's rows += alpha_i * (dKc, dVc)
    const int per_row = p.Hkv * kBwdD / 4;         // float4 per row
    for (int e = threadIdx.x; e < p.blk * per_row; e += kPoolThreads) {
        const int i = e / per_row, c4 = e - i * per_row;
        const float a = alpha[i];
        const float4 gk = reinterpret_cast<const float4*>(p.dkc + (((size_t)b * p.Nc + j) * p.Hkv) * kBwdD)[c4];
        const float4 gv = reinterpret_cast<const float4*>(p.dvc + (((size_t)b * p.Nc + j) * p.Hkv) * kBwdD)[c4];
        float4* dk4 = reinterpret_cast<float4*>(p.dk + (pos0 + i) * p.Hkv * kBwdD) + c4;
        float4* dv4 = reinterpret_cast<float4*>(p.dv + (pos0 + i) * p.Hkv * kBwdD) + c4;
        float4 x = *dk4, y = *dv4;
        x.x = fmaf(a, gk.x, x.x); x.y = fmaf(a, gk.y, x.y); x.z = fmaf(a, gk.z, x.z); x.w = fmaf(a, gk.w, x.w);
        y.x = fmaf(a, gv.x, y.x); y.y = fmaf(a, gv.y, y.y); y.z = fmaf(a, gv.z, y.z); y.w = fmaf(a, gv.w, y.w);
        *dk4 = x;
        *dv4 = y;
    }
}

}  // namespace hca
