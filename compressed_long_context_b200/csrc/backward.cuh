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
// Kernels (every contraction on tcgen05, 512-dim heads):
//   bwd_pre_kernel   D for every (token, head) row (one warp per row).
//   bwd_dq_kernel    one CTA per row tile of 128 (token, head) rows: for every key tile it
//                    recomputes S = Q K^T and dP = dO V^T (TMEM, 128 columns each), the
//                    softmax warps form dS (bf16, shared memory), and dq += dS K accumulates in
//                    TMEM -- 256 columns, so the 512 channels take two passes.
//   bwd_dkv_kernel   one CTA per (key tile, range of query row tiles): S^T = K Q^T and, for dK,
//                    dP^T = V dO^T; dV += P^T dO and dK += dS^T Q in channel halves (four passes),
//                    added with fp32 atomics into the entries' gradients (workspace) or the raw
//                    window keys' gradients.
//   bwd_pool_kernel  one CTA per (sequence, block): pooling backward into dk, dv and dw.
// Operands stream through one ring of six 32 KB slots (an A slab and a B slab of 128 rows x 64
// channels each); the MMA issuer consumes the ops in the producer's order.  Every wait is
// bounded (common.cuh).
#pragma once

#include "common.cuh"

namespace hca {

constexpr int kBwdD = 512;
constexpr int kBwdThreads = 192;            // producer, MMA issuer, 4 softmax / epilogue warps
constexpr int kBwdRing = 6;
constexpr uint32_t kBwdSlab = 16384;         // 128 rows x 64 channels bf16, 128-byte swizzle
constexpr uint32_t kBwdSlot = 2 * kBwdSlab;  // A slab + B slab
constexpr uint32_t kBwdSmRing = 0;
constexpr uint32_t kBwdSmX = kBwdSmRing + kBwdRing * kBwdSlot;      // dS (or P^T / dS^T): 2 slabs
constexpr uint32_t kBwdSmCol = kBwdSmX + 2 * kBwdSlab;              // per-column data (dkv): 128 x float4
constexpr uint32_t kBwdSmBar = kBwdSmCol + 4 * 128 * 4;
constexpr int kBwdNumBars = 2 * kBwdRing + 8;
constexpr uint32_t kBwdSmMisc = kBwdSmBar + kBwdNumBars * 8;
constexpr uint32_t kBwdSmem = kBwdSmMisc + 16;
static_assert(kBwdSmem <= 232448, "backward shared memory exceeds the per-block limit");
static_assert(kBwdSmX % 1024 == 0 && kBwdSlot % 1024 == 0, "swizzled operands 1024-aligned");

// TMEM columns
constexpr uint32_t kBwdTmS = 0;      // S (or S^T): 128 columns
constexpr uint32_t kBwdTmP = 128;    // dP (or dP^T): 128 columns
constexpr uint32_t kBwdTmAcc = 256;  // dq / dk / dv half: 256 columns

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
    int B, T, Hq, Hkv, G, tpt, blk, W, Nc, ntile_t, out_f32;
    long long dq_items;           // B * Hkv * ntile_t
    int nkc, nkw;                 // compressed / raw key tiles per (b, g)
    int chc, chw;                 // row-tile chunks per compressed / raw key tile
    int rt_chunk;                 // row tiles per chunk
    long long kv_items;
    float scale, scale_log2;
};

__device__ __forceinline__ int bwd_visible(int t, int W, int blk) {
    const int a = t - W + 1;
    return a > 0 ? a / blk : 0;
}

// Row tile of a dq item: rows (token t0 + r / G, head g * G + r % G).
struct BwdRows {
    int b, g, t0, tlast, ncomp, nct, wlo, nwin, nwt;
};

__device__ __forceinline__ BwdRows bwd_rows(const BwdParams& p, int b, int g, int rt) {
    BwdRows it;
    it.b = b;
    it.g = g;
    it.t0 = rt * p.tpt;
    it.tlast = min(it.t0 + p.tpt, p.T) - 1;
    it.ncomp = bwd_visible(it.tlast, p.W, p.blk);
    it.nct = (it.ncomp + 127) / 128;
    it.wlo = max(0, it.t0 - p.W + 1);
    it.nwin = it.tlast - it.wlo + 1;
    it.nwt = (it.nwin + 127) / 128;
    return it;
}

// Named barrier among the four softmax / epilogue warps.
__device__ __forceinline__ void bwd_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ bool bwd_group_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
    const bool ok = mbar_wait(bar, parity, abort);
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
                 "barrier.red.and.pred q, 2, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r) : "r"((uint32_t)ok) : "memory");
    return r != 0;
}

// Byte offset of 16-byte chunk c of row r in a 128-byte-swizzled slab.
__device__ __forceinline__ uint32_t bwd_sw(uint32_t r, uint32_t c) { return r * 128u + (((c ^ r) & 7u) << 4); }

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

// -------------------------------------------------------------------------------- dq

// Ops of one key tile of a dq pass: 8 x (Q slab, K slab) for S, 8 x (dO slab, V slab) for dP,
// then two ops that each carry two of the pass's four K channel blocks (channels 256 h + 128 d
// and + 64, in the slot's A and B halves): the N = 128 B operands of dq[:, 128 d ..] += dS K.
constexpr int kDqPairs = 16;
constexpr int kDqOps = kDqPairs + 2;

// Softmax-gradient columns c0 .. c0 + 15 of row r, packed to bf16, into the K-major 128-byte-
// swizzled operand buffer (two slabs of 64 columns).
__device__ __forceinline__ void bwd_put16(uint8_t* xs, int r, int c0, const uint32_t* pk) {
    uint8_t* dst = xs + (c0 >> 6) * kBwdSlab;
    const uint32_t ch = (uint32_t)(c0 & 63) >> 3;
    *reinterpret_cast<uint4*>(dst + bwd_sw(r, ch)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    *reinterpret_cast<uint4*>(dst + bwd_sw(r, ch + 1)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
}

__global__ void __launch_bounds__(kBwdThreads, 1)
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
    uint64_t* sdp_full = empty + kBwdRing;
    uint64_t* sdp_empty = sdp_full + 1;
    uint64_t* ds_full = sdp_full + 2;
    uint64_t* ds_empty = sdp_full + 3;
    uint64_t* acc_full = sdp_full + 4;
    uint64_t* acc_empty = sdp_full + 5;
    uint64_t* drain = sdp_full + 6;
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
        mbar_init(sdp_full, 1);
        mbar_init(sdp_empty, 4);
        mbar_init(ds_full, 4);
        mbar_init(ds_empty, 1);
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
    auto decode_item = [&](long long i, int& b, int& g, int& rt) {
        g = (int)(i % p.Hkv);
        long long r = i / p.Hkv;
        b = (int)(r % p.B);
        rt = p.ntile_t - 1 - (int)(r / p.B);        // heavy (late) row tiles first
    };

    if (warp == 0) {
        // ================================================================ TMA producer
        if (lane == 0) {
            uint32_t op = 0;
            bool ok = true;
            for (long long i = blockIdx.x; ok && i < p.dq_items; i += stride) {
                int b, g, rt;
                decode_item(i, b, g, rt);
                const BwdRows it = bwd_rows(p, b, g, rt);
                const int nt = it.nct + it.nwt;
                for (int h = 0; ok && h < 2; ++h)
                    for (int j = 0; ok && j < nt; ++j) {
                        const bool comp = j < it.nct;
                        const int row = comp ? 128 * j : it.wlo + 128 * (j - it.nct);
                        for (int o = 0; o < kDqOps; ++o, ++op) {
                            const uint32_t st = op % kBwdRing;
                            if (!mbar_wait(&empty[st], ((op / kBwdRing) & 1) ^ 1, abort_flag)) {
                                ok = false;
                                break;
                            }
                            uint8_t* base = sm + kBwdSmRing + st * kBwdSlot;
                            mbar_arrive_expect_tx(&full[st], kBwdSlot);
                            if (o < kDqPairs) {
                                const int s = o & 7;
                                tma_load_4d(base, o < 8 ? &tm_q : &tm_do, &full[st], 64 * s, g * p.G, it.t0, b);
                                tma_load_4d(base + kBwdSlab, o < 8 ? (comp ? &tm_kc : &tm_k) : (comp ? &tm_vc : &tm_v),
                                            &full[st], 64 * s, g, row, b);
                            } else {
                                const int c = 256 * h + 128 * (o - kDqPairs);
                                const CUtensorMap* km = comp ? &tm_kc : &tm_k;
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
        const uint32_t id_q = idesc_bf16(128, 128, 0, 1);
        const uint32_t ring = smem_u32(sm + kBwdSmRing), xs = smem_u32(sm + kBwdSmX);
        uint32_t op = 0, nkt = 0, npass = 0;
        bool ok = true;
        for (long long i = blockIdx.x; ok && i < p.dq_items; i += stride) {
            int b, g, rt;
            decode_item(i, b, g, rt);
            const BwdRows it = bwd_rows(p, b, g, rt);
            const int nt = it.nct + it.nwt;
            for (int h = 0; ok && h < 2; ++h, ++npass) {
                for (int j = 0; ok && j < nt; ++j, ++nkt) {
                    // S and dP of the previous key tile have been read by the softmax warps
                    if (!warp_wait(sdp_empty, (nkt & 1) ^ 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    for (int o = 0; o < kDqPairs; ++o, ++op) {
                        const uint32_t st = op % kBwdRing;
                        if (!warp_wait(&full[st], (op / kBwdRing) & 1, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        if (lane == 0) {
                            const uint32_t a = ring + st * kBwdSlot, bb = a + kBwdSlab;
                            const uint32_t d = tmem + (o < 8 ? kBwdTmS : kBwdTmP);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_ss(d, smem_desc_sw128(a + kk * 32, 16, 1024), smem_desc_sw128(bb + kk * 32, 16, 1024),
                                       id_s, ((o & 7) | kk) ? 1u : 0u);
                            mma_commit(&empty[st]);
                        }
                        __syncwarp();
                    }
                    if (!ok) break;
                    if (lane == 0) mma_commit(sdp_full);
                    __syncwarp();
                    // dq half += dS K_half, once dS is in shared memory (and, on the pass's first
                    // key tile, once the previous pass's accumulator has been read out)
                    if (j == 0 && !warp_wait(acc_empty, (npass & 1) ^ 1, abort_flag)) { ok = false; break; }
                    if (!warp_wait(ds_full, nkt & 1, abort_flag)) { ok = false; break; }
                    if (!warp_wait(&full[op % kBwdRing], (op / kBwdRing) & 1, abort_flag) ||
                        !warp_wait(&full[(op + 1) % kBwdRing], ((op + 1) / kBwdRing) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint64_t ad = smem_desc_sw128(xs + (kk >> 2) * kBwdSlab + (kk & 3) * 32, 16, 1024);
#pragma unroll
                            for (int d = 0; d < 2; ++d)
                                mma_ss(tmem + kBwdTmAcc + 128 * d, ad,
                                       smem_desc_sw128(ring + ((op + d) % kBwdRing) * kBwdSlot + kk * 2048, kBwdSlab,
                                                       1024),
                                       id_q, (j | kk) ? 1u : 0u);
                        }
                        mma_commit(&empty[op % kBwdRing]);
                        mma_commit(&empty[(op + 1) % kBwdRing]);
                        mma_commit(ds_empty);
                        if (j == nt - 1) mma_commit(acc_full);
                    }
                    __syncwarp();
                    op += 2;
                }
            }
        }
        // every MMA has completed before the CTA releases its shared and tensor memory
        if (lane == 0) {
            mma_commit(drain);
            mbar_drain_wait(drain, 0);
        }
        __syncwarp();
    } else {
        // ================================================================ dS and the epilogue
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        uint8_t* xsp = sm + kBwdSmX;
        uint32_t nkt = 0, npass = 0;
        bool ok = true;
        for (long long i = blockIdx.x; ok && i < p.dq_items; i += stride) {
            int b, g, rt;
            decode_item(i, b, g, rt);
            const BwdRows it = bwd_rows(p, b, g, rt);
            const int nt = it.nct + it.nwt;
            const int tok = it.t0 + r / p.G;
            const bool live = tok < p.T;
            const int t = live ? tok : p.T - 1;
            const int head = g * p.G + r % p.G;
            const float lse2 = live ? __ldg(p.lse + ((size_t)b * p.Hq + head) * p.T + t) * 1.4426950408889634f : 0.f;
            const float Dr = live ? __ldg(p.drow + ((size_t)b * p.T + t) * p.Hq + head) : 0.f;
            const int nc_t = bwd_visible(t, p.W, p.blk);
            for (int h = 0; ok && h < 2; ++h, ++npass) {
                for (int j = 0; ok && j < nt; ++j, ++nkt) {
                    if (!bwd_group_wait(sdp_full, nkt & 1, abort_flag)) { ok = false; break; }
                    // the previous key tile's dS has been consumed
                    if (!bwd_group_wait(ds_empty, (nkt & 1) ^ 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    int lo, hi;   // valid columns of this row in the tile
                    if (j < it.nct) {
                        lo = 0;
                        hi = min(128, nc_t - 128 * j);
                    } else {
                        const int u0 = it.wlo + 128 * (j - it.nct);
                        lo = max(0, t - p.W + 1 - u0);
                        hi = min(128, t - u0 + 1);
                    }
                    if (!live) hi = lo;
#pragma unroll 1
                    for (int c0 = 0; c0 < 128; c0 += 16) {
                        float sv[16], dpv[16];
                        tmem_ld16(tmem + lane_off + kBwdTmS + c0, sv);
                        tmem_ld16(tmem + lane_off + kBwdTmP + c0, dpv);
                        tmem_wait_ld();
                        uint32_t pk[8];
#pragma unroll
                        for (int e = 0; e < 16; e += 2) {
                            const int c = c0 + e;
                            const float p0 = (c >= lo && c < hi) ? ex2(fmaf(sv[e], p.scale_log2, -lse2)) : 0.f;
                            const float p1 = (c + 1 >= lo && c + 1 < hi) ? ex2(fmaf(sv[e + 1], p.scale_log2, -lse2)) : 0.f;
                            pk[e >> 1] = pack_bf16x2(p0 * (dpv[e] - Dr), p1 * (dpv[e + 1] - Dr));
                        }
                        bwd_put16(xsp, r, c0, pk);
                    }
                    tc_fence_before();
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(sdp_empty);
                        mbar_arrive(ds_full);
                    }
                }
                if (!ok) break;
                // ---- the pass's dq half: scale * accumulator -> dq[b, t, head, 256 h ..]
                if (!bwd_group_wait(acc_full, npass & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                float* dst = p.dq + (((size_t)b * p.T + t) * p.Hq + head) * kBwdD + 256 * h;
#pragma unroll 1
                for (int c0 = 0; c0 < 256; c0 += 16) {
                    float a[16];
                    tmem_ld16(tmem + lane_off + kBwdTmAcc + c0, a);
                    tmem_wait_ld();
                    if (live)
#pragma unroll
                        for (int e = 0; e < 16; e += 4)
                            *reinterpret_cast<float4*>(dst + c0 + e) =
                                make_float4(p.scale * a[e], p.scale * a[e + 1], p.scale * a[e + 2], p.scale * a[e + 3]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acc_empty);
            }
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

// Key tile kt of (b, g): kt < nkc are entries 128 kt .., else raw tokens 128 (kt - nkc) ..; its
// query row tiles [lo, hi), cut into chunks of rt_chunk.
struct BwdKeys {
    int b, g, kt, comp, k0, nk, rt_lo, rt_hi;
};

__device__ __forceinline__ bool bwd_keys(const BwdParams& p, long long i, BwdKeys& kk) {
    const long long ncomp_items = (long long)p.B * p.Hkv * p.nkc * p.chc;
    int chunk;
    long long r;
    if (i < ncomp_items) {
        kk.comp = 1;
        chunk = (int)(i % p.chc);
        r = i / p.chc;
        kk.kt = (int)(r % p.nkc);
        r /= p.nkc;
    } else {
        i -= ncomp_items;
        kk.comp = 0;
        chunk = (int)(i % p.chw);
        r = i / p.chw;
        kk.kt = (int)(r % p.nkw);
        r /= p.nkw;
    }
    kk.g = (int)(r % p.Hkv);
    kk.b = (int)(r / p.Hkv);
    int lo, hi;
    if (kk.comp) {
        kk.k0 = 128 * kk.kt;
        kk.nk = min(128, p.Nc - kk.k0);
        // the first token that sees entry k0: n_c(t) > k0  <=>  t >= blk (k0 + 1) + W - 1
        const long long tmin = (long long)p.blk * (kk.k0 + 1) + p.W - 1;
        lo = tmin >= p.T ? p.ntile_t : (int)(tmin / p.tpt);
        hi = p.ntile_t;
    } else {
        kk.k0 = 128 * kk.kt;
        kk.nk = min(128, p.T - kk.k0);
        const int tmax = min(p.T - 1, kk.k0 + kk.nk - 1 + p.W - 1);
        lo = kk.k0 / p.tpt;
        hi = tmax / p.tpt + 1;
    }
    kk.rt_lo = lo + chunk * p.rt_chunk;
    kk.rt_hi = min(hi, kk.rt_lo + p.rt_chunk);
    return kk.rt_lo < kk.rt_hi && kk.nk > 0;
}

// Per query row (column of S^T) of row tile rt: its log2-domain LSE, D, and the key rows of the
// tile it sees, [rlo, rhi) relative to k0 (empty for rows past the sequence end).
__device__ __forceinline__ float4 bwd_col(const BwdParams& p, const BwdKeys& kk, int rt, int c) {
    const int tok = rt * p.tpt + c / p.G;
    if (tok >= p.T) return make_float4(0.f, 0.f, __int_as_float(0), __int_as_float(0));
    const int head = kk.g * p.G + c % p.G;
    const float l2 = __ldg(p.lse + ((size_t)kk.b * p.Hq + head) * p.T + tok) * 1.4426950408889634f;
    const float D = __ldg(p.drow + ((size_t)kk.b * p.T + tok) * p.Hq + head);
    int rlo, rhi;
    if (kk.comp) {
        rlo = 0;
        rhi = bwd_visible(tok, p.W, p.blk) - kk.k0;
    } else {
        rlo = tok - p.W + 1 - kk.k0;
        rhi = tok - kk.k0 + 1;
    }
    return make_float4(l2, D, __int_as_float(rlo), __int_as_float(rhi));
}

// Ops of one query row tile in pass ps (0, 1: dV halves; 2, 3: dK halves): 8 x (K slab, Q slab)
// for S^T; for dK, 8 x (V slab, dO slab) for dP^T; then two ops carrying the half's four dO (dV)
// or Q (dK) channel blocks, two per op, as the N = 128 B operands of the accumulation.
__device__ __forceinline__ int bwd_kv_pairs(int ps) { return ps < 2 ? 8 : 16; }

__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_dkv_kernel(const BwdParams p, const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
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
    uint64_t* sdp_full = empty + kBwdRing;
    uint64_t* sdp_empty = sdp_full + 1;
    uint64_t* x_full = sdp_full + 2;
    uint64_t* x_empty = sdp_full + 3;
    uint64_t* acc_full = sdp_full + 4;
    uint64_t* acc_empty = sdp_full + 5;
    uint64_t* drain = sdp_full + 6;
    float4* colv = reinterpret_cast<float4*>(sm + kBwdSmCol);      // [128] per query row (column)
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
        mbar_init(sdp_full, 1);
        mbar_init(sdp_empty, 4);
        mbar_init(x_full, 4);
        mbar_init(x_empty, 1);
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
        if (lane == 0) {
            uint32_t op = 0;
            bool ok = true;
            for (long long i = blockIdx.x; ok && i < p.kv_items; i += stride) {
                BwdKeys kk;
                if (!bwd_keys(p, i, kk)) continue;
                for (int ps = 0; ok && ps < 4; ++ps)
                    for (int rt = kk.rt_lo; ok && rt < kk.rt_hi; ++rt) {
                        const int t0 = rt * p.tpt;
                        const int pairs = bwd_kv_pairs(ps);
                        for (int o = 0; o < pairs + 2; ++o, ++op) {
                            const uint32_t st = op % kBwdRing;
                            if (!mbar_wait(&empty[st], ((op / kBwdRing) & 1) ^ 1, abort_flag)) {
                                ok = false;
                                break;
                            }
                            uint8_t* base = sm + kBwdSmRing + st * kBwdSlot;
                            mbar_arrive_expect_tx(&full[st], kBwdSlot);
                            if (o < pairs) {
                                const int s = o & 7;
                                const bool sk = o < 8;        // S^T: (K, Q); dP^T: (V, dO)
                                tma_load_4d(base, sk ? (kk.comp ? &tm_kc : &tm_k) : (kk.comp ? &tm_vc : &tm_v), &full[st],
                                            64 * s, kk.g, kk.k0, kk.b);
                                tma_load_4d(base + kBwdSlab, sk ? &tm_q : &tm_do, &full[st], 64 * s, kk.g * p.G, t0, kk.b);
                            } else {
                                const int c = 256 * (ps & 1) + 128 * (o - pairs);
                                const CUtensorMap* m = ps < 2 ? &tm_do : &tm_q;
                                tma_load_4d(base, m, &full[st], c, kk.g * p.G, t0, kk.b);
                                tma_load_4d(base + kBwdSlab, m, &full[st], c + 64, kk.g * p.G, t0, kk.b);
                            }
                        }
                    }
            }
            mbar_drain_ring(full, op, kBwdRing);
        }
    } else if (warp == 1) {
        const uint32_t id_s = idesc_bf16(128, 128, 0, 0);
        const uint32_t id_a = idesc_bf16(128, 128, 0, 1);
        const uint32_t ring = smem_u32(sm + kBwdSmRing), xs = smem_u32(sm + kBwdSmX);
        uint32_t op = 0, nrt = 0, npass = 0;
        bool ok = true;
        for (long long i = blockIdx.x; ok && i < p.kv_items; i += stride) {
            BwdKeys kk;
            if (!bwd_keys(p, i, kk)) continue;
            for (int ps = 0; ok && ps < 4; ++ps, ++npass) {
                const int pairs = bwd_kv_pairs(ps);
                for (int rt = kk.rt_lo; ok && rt < kk.rt_hi; ++rt, ++nrt) {
                    if (!warp_wait(sdp_empty, (nrt & 1) ^ 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    for (int o = 0; o < pairs; ++o, ++op) {
                        const uint32_t st = op % kBwdRing;
                        if (!warp_wait(&full[st], (op / kBwdRing) & 1, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        if (lane == 0) {
                            const uint32_t a = ring + st * kBwdSlot, bb = a + kBwdSlab;
                            const uint32_t d = tmem + (o < 8 ? kBwdTmS : kBwdTmP);
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                mma_ss(d, smem_desc_sw128(a + q * 32, 16, 1024), smem_desc_sw128(bb + q * 32, 16, 1024),
                                       id_s, ((o & 7) | q) ? 1u : 0u);
                            mma_commit(&empty[st]);
                        }
                        __syncwarp();
                    }
                    if (!ok) break;
                    if (lane == 0) mma_commit(sdp_full);
                    __syncwarp();
                    const bool first_rt = rt == kk.rt_lo;
                    if (first_rt && !warp_wait(acc_empty, (npass & 1) ^ 1, abort_flag)) { ok = false; break; }
                    if (!warp_wait(x_full, nrt & 1, abort_flag)) { ok = false; break; }
                    if (!warp_wait(&full[op % kBwdRing], (op / kBwdRing) & 1, abort_flag) ||
                        !warp_wait(&full[(op + 1) % kBwdRing], ((op + 1) / kBwdRing) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const uint64_t ad = smem_desc_sw128(xs + (q >> 2) * kBwdSlab + (q & 3) * 32, 16, 1024);
#pragma unroll
                            for (int d = 0; d < 2; ++d)
                                mma_ss(tmem + kBwdTmAcc + 128 * d, ad,
                                       smem_desc_sw128(ring + ((op + d) % kBwdRing) * kBwdSlot + q * 2048, kBwdSlab, 1024),
                                       id_a, (!first_rt || q) ? 1u : 0u);
                        }
                        mma_commit(&empty[op % kBwdRing]);
                        mma_commit(&empty[(op + 1) % kBwdRing]);
                        mma_commit(x_empty);
                        if (rt == kk.rt_hi - 1) mma_commit(acc_full);
                    }
                    __syncwarp();
                    op += 2;
                }
            }
        }
        // every MMA has completed before the CTA releases its shared and tensor memory
        if (lane == 0) {
            mma_commit(drain);
            mbar_drain_wait(drain, 0);
        }
        __syncwarp();
    } else {
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;              // key row of the tile
        const int sidx = threadIdx.x - 64;         // 0..127: column (query row) this thread stages
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        uint8_t* xsp = sm + kBwdSmX;
        uint32_t nrt = 0, npass = 0;
        bool ok = true;
        for (long long i = blockIdx.x; ok && i < p.kv_items; i += stride) {
            BwdKeys kk;
            if (!bwd_keys(p, i, kk)) continue;
            const int key = kk.k0 + r;
            const bool key_live = r < kk.nk;
            float4 nx = bwd_col(p, kk, kk.rt_lo, sidx);
            for (int ps = 0; ok && ps < 4; ++ps, ++npass) {
                const bool dkpass = ps >= 2;
                for (int rt = kk.rt_lo; ok && rt < kk.rt_hi; ++rt, ++nrt) {
                    bwd_bar();    // every thread is done with the previous row tile's columns
                    colv[sidx] = nx;
                    bwd_bar();
                    // the next row tile's columns load while this one is computed
                    nx = bwd_col(p, kk, rt + 1 < kk.rt_hi ? rt + 1 : kk.rt_lo, sidx);
                    if (!bwd_group_wait(sdp_full, nrt & 1, abort_flag)) { ok = false; break; }
                    if (!bwd_group_wait(x_empty, (nrt & 1) ^ 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll 1
                    for (int c0 = 0; c0 < 128; c0 += 16) {
                        float sv[16], dpv[16];
                        tmem_ld16(tmem + lane_off + kBwdTmS + c0, sv);
                        if (dkpass) tmem_ld16(tmem + lane_off + kBwdTmP + c0, dpv);
                        tmem_wait_ld();
                        uint32_t pk[8];
#pragma unroll
                        for (int e = 0; e < 16; e += 2) {
                            float x[2];
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const float4 cd = colv[c0 + e + u];
                                const bool vis = r >= __float_as_int(cd.z) && r < __float_as_int(cd.w);
                                const float pr = vis ? ex2(fmaf(sv[e + u], p.scale_log2, -cd.x)) : 0.f;
                                x[u] = dkpass ? pr * (dpv[e + u] - cd.y) : pr;
                            }
                            pk[e >> 1] = pack_bf16x2(x[0], x[1]);
                        }
                        bwd_put16(xsp, r, c0, pk);
                    }
                    tc_fence_before();
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(sdp_empty);
                        mbar_arrive(x_full);
                    }
                }
                if (!ok) break;
                // ---- the pass's half of dV (ps 0, 1) or dK (ps 2, 3), added to the key's gradient
                if (!bwd_group_wait(acc_full, npass & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const float mul = dkpass ? p.scale : 1.f;
                float* base = kk.comp ? (dkpass ? p.dkc : p.dvc) : (dkpass ? p.dk : p.dv);
                const size_t rows = kk.comp ? (size_t)p.Nc : (size_t)p.T;
                float* dst = base + (((size_t)kk.b * rows + (key_live ? key : 0)) * p.Hkv + kk.g) * kBwdD + 256 * (ps & 1);
#pragma unroll 1
                for (int c0 = 0; c0 < 256; c0 += 16) {
                    float a[16];
                    tmem_ld16(tmem + lane_off + kBwdTmAcc + c0, a);
                    tmem_wait_ld();
                    if (key_live)
#pragma unroll
                        for (int e = 0; e < 16; e += 4)
                            atomicAdd(reinterpret_cast<float4*>(dst + c0 + e),
                                      make_float4(mul * a[e], mul * a[e + 1], mul * a[e + 2], mul * a[e + 3]));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acc_empty);
            }
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
