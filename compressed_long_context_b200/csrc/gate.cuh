// gate.cuh -- the low-rank gate projection of Low-Rank Gated Attention on tcgen05 (sm_100a).
//
// The attention output's gate logits are computed from the token's query latent instead of the
// hidden state (Zhidx article, section "1. Latent-Gated Sparse Attention": the latent is a
// quarter of the hidden size, so the projection has 75% fewer weights):
//     gate[n, j] = sum_k cq[n, k] * Wg[k, j],   j = h * dv + c
// cq [n, rq] bf16, Wg [rq, Hq*dv] bf16, both row-major; gate [n, Hq*dv] bf16 (fp32 accumulation,
// one rounding).  hca_decode then scales its output by sigmoid(gate).
//
// One CTA per (256 output columns, 128 latent rows): D[128 x 256] (fp32, 256 TMEM columns) =
// A[128 x rq] * B[rq x 256], A K-major (cq rows), B MN-major (Wg rows are output columns).  The
// K loop runs in stages of 64: A 128 x 64 (16 KB) and B 64 x 256 (four 8 KB boxes) per stage,
// through a 4-stage TMA ring.  At the pages' sizes (rq = 1024, Hq * dv = 32768) the weights are
// 64 MB read once, so the kernel is bound by HBM; cq stays in L2 for every CTA.
#pragma once

#include "common.cuh"

namespace hca {

constexpr int kGateThreads = 128;
constexpr int kGateStages = 4;
constexpr int kGateN = 256;                                   // output columns per CTA
constexpr uint32_t kGateABytes = 128 * 64 * 2;                // 16 KB
constexpr uint32_t kGateBBytes = 64 * kGateN * 2;             // 32 KB
constexpr uint32_t kGateStageBytes = kGateABytes + kGateBBytes;
constexpr uint32_t kGateSmBar = kGateStages * kGateStageBytes;
constexpr uint32_t kGateSmem = kGateSmBar + 256;
static_assert(kGateSmem <= 232448, "gate shared memory exceeds the per-block limit");

struct GateParams {
    __nv_bfloat16* out;   // [n, J]
    int n, rq, J;
};

__global__ void __launch_bounds__(kGateThreads, 1)
gate_logits_kernel(const GateParams p, const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b) {
    extern __shared__ __align__(1024) uint8_t dsmem[];
    if (smem_u32(dsmem) & 1023u) {
        if (threadIdx.x == 0) record_error(HCA_ERR_INTERNAL);
        return;
    }
    uint8_t* sm = dsmem;
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kGateSmBar);
    uint64_t* empty = full + kGateStages;
    uint64_t* done = empty + kGateStages;
    int* misc = reinterpret_cast<int*>(done + 1);
    volatile int* abort_flag = misc;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j0 = blockIdx.x * kGateN, m0 = blockIdx.y * 128;
    const int nk = p.rq / 64;
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int i = 0; i < kGateStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(done, 1);
        fence_mbar_init();
        prefetch_tmap(&tm_a);
        prefetch_tmap(&tm_b);
    }
    if (warp == 1) tmem_alloc(tmem_slot, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // TMA producer: stage ks = cq[m0.., 64 ks ..] and Wg[64 ks .., j0 ..] (four 64-column boxes)
            for (int ks = 0; ks < nk; ++ks) {
                const int st = ks % kGateStages;
                if (ks >= kGateStages && !mbar_wait(&empty[st], ((ks / kGateStages) - 1) & 1, abort_flag)) break;
                uint8_t* base = sm + st * kGateStageBytes;
                mbar_arrive_expect_tx(&full[st], kGateStageBytes);
                tma_load_4d(base, &tm_a, &full[st], 64 * ks, m0, 0, 0);
                for (int s = 0; s < kGateN / 64; ++s)
                    tma_load_4d(base + kGateABytes + s * 8192, &tm_b, &full[st], j0 + 64 * s, 64 * ks, 0, 0);
            }
        }
    } else if (warp == 1) {
        // MMA issuer: A K-major (SW128 rows of 64 latent values), B MN-major (SW128 rows of 64 columns)
        const uint32_t id = idesc_bf16(128, kGateN, 0, 1);
        bool ok = true;
        for (int ks = 0; ks < nk && ok; ++ks) {
            const int st = ks % kGateStages;
            if (!warp_wait(&full[st], (ks / kGateStages) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t a = smem_u32(sm + st * kGateStageBytes), b = a + kGateABytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ss(tmem, smem_desc_sw128(a + kk * 32, 16, 1024), smem_desc_sw128(b + kk * 2048, 8192, 1024), id,
                           (ks | kk) ? 1u : 0u);
                mma_commit(&empty[st]);
                if (ks == nk - 1) mma_commit(done);
            }
            __syncwarp();
        }
    }
    // epilogue, all four warps: thread = output row m0 + 32 * warp + lane
    __syncwarp();
    if (warp_wait(done, 0, abort_flag)) {
        tc_fence_after();
        const int row = m0 + 32 * warp + lane;
        const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
#pragma unroll 1
        for (int c = 0; c < kGateN; c += 16) {
            float v[16];
            tmem_ld16(tmem + lane_off + c, v);
            tmem_wait_ld();
            if (row < p.n) {
                uint4* dst = reinterpret_cast<uint4*>(p.out + (size_t)row * p.J + j0 + c);
                dst[0] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                    pack_bf16x2(v[6], v[7]));
                dst[1] = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                                    pack_bf16x2(v[14], v[15]));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

}  // namespace hca
