// hca_api.cu -- the C ABI of libhca (declared in include/hca.h): argument checks,
// TMA tensor maps and kernel launches.  Everything here is host code except the
// kernels pulled in from the .cuh files of this directory.
#include <cudaTypedefs.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "append.cuh"
#include "backward.cuh"
#include "common.cuh"
#include "compress.cuh"
#include "decode.cuh"
#include "dsa.cuh"
#include "gate.cuh"
#include "prefill.cuh"
#include "prefill_pair.cuh"
#include "vha.cuh"

namespace {

using hca::g_error;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

hca_status_t launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? HCA_OK : HCA_ERR_CUDA;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

}  // namespace

namespace hca {

// 4-D bf16 tensor map over a [d3][d2][d1][d0] array (d0 innermost, contiguous), box
// {b0, b1, b2, b3}, 128-byte swizzle (b0 * 2 bytes must be 128).  Strides are in
// elements for dims 1..3.  Returns false if the driver rejects the map.
bool make_tmap_4d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3,
                  uint64_t s1, uint64_t s2, uint64_t s3, uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {d0, d1, d2, d3};
    cuuint64_t strides[3] = {s1 * 2, s2 * 2, s3 * 2};
    cuuint32_t box[4] = {b0, b1, b2, b3};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 4-D tensor map with 128-byte swizzle for TMA stores of 128-byte rows: element type bf16
// or fp32 (esize 2 or 4); strides in elements for dims 1..3.
bool make_tmap_4d_plain(CUtensorMap* m, void* base, int esize, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3,
                        uint64_t s1, uint64_t s2, uint64_t s3, uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {d0, d1, d2, d3};
    cuuint64_t strides[3] = {s1 * esize, s2 * esize, s3 * esize};
    cuuint32_t box[4] = {b0, b1, b2, b3};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, esize == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D bf16 tensor map over `rows` rows of d0 contiguous elements, box {b0, 1} (one row high, as
// tile::gather4 copies need), 128-byte swizzle (b0 * 2 bytes must be 128).
bool make_tmap_rows(CUtensorMap* m, const void* base, uint64_t d0, uint64_t rows, uint32_t b0) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {d0, rows};
    cuuint64_t strides[1] = {d0 * 2};
    cuuint32_t box[2] = {b0, 1};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (kernel slot, device).
bool set_smem_attr_once(const void* fn, int bytes, int slot) {
    static std::mutex mu;
    static bool done[16][64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 || slot < 0 || slot >= 16) return false;
    std::lock_guard<std::mutex> g(mu);
    if (done[slot][dev]) return true;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
    done[slot][dev] = true;
    return true;
}

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

__device__ unsigned int g_error_taken = 0;

__global__ void take_error_kernel() { g_error_taken = atomicExch(&g_error, 0u); }

// One CTA that waits on an mbarrier which can never complete (two arrivals expected, one
// made), with the same bounded wait the attention kernels use: it runs out after the
// device's wait limit, records HCA_ERR_TIMEOUT and returns.  Nothing is in flight.
__global__ void wait_probe_kernel() {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(&bar, 2);
        fence_mbar_init();
        mbar_arrive(&bar);
        mbar_wait(&bar, 0, &abort_flag);
    }
    __syncthreads();
}

}  // namespace hca

extern "C" {

hca_status_t hca_debug_set_wait_limit(unsigned long long limit_ns, hca_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    static const unsigned long long kDefault = hca::kWaitLimitNs;
    const unsigned long long v = limit_ns ? limit_ns : kDefault;
    if (cudaMemcpyToSymbolAsync(hca::g_wait_limit_ns, &v, sizeof v, 0, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return HCA_ERR_CUDA;
    return HCA_OK;
}

hca_status_t hca_debug_set_drop_slab(int on, hca_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int v = on ? 1 : 0;
    if (cudaMemcpyToSymbolAsync(hca::g_debug_drop_slab, &v, sizeof v, 0, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return HCA_ERR_CUDA;
    return HCA_OK;
}

hca_status_t hca_debug_wait_probe(hca_stream_t stream) {
    hca::wait_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>();
    return launch_status();
}

const char* hca_status_string(hca_status_t s) {
    switch (s) {
        case HCA_OK: return "HCA_OK";
        case HCA_ERR_INVALID_ARG: return "HCA_ERR_INVALID_ARG: null/misaligned pointer or size out of range";
        case HCA_ERR_UNSUPPORTED: return "HCA_ERR_UNSUPPORTED: shape or flag combination not supported";
        case HCA_ERR_CUDA: return "HCA_ERR_CUDA: a CUDA launch or query failed";
        case HCA_ERR_TIMEOUT: return "HCA_ERR_TIMEOUT: a bounded device wait ran out";
        case HCA_ERR_DEVICE_INPUT: return "HCA_ERR_DEVICE_INPUT: a device-resident input was out of range";
        case HCA_ERR_INTERNAL: return "HCA_ERR_INTERNAL: a kernel found its launch environment unusable";
    }
    return "unknown hca_status_t";
}

hca_status_t hca_get_device_error(hca_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned int word = 0;
    // read and clear in one atomic step on the device, so that an error recorded by a kernel on
    // another stream between a read and a separate clear cannot be lost
    hca::take_error_kernel<<<1, 1, 0, s>>>();
    if (cudaGetLastError() != cudaSuccess) return HCA_ERR_CUDA;
    if (cudaMemcpyFromSymbolAsync(&word, hca::g_error_taken, sizeof word, 0, cudaMemcpyDeviceToHost, s) !=
        cudaSuccess)
        return HCA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return HCA_ERR_CUDA;
    if (word == HCA_ERR_TIMEOUT || word == HCA_ERR_DEVICE_INPUT || word == HCA_ERR_INTERNAL)
        return static_cast<hca_status_t>(word);
    return word == 0 ? HCA_OK : HCA_ERR_CUDA;
}

hca_status_t hca_compress(const void* k, const void* v, const float* w, void* kc, void* vc,
                          int B, int T, int Hkv, int d, int dv, int blk, hca_stream_t stream) {
    if (B < 0 || T < 0 || Hkv < 1 || blk < 1) return HCA_ERR_INVALID_ARG;
    auto ok_dim = [](int x) { return x == 64 || x == 128 || x == 256 || x == 512; };
    if (!ok_dim(d) || !ok_dim(dv) || blk > 128) return HCA_ERR_UNSUPPORTED;
    const int64_t Nc = T / blk;
    const int64_t entries = (int64_t)B * Nc * Hkv;
    if (entries == 0) return HCA_OK;
    if (entries > 0x7fffffffLL) return HCA_ERR_INVALID_ARG;
    if (!k || !v || !kc || !vc) return HCA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(kc) || !aligned16(vc) || (w && !aligned16(w)))
        return HCA_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const dim3 grid((unsigned)entries);
    const auto* K = static_cast<const __nv_bfloat16*>(k);
    const auto* V = static_cast<const __nv_bfloat16*>(v);
    auto* KC = static_cast<__nv_bfloat16*>(kc);
    auto* VC = static_cast<__nv_bfloat16*>(vc);
#define HCA_COMPRESS_CASE(DK, DV)                                                                       \
    if (d == DK && dv == DV) {                                                                          \
        hca::compress_kernel<DK, DV><<<grid, hca::kCompressThreads, 0, s>>>(K, V, w, KC, VC, T, Hkv, blk, \
                                                                            (int)Nc);                   \
        return launch_status();                                                                         \
    }
#define HCA_COMPRESS_ROW(DK) \
    HCA_COMPRESS_CASE(DK, 64) HCA_COMPRESS_CASE(DK, 128) HCA_COMPRESS_CASE(DK, 256) HCA_COMPRESS_CASE(DK, 512)
    HCA_COMPRESS_ROW(64) HCA_COMPRESS_ROW(128) HCA_COMPRESS_ROW(256) HCA_COMPRESS_ROW(512)
#undef HCA_COMPRESS_ROW
#undef HCA_COMPRESS_CASE
    return HCA_ERR_UNSUPPORTED;
}

}  // extern "C"

namespace {
template <bool F32, int RP>
hca_status_t vha_launch(const hca::VhaParams& p, cudaStream_t s) {
    const auto kern = hca::vha_kernel<F32, RP>;
    const int smem = hca::vha_smem_bytes(p.Hq, RP, F32);      // <= 32 KB: no opt-in needed
    const int sms = hca::num_sms();
    int per_sm = 0;
    if (sms <= 0 || cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, hca::kVhaThreads, smem) != cudaSuccess ||
        per_sm < 1)
        return HCA_ERR_CUDA;
    // persistent: every resident CTA slot filled once, warps stride over the work items
    const long long items = p.n * (p.dv / (F32 ? 32 : 64));
    const long long need = (items + hca::kVhaThreads / 32 - 1) / (hca::kVhaThreads / 32);
    const long long grid = std::min<long long>(need, (long long)sms * per_sm);
    kern<<<(unsigned)grid, hca::kVhaThreads, smem, s>>>(p);
    return launch_status();
}
}  // namespace

extern "C" hca_status_t hca_vha(void* out, const float* U, const float* V, long long n, int Hq, int dv, int r,
                                unsigned flags, hca_stream_t stream) {
    if (n < 0 || Hq < 1 || dv < 1 || r < 1) return HCA_ERR_INVALID_ARG;
    if (flags & ~(unsigned)HCA_OUT_F32) return HCA_ERR_UNSUPPORTED;
    if (Hq > hca::kVhaMaxHeads || r > hca::kVhaMaxRank || dv % hca::kVhaCh) return HCA_ERR_UNSUPPORTED;
    if (n == 0) return HCA_OK;
    if (!out || !U || !V || !aligned16(out) || (reinterpret_cast<uintptr_t>(U) & 3) ||
        (reinterpret_cast<uintptr_t>(V) & 3))
        return HCA_ERR_INVALID_ARG;
    hca::VhaParams p;
    p.out = out; p.U = U; p.V = V; p.n = n; p.Hq = Hq; p.dv = dv; p.r = r;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool f32 = flags & HCA_OUT_F32;
    // rank padded with zero factors to the next of 4, 8, 16, 32
    if (r <= 4) return f32 ? vha_launch<true, 4>(p, s) : vha_launch<false, 4>(p, s);
    if (r <= 8) return f32 ? vha_launch<true, 8>(p, s) : vha_launch<false, 8>(p, s);
    if (r <= 16) return f32 ? vha_launch<true, 16>(p, s) : vha_launch<false, 16>(p, s);
    return f32 ? vha_launch<true, 32>(p, s) : vha_launch<false, 32>(p, s);
}

extern "C" {

size_t hca_append_state_size(int B, int Hkv, int d, int dv) {
    if (B < 0 || Hkv < 1 || d < 0 || dv < 0) return 0;
    return (size_t)B * Hkv * (size_t)(hca::kAppendHeader + d + dv) * sizeof(float);
}

hca_status_t hca_append(const void* k_new, const void* v_new, const float* w_new, const int* seqlens, void* kw,
                        void* vw, void* kc, void* vc, const int* page_table, int page_size, int max_pages,
                        int num_pages, void* state, int B, int Hkv, int d, int dv, int blk, int W, int Nmax,
                        unsigned flags, hca_stream_t stream) {
    if (B < 0 || Hkv < 1 || blk < 1 || W < 1) return HCA_ERR_INVALID_ARG;
    if (flags & ~(unsigned)HCA_PAGED) return HCA_ERR_UNSUPPORTED;
    auto ok_dim = [](int x) { return x == 64 || x == 128 || x == 256 || x == 512; };
    if (!ok_dim(d) || !ok_dim(dv) || blk > 128) return HCA_ERR_UNSUPPORTED;
    if (B == 0) return HCA_OK;
    if ((long long)B * Hkv > 0x7fffffffLL) return HCA_ERR_INVALID_ARG;
    const bool paged = flags & HCA_PAGED;
    if (!k_new || !v_new || !seqlens || !kw || !vw || !kc || !vc || !state) return HCA_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(kw) || !aligned16(vw) || !aligned16(kc) ||
        !aligned16(vc) || !aligned16(state) || (reinterpret_cast<uintptr_t>(seqlens) & 3) ||
        (w_new && (reinterpret_cast<uintptr_t>(w_new) & 3)))
        return HCA_ERR_INVALID_ARG;
    if (paged) {
        if (!page_table || page_size < 64 || page_size % 64 || max_pages < 1 || num_pages < 1 ||
            (reinterpret_cast<uintptr_t>(page_table) & 3))
            return HCA_ERR_INVALID_ARG;
    } else if (Nmax < 1) {
        return HCA_ERR_INVALID_ARG;
    }
    hca::AppendParams p;
    p.k_new = static_cast<const __nv_bfloat16*>(k_new);
    p.v_new = static_cast<const __nv_bfloat16*>(v_new);
    p.w = w_new;
    p.seqlens = seqlens;
    p.kw = static_cast<__nv_bfloat16*>(kw);
    p.vw = static_cast<__nv_bfloat16*>(vw);
    p.kc = static_cast<__nv_bfloat16*>(kc);
    p.vc = static_cast<__nv_bfloat16*>(vc);
    p.page_table = paged ? page_table : nullptr;
    p.state = static_cast<float*>(state);
    p.B = B; p.Hkv = Hkv; p.d = d; p.dv = dv; p.blk = blk; p.W = W;
    p.Nmax = paged ? 0 : Nmax;
    p.page_size = paged ? page_size : 0; p.max_pages = paged ? max_pages : 0; p.num_pages = paged ? num_pages : 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    hca::append_kernel<<<(unsigned)(B * Hkv), hca::kAppendThreads, 0, s>>>(p);
    return launch_status();
}

}  // extern "C"

namespace {

// Workspace layout of hca_decode: [header 256 B: total tiles][meta: U x 2 int][records]
struct DecodeWs {
    size_t meta_off, m_off, l_off, o_off, bytes;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

DecodeWs decode_ws_layout(long long U, long long nsplit) {
    DecodeWs w;
    const long long R = nsplit + U;
    w.meta_off = 256;
    w.m_off = align256(w.meta_off + (size_t)U * 2 * sizeof(int));
    w.l_off = align256(w.m_off + (size_t)R * 64 * sizeof(float));
    w.o_off = align256(w.l_off + (size_t)R * 64 * sizeof(float));
    w.bytes = align256(w.o_off + (size_t)R * 64 * hca::kDecD * sizeof(float));
    return w;
}

}  // namespace

extern "C" {

size_t hca_decode_workspace_size(int B, int Hq, int Hkv, int dv) {
    if (B < 0 || Hq < 1 || Hkv < 1 || dv < 1) return 0;
    const int ns = hca::num_sms();
    if (ns <= 0) return 0;
    return decode_ws_layout((long long)B * Hkv, ns).bytes;
}

}  // extern "C"

namespace {

// hca_decode and hca_decode_vha: the split kernel, then the combine kernel (merge, gate and,
// with factors, Virtual Head Attention).
hca_status_t decode_impl(const void* q, const void* kc, const void* vc, const int* page_table, int page_size,
                         int max_pages, int num_pages, const void* kw, const void* vw, const int* seqlens,
                         const float* gq, const float* gk, float eps, const void* gate, float* out,
                         void* workspace, size_t ws_bytes, int B, int Hq, int Hkv, int d, int dv, int blk, int W,
                         int Nmax, float scale, unsigned flags, const float* vha_u, const float* vha_v, int vha_r,
                         hca_stream_t stream) {
    using namespace hca;
    if (B < 0 || Hq < 1 || Hkv < 1 || blk < 1 || W < 1) return HCA_ERR_INVALID_ARG;
    if (flags & ~(unsigned)(HCA_QK_NORM | HCA_OUT_GATE | HCA_PAGED | HCA_WINDOW_RING)) return HCA_ERR_UNSUPPORTED;
    if (d != kDecD || dv != kDecD || Hq % Hkv != 0 || Hq / Hkv > kDecHeads || blk > 128)
        return HCA_ERR_UNSUPPORTED;
    if (!(scale == scale) || !(eps >= 0.f)) return HCA_ERR_INVALID_ARG;
    if (B == 0) return HCA_OK;
    const bool paged = flags & HCA_PAGED;
    const bool norm = flags & HCA_QK_NORM;
    const bool gated = flags & HCA_OUT_GATE;
    if (!q || !kc || !vc || !kw || !vw || !seqlens || !out || !workspace) return HCA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(kc) || !aligned16(vc) || !aligned16(kw) || !aligned16(vw) ||
        !aligned16(out) || !aligned16(workspace) || (reinterpret_cast<uintptr_t>(seqlens) & 3))
        return HCA_ERR_INVALID_ARG;
    if (paged) {
        if (!page_table || page_size < 64 || page_size % 64 || max_pages < 1 || num_pages < 1)
            return HCA_ERR_INVALID_ARG;
        if (reinterpret_cast<uintptr_t>(page_table) & 3) return HCA_ERR_INVALID_ARG;
    } else if (Nmax < 1) {
        return HCA_ERR_INVALID_ARG;
    }
    if (norm && (!gq || !gk || (reinterpret_cast<uintptr_t>(gq) & 3) || (reinterpret_cast<uintptr_t>(gk) & 3)))
        return HCA_ERR_INVALID_ARG;
    if (gated && (!gate || !aligned16(gate))) return HCA_ERR_INVALID_ARG;   // read 16 bytes per thread
    if (vha_u || vha_v) {
        if (!vha_u || !vha_v || vha_r < 1 || (reinterpret_cast<uintptr_t>(vha_u) & 3) ||
            (reinterpret_cast<uintptr_t>(vha_v) & 3))
            return HCA_ERR_INVALID_ARG;
        // the mixing spans all Hq heads of a token: one KV group must hold them all
        if (Hkv != 1 || vha_r > kDecVhaMaxRank) return HCA_ERR_UNSUPPORTED;
    }
    const int nsplit = num_sms();
    if (nsplit <= 0) return HCA_ERR_CUDA;
    const long long U = (long long)B * Hkv;
    if (U > (1 << 24)) return HCA_ERR_INVALID_ARG;
    const DecodeWs lay = decode_ws_layout(U, nsplit);
    if (ws_bytes < lay.bytes) return HCA_ERR_INVALID_ARG;

    const uint64_t hd = (uint64_t)Hkv * kDecD;
    CUtensorMap tq, tk, tv, tkw, tvw;
    bool ok = true;
    // queries [B, Hq, 512]: a box of 64 heads starting at the group's first head
    ok &= make_tmap_4d(&tq, q, kDecD, Hq, B, 1, kDecD, (uint64_t)Hq * kDecD, (uint64_t)B * Hq * kDecD, 64, 64, 1, 1);
    if (paged) {
        ok &= make_tmap_4d(&tk, kc, kDecD, Hkv, page_size, num_pages, kDecD, hd, hd * page_size, 64, 1, 64, 1);
        ok &= make_tmap_4d(&tv, vc, kDecD, Hkv, page_size, num_pages, kDecD, hd, hd * page_size, 64, 1, 64, 1);
    } else {
        ok &= make_tmap_4d(&tk, kc, kDecD, Hkv, Nmax, B, kDecD, hd, hd * Nmax, 64, 1, 128, 1);
        ok &= make_tmap_4d(&tv, vc, kDecD, Hkv, Nmax, B, kDecD, hd, hd * Nmax, 64, 1, 128, 1);
    }
    ok &= make_tmap_4d(&tkw, kw, kDecD, Hkv, W, B, kDecD, hd, hd * W, 64, 1, 128, 1);
    ok &= make_tmap_4d(&tvw, vw, kDecD, Hkv, W, B, kDecD, hd, hd * W, 64, 1, 128, 1);
    if (!ok) return HCA_ERR_CUDA;

    DecodeParams p;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.seqlens = seqlens;
    p.page_table = paged ? page_table : nullptr;
    p.gq = norm ? gq : nullptr;
    p.gk = norm ? gk : nullptr;
    p.gate = gated ? static_cast<const __nv_bfloat16*>(gate) : nullptr;
    p.out = out;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p.total = reinterpret_cast<long long*>(ws);
    p.meta = reinterpret_cast<int*>(ws + lay.meta_off);
    p.rec_m = reinterpret_cast<float*>(ws + lay.m_off);
    p.rec_l = reinterpret_cast<float*>(ws + lay.l_off);
    p.rec_o = reinterpret_cast<float*>(ws + lay.o_off);
    p.vha_u = vha_u;
    p.vha_v = vha_v;
    p.vha_r = vha_u ? vha_r : 0;
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.G = Hq / Hkv; p.blk = blk; p.W = W; p.Nmax = paged ? 0 : Nmax;
    p.page_size = paged ? page_size : 0; p.max_pages = paged ? max_pages : 0; p.num_pages = paged ? num_pages : 0;
    p.flags = (int)flags; p.nsplit = nsplit;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.eps = eps;

    // compile-time variants: QK normalisation x paged cache
    using SplitFn = void (*)(const DecodeParams, const CUtensorMap, const CUtensorMap, const CUtensorMap,
                             const CUtensorMap, const CUtensorMap);
    const SplitFn split = norm ? (paged ? decode_split_kernel<true, true> : decode_split_kernel<true, false>)
                               : (paged ? decode_split_kernel<false, true> : decode_split_kernel<false, false>);
    if (!set_smem_attr_once(reinterpret_cast<const void*>(split), (int)kDecSmemBytes, 4 + 2 * norm + paged))
        return HCA_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    split<<<nsplit, kDecThreads, kDecSmemBytes, s>>>(p, tq, tk, tv, tkw, tvw);
    if (cudaGetLastError() != cudaSuccess) return HCA_ERR_CUDA;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)U, (unsigned)(kDecD / kMergeCh));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = p.vha_u ? combine_vha_smem(p.vha_r) : 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // records loaded per round, from the average number of pieces per unit (about nsplit / U)
    const int chunk = (long long)nsplit >= 6 * U ? 8 : ((long long)nsplit >= 3 * U ? 4 : 2);
    cudaError_t e;
    if (p.vha_u)
        e = chunk == 8 ? cudaLaunchKernelEx(&cfg, decode_combine_kernel<8, true>, p)
            : chunk == 4 ? cudaLaunchKernelEx(&cfg, decode_combine_kernel<4, true>, p)
                         : cudaLaunchKernelEx(&cfg, decode_combine_kernel<2, true>, p);
    else
        e = chunk == 8 ? cudaLaunchKernelEx(&cfg, decode_combine_kernel<8, false>, p)
            : chunk == 4 ? cudaLaunchKernelEx(&cfg, decode_combine_kernel<4, false>, p)
                         : cudaLaunchKernelEx(&cfg, decode_combine_kernel<2, false>, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return HCA_ERR_CUDA;
    }
    return HCA_OK;
}

}  // namespace

extern "C" {

hca_status_t hca_decode(const void* q, const void* kc, const void* vc, const int* page_table, int page_size,
                        int max_pages, int num_pages, const void* kw, const void* vw, const int* seqlens,
                        const float* gq, const float* gk, float eps, const void* gate, float* out,
                        void* workspace, size_t ws_bytes, int B, int Hq, int Hkv, int d, int dv, int blk, int W,
                        int Nmax, float scale, unsigned flags, hca_stream_t stream) {
    return decode_impl(q, kc, vc, page_table, page_size, max_pages, num_pages, kw, vw, seqlens, gq, gk, eps, gate,
                       out, workspace, ws_bytes, B, Hq, Hkv, d, dv, blk, W, Nmax, scale, flags, nullptr, nullptr, 0,
                       stream);
}

hca_status_t hca_decode_vha(const void* q, const void* kc, const void* vc, const int* page_table, int page_size,
                            int max_pages, int num_pages, const void* kw, const void* vw, const int* seqlens,
                            const float* gq, const float* gk, float eps, const void* gate, const float* vha_u,
                            const float* vha_v, int vha_rank, float* out, void* workspace, size_t ws_bytes, int B,
                            int Hq, int Hkv, int d, int dv, int blk, int W, int Nmax, float scale, unsigned flags,
                            hca_stream_t stream) {
    if (!vha_u || !vha_v) return HCA_ERR_INVALID_ARG;
    return decode_impl(q, kc, vc, page_table, page_size, max_pages, num_pages, kw, vw, seqlens, gq, gk, eps, gate,
                       out, workspace, ws_bytes, B, Hq, Hkv, d, dv, blk, W, Nmax, scale, flags, vha_u, vha_v,
                       vha_rank, stream);
}

}  // extern "C"

namespace {

template <int D>
hca_status_t launch_prefill(const hca::PrefillParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                            const CUtensorMap& tv, const CUtensorMap& tkc, const CUtensorMap& tvc,
                            cudaStream_t s) {
    using C = hca::PfCfg<D>;
    if (!hca::set_smem_attr_once(reinterpret_cast<const void*>(&hca::prefill_kernel<D>), (int)C::kSmem,
                                 D == 512 ? 1 : 2))
        return HCA_ERR_CUDA;
    const int ns = hca::num_sms();
    if (ns <= 0) return HCA_ERR_CUDA;
    const long long grid = p.items < ns ? p.items : ns;
    hca::prefill_kernel<D><<<(unsigned)grid, hca::kPfThreads, C::kSmem, s>>>(p, tq, tk, tv, tkc, tvc);
    return cudaGetLastError() == cudaSuccess ? HCA_OK : HCA_ERR_CUDA;
}

// Clusters of two CTAs (one per SM) that can be resident at once on the current device.
int pair_clusters_resident(cudaStream_t s) {
    static std::mutex mu;
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> g(mu);
    if (cached[dev] > 0) return cached[dev];
    // the occupancy query needs the kernel's shared-memory opt-in in place
    if (!hca::set_smem_attr_once(reinterpret_cast<const void*>(&hca::prefill_pair_kernel), (int)hca::kPpSmem, 3))
        return 0;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * 74, 1, 1);
    cfg.blockDim = dim3(hca::kPpThreads, 1, 1);
    cfg.dynamicSmemBytes = hca::kPpSmem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(&hca::prefill_pair_kernel), &cfg) !=
        cudaSuccess)
        return 0;
    cached[dev] = n;
    return n;
}

hca_status_t launch_prefill_pair(const hca::PrefillParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                                 const CUtensorMap& tv, const CUtensorMap& tkc, const CUtensorMap& tvc,
                                 const CUtensorMap& tout, cudaStream_t s) {
    if (!hca::set_smem_attr_once(reinterpret_cast<const void*>(&hca::prefill_pair_kernel), (int)hca::kPpSmem, 3))
        return HCA_ERR_CUDA;
    const int nc = pair_clusters_resident(s);
    if (nc <= 0) return HCA_ERR_CUDA;
    const long long npairs = p.items < nc ? p.items : nc;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)(2 * npairs), 1, 1);
    cfg.blockDim = dim3(hca::kPpThreads, 1, 1);
    cfg.dynamicSmemBytes = hca::kPpSmem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, hca::prefill_pair_kernel, p, tq, tk, tv, tkc, tvc, tout) != cudaSuccess) {
        cudaGetLastError();
        return HCA_ERR_CUDA;
    }
    return HCA_OK;
}

}  // namespace

extern "C" hca_status_t hca_prefill(const void* q, const void* k, const void* v, const void* kc, const void* vc,
                                    void* out, float* lse,
                                    int B, int T, int Hq, int Hkv, int d, int dv, int blk,
                                    int W, float scale, unsigned flags, hca_stream_t stream) {
    using namespace hca;
    if (B < 0 || T < 0 || Hq < 1 || Hkv < 1 || blk < 1 || W < 1) return HCA_ERR_INVALID_ARG;
    if (flags & ~(unsigned)(HCA_WRITE_LSE | HCA_OUT_F32)) return HCA_ERR_UNSUPPORTED;
    if (d != dv || (d != 64 && d != 512) || blk > 128 || Hq % Hkv) return HCA_ERR_UNSUPPORTED;
    const int G = Hq / Hkv;
    if (G > 128 || (G & (G - 1))) return HCA_ERR_UNSUPPORTED;
    if (!(scale == scale)) return HCA_ERR_INVALID_ARG;
    if ((long long)B * T == 0) return HCA_OK;
    const int Nc = T / blk;
    const bool want_lse = flags & HCA_WRITE_LSE;
    if (!q || !k || !v || !out || (Nc > 0 && (!kc || !vc)) || (want_lse && !lse)) return HCA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || (Nc > 0 && (!aligned16(kc) ||
        !aligned16(vc))) || (want_lse && (reinterpret_cast<uintptr_t>(lse) & 3)))
        return HCA_ERR_INVALID_ARG;

    PrefillParams p;
    p.out = out;
    p.lse = want_lse ? lse : nullptr;
    p.B = B; p.T = T; p.Hq = Hq; p.Hkv = Hkv; p.G = G; p.tpt = 128 / G; p.blk = blk; p.W = W; p.Nc = Nc;
    p.ntile_t = (T + p.tpt - 1) / p.tpt;
    p.flags = (int)flags;
    // d = 512: one item per row tile, processed by a CTA pair; d = 64: one CTA per row tile
    p.items = (long long)p.ntile_t * B * Hkv;
    p.scale_log2 = scale * 1.4426950408889634f;

    const uint64_t D = (uint64_t)d;
    CUtensorMap tq, tk, tv, tkc, tvc;
    bool ok = true;
    ok &= make_tmap_4d(&tq, q, D, Hq, T, B, D, D * Hq, D * Hq * T, 64, G, p.tpt, 1);
    // key rows per TMA box: 256 for K (and 64 for V) on the pair kernel, 128 otherwise
    const uint32_t kbox = d == 512 ? 256 : 128, vbox = d == 512 ? 64 : 128;
    ok &= make_tmap_4d(&tk, k, D, Hkv, T, B, D, D * Hkv, D * Hkv * T, 64, 1, kbox, 1);
    ok &= make_tmap_4d(&tv, v, D, Hkv, T, B, D, D * Hkv, D * Hkv * T, 64, 1, vbox, 1);
    if (Nc > 0) {
        ok &= make_tmap_4d(&tkc, kc, D, Hkv, Nc, B, D, D * Hkv, D * Hkv * Nc, 64, 1, kbox, 1);
        ok &= make_tmap_4d(&tvc, vc, D, Hkv, Nc, B, D, D * Hkv, D * Hkv * Nc, 64, 1, vbox, 1);
    } else {   // never read: no entry is visible when T < blk
        tkc = tk;
        tvc = tv;
    }
    if (!ok) return HCA_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (d != 512) return launch_prefill<64>(p, tq, tk, tv, tkc, tvc, s);
    // output boxes of 32 rows x 128 bytes: the 32 rows of a warp are (tokens, heads) in order
    CUtensorMap tout;
    const uint32_t bh = G < 32 ? (uint32_t)G : 32u, bt = 32u / bh;
    const int es = (flags & HCA_OUT_F32) ? 4 : 2;
    if (!make_tmap_4d_plain(&tout, out, es, D, Hq, T, B, D, D * Hq, D * Hq * T, 128 / es, bh, bt, 1))
        return HCA_ERR_CUDA;
    return launch_prefill_pair(p, tq, tk, tv, tkc, tvc, tout, s);
}


// ---------------------------------------------------------------------------------------
// hca_decode_noalloc: hca_decode with library-owned scratch.
//
// The split records live in a fixed array in the library's device image instead of a
// caller-provided workspace, for callers that cannot allocate device memory when they
// decode.  Host code must not pass the array's name to a kernel (on the host it is only
// a stand-in for the symbol); its device address is looked up once per device.
static __device__ __align__(256) unsigned char hca_decode_scratch[HCA_DECODE_NOALLOC_MAX_BYTES];

namespace {

std::mutex g_scratch_mu;
void* g_scratch_addr[64] = {};

// Device address of hca_decode_scratch on the current device; nullptr on failure.
void* decode_scratch_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> g(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, hca_decode_scratch) != cudaSuccess || !ptr) {
            cudaGetLastError();
            return nullptr;
        }
        g_scratch_addr[dev] = ptr;
    }
    return g_scratch_addr[dev];
}

}  // namespace

extern "C" hca_status_t hca_decode_noalloc(const void* q, const void* kc, const void* vc, const int* page_table,
                                           int page_size, int max_pages, int num_pages, const void* kw,
                                           const void* vw, const int* seqlens, const float* gq, const float* gk,
                                           float eps, const void* gate, float* out, int B, int Hq, int Hkv, int d,
                                           int dv, int blk, int W, int Nmax, float scale, unsigned flags,
                                           hca_stream_t stream) {
    if (B < 0 || Hq < 1 || Hkv < 1 || dv < 1) return HCA_ERR_INVALID_ARG;
    if (B == 0) return HCA_OK;
    const size_t need = hca_decode_workspace_size(B, Hq, Hkv, dv);
    if (need == 0) return HCA_ERR_CUDA;
    if (need > (size_t)HCA_DECODE_NOALLOC_MAX_BYTES) return HCA_ERR_INVALID_ARG;
    void* ws = decode_scratch_address();
    if (!ws) return HCA_ERR_CUDA;
    return hca_decode(q, kc, vc, page_table, page_size, max_pages, num_pages, kw, vw, seqlens, gq, gk, eps, gate,
                      out, ws, (size_t)HCA_DECODE_NOALLOC_MAX_BYTES, B, Hq, Hkv, d, dv, blk, W, Nmax, scale, flags,
                      stream);
}

// ---------------------------------------------------------------------------------------
// hca_gate_logits: the low-rank gate projection (gate.cuh).
extern "C" hca_status_t hca_gate_logits(const void* cq, const void* wg, void* gate, int n, int rq, int Hq, int dv,
                                        hca_stream_t stream) {
    if (n < 0 || rq < 1 || Hq < 1 || dv < 1) return HCA_ERR_INVALID_ARG;
    const long long J = (long long)Hq * dv;
    if (rq % 64 || J % hca::kGateN || J > 0x7fffffffLL) return HCA_ERR_UNSUPPORTED;
    if (n == 0) return HCA_OK;
    if (!cq || !wg || !gate || !aligned16(cq) || !aligned16(wg) || !aligned16(gate)) return HCA_ERR_INVALID_ARG;
    CUtensorMap ta, tb;
    // cq [n][rq]: boxes of 64 latent values x 128 rows (rows past n read as zero)
    if (!hca::make_tmap_4d(&ta, cq, (uint64_t)rq, (uint64_t)n, 1, 1, (uint64_t)rq, (uint64_t)rq * n, (uint64_t)rq * n,
                           64, 128, 1, 1))
        return HCA_ERR_CUDA;
    // Wg [rq][J]: boxes of 64 output columns x 64 latent rows
    if (!hca::make_tmap_4d(&tb, wg, (uint64_t)J, (uint64_t)rq, 1, 1, (uint64_t)J, (uint64_t)J * rq, (uint64_t)J * rq, 64,
                           64, 1, 1))
        return HCA_ERR_CUDA;
    if (!hca::set_smem_attr_once(reinterpret_cast<const void*>(&hca::gate_logits_kernel), (int)hca::kGateSmem, 0))
        return HCA_ERR_CUDA;
    hca::GateParams p;
    p.out = static_cast<__nv_bfloat16*>(gate);
    p.n = n;
    p.rq = rq;
    p.J = (int)J;
    const dim3 grid((unsigned)(J / hca::kGateN), (unsigned)((n + 127) / 128));
    hca::gate_logits_kernel<<<grid, hca::kGateThreads, hca::kGateSmem, reinterpret_cast<cudaStream_t>(stream)>>>(p, ta, tb);
    return launch_status();
}

// ---------------------------------------------------------------------------------------
// hca_prefill_backward: the layer's gradients (backward.cuh).
namespace {

size_t bwd_align(size_t x) { return (x + 255) & ~(size_t)255; }

// Bytes of P / dS records one segment may hold: the records of a segment are written by its dq
// launch and read by its dk/dv launch, so this bounds the workspace whatever the length.
constexpr size_t kBwdRecordCap = (size_t)2 << 30;

// Row tiles per segment forced by hca_debug_set_backward_segment (0: from the cap).
std::atomic<int> g_bwd_seg_rows{0};

struct BwdLayout {
    int tpt, ntile, nkc, nkw, nt_max, seg;
    size_t drow, dkc, dvc, rec, total;
};

BwdLayout bwd_layout(long long B, long long T, long long Hq, long long Hkv, long long blk, long long W) {
    BwdLayout l;
    const long long Nc = T / blk;
    l.tpt = (int)(128 / (Hq / Hkv));
    l.ntile = (int)((T + l.tpt - 1) / l.tpt);
    l.nkc = (int)((Nc + 127) / 128);
    l.nkw = (int)((T + 127) / 128);
    // key tiles of one row tile: the entry tiles, then the 128-aligned raw tiles that hold the
    // windows of its tpt tokens
    const long long nwt = std::min<long long>((l.tpt + W - 2) / 128 + 2, l.nkw);
    l.nt_max = (int)(l.nkc + nwt);
    const long long per_row_tile = B * Hkv * (long long)l.nt_max * hca::kBwdRec;
    l.seg = (int)std::max<long long>(1, std::min<long long>(l.ntile, (long long)(kBwdRecordCap / per_row_tile)));
    const int forced = g_bwd_seg_rows.load();
    if (forced > 0) l.seg = std::min(l.seg, forced);
    l.drow = 0;
    l.dkc = bwd_align((size_t)(B * T * Hq) * 4);
    l.dvc = l.dkc + bwd_align((size_t)(B * Nc * Hkv * hca::kBwdD) * 4);
    l.rec = l.dvc + bwd_align((size_t)(B * Nc * Hkv * hca::kBwdD) * 4);
    l.total = l.rec + (size_t)per_row_tile * l.seg;
    return l;
}

}  // namespace

namespace {
// Row bound of one attention launch's key / value maps forced by hca_debug_set_dsa_rows_limit
// (0: 2^31 - 1, the 32-bit coordinate range).
std::atomic<long long> g_dsa_rows_limit{0};
}  // namespace

extern "C" hca_status_t hca_debug_set_dsa_rows_limit(long long rows) {
    if (rows < 0) return HCA_ERR_INVALID_ARG;
    g_dsa_rows_limit.store(rows);
    return HCA_OK;
}

extern "C" hca_status_t hca_debug_set_backward_segment(int rows) {
    if (rows < 0) return HCA_ERR_INVALID_ARG;
    g_bwd_seg_rows.store(rows);
    return HCA_OK;
}

extern "C" size_t hca_prefill_backward_workspace_size(int B, int T, int Hq, int Hkv, int dv, int blk, int W) {
    if (B < 0 || T < 0 || Hq < 1 || Hkv < 1 || dv != hca::kBwdD || blk < 1 || W < 1 || Hq % Hkv) return 0;
    const int G = Hq / Hkv;
    if (G > 128 || (G & (G - 1))) return 0;
    return bwd_layout(B, T, Hq, Hkv, blk, W).total;
}

extern "C" hca_status_t hca_prefill_backward(const void* q, const void* k, const void* v, const float* w,
                                             const void* kc, const void* vc, const void* out, const float* lse,
                                             const void* dout, float* dq, float* dk, float* dv, float* dw,
                                             void* workspace, size_t workspace_bytes, int B, int T, int Hq, int Hkv,
                                             int d, int dv_dim, int blk, int W, float scale, unsigned flags,
                                             hca_stream_t stream) {
    using namespace hca;
    if (B < 0 || T < 0 || Hq < 1 || Hkv < 1 || blk < 1 || W < 1) return HCA_ERR_INVALID_ARG;
    if (flags & ~(unsigned)HCA_OUT_F32) return HCA_ERR_UNSUPPORTED;
    if (d != kBwdD || dv_dim != kBwdD || blk > 128 || Hq % Hkv) return HCA_ERR_UNSUPPORTED;
    const int G = Hq / Hkv;
    if (G > 128 || (G & (G - 1))) return HCA_ERR_UNSUPPORTED;
    if (!(scale == scale)) return HCA_ERR_INVALID_ARG;
    if ((long long)B * T == 0) return HCA_OK;
    const int Nc = T / blk;
    if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv || !workspace || (Nc > 0 && (!kc || !vc)))
        return HCA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv) || (Nc > 0 && (!aligned16(kc) || !aligned16(vc))) ||
        (reinterpret_cast<uintptr_t>(lse) & 3) || (w && (reinterpret_cast<uintptr_t>(w) & 3)) ||
        (dw && (reinterpret_cast<uintptr_t>(dw) & 3)) || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return HCA_ERR_INVALID_ARG;
    const BwdLayout lay = bwd_layout(B, T, Hq, Hkv, blk, W);
    if (workspace_bytes < lay.total) return HCA_ERR_INVALID_ARG;
    const int ns = num_sms();
    if (ns <= 0) return HCA_ERR_CUDA;

    BwdParams p;
    char* ws = static_cast<char*>(workspace);
    p.lse = lse;
    p.drow = reinterpret_cast<float*>(ws + lay.drow);
    p.out = out;
    p.dout = static_cast<const __nv_bfloat16*>(dout);
    p.k = static_cast<const __nv_bfloat16*>(k);
    p.v = static_cast<const __nv_bfloat16*>(v);
    p.w = w;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.dkc = reinterpret_cast<float*>(ws + lay.dkc);
    p.dvc = reinterpret_cast<float*>(ws + lay.dvc);
    p.dw = dw;
    p.rec = reinterpret_cast<uint8_t*>(ws + lay.rec);
    p.B = B; p.T = T; p.Hq = Hq; p.Hkv = Hkv; p.G = G; p.tpt = lay.tpt; p.blk = blk; p.W = W; p.Nc = Nc;
    p.ntile_t = lay.ntile;
    p.out_f32 = (flags & HCA_OUT_F32) ? 1 : 0;
    p.nkc = lay.nkc;
    p.nkw = lay.nkw;
    p.nt_max = lay.nt_max;
    p.seg = lay.seg;
    // row tiles per item of an entry tile: about the rows a raw key tile reaches, so that items
    // are of similar length
    const int raw_span = (127 + W - 1) / p.tpt + 2;
    p.ch_rows = std::max(16, std::min(128, raw_span));
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;

    const uint64_t D = kBwdD;
    CUtensorMap tq, tdo, tk, tv, tkc, tvc;
    bool ok = true;
    ok &= make_tmap_4d(&tq, q, D, Hq, T, B, D, D * Hq, D * Hq * T, 64, G, p.tpt, 1);
    ok &= make_tmap_4d(&tdo, dout, D, Hq, T, B, D, D * Hq, D * Hq * T, 64, G, p.tpt, 1);
    ok &= make_tmap_4d(&tk, k, D, Hkv, T, B, D, D * Hkv, D * Hkv * T, 64, 1, 128, 1);
    ok &= make_tmap_4d(&tv, v, D, Hkv, T, B, D, D * Hkv, D * Hkv * T, 64, 1, 128, 1);
    if (Nc > 0) {
        ok &= make_tmap_4d(&tkc, kc, D, Hkv, Nc, B, D, D * Hkv, D * Hkv * Nc, 64, 1, 128, 1);
        ok &= make_tmap_4d(&tvc, vc, D, Hkv, Nc, B, D, D * Hkv, D * Hkv * Nc, 64, 1, 128, 1);
    } else {   // never read: no entry exists when T < blk
        tkc = tk;
        tvc = tv;
    }
    if (!ok) return HCA_ERR_CUDA;
    if (!set_smem_attr_once(reinterpret_cast<const void*>(&bwd_dq_kernel), (int)kBwdSmem, 8) ||
        !set_smem_attr_once(reinterpret_cast<const void*>(&bwd_dkv_kernel), (int)kBwdSmem, 9))
        return HCA_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const long long rows = (long long)B * T * Hq;
    const long long pre_grid = std::min<long long>((rows + 7) / 8, 8LL * ns);
    bwd_pre_kernel<<<(unsigned)pre_grid, 256, 0, s>>>(p);
    for (int s0 = 0; s0 < p.ntile_t; s0 += p.seg) {
        p.s0 = s0;
        p.s1 = std::min(p.ntile_t, s0 + p.seg);
        p.dq_items = (long long)B * Hkv * (p.s1 - s0);
        p.nch = (p.s1 - s0 + p.ch_rows - 1) / p.ch_rows;
        const long long num = (long long)s0 * p.tpt - 126 - W;
        p.kta = num > 0 ? (int)(num / 128) : 0;
        const int ktb = std::min(p.nkw - 1, (int)(((long long)p.s1 * p.tpt - 1) / 128));
        p.nraw = std::max(0, ktb - p.kta + 1);
        p.kv_items = (long long)B * Hkv * (2LL * p.nkc * p.nch + 2LL * p.nraw);
        bwd_dq_kernel<<<(unsigned)std::min<long long>(p.dq_items, ns), kDqThreads, kBwdSmem, s>>>(p, tq, tdo, tk, tv,
                                                                                                  tkc, tvc);
        if (p.kv_items > 0)
            bwd_dkv_kernel<<<(unsigned)std::min<long long>(p.kv_items, ns), kKvThreads, kBwdSmem, s>>>(p, tq, tdo);
    }
    if (Nc > 0) bwd_pool_kernel<<<(unsigned)((long long)B * Nc), kPoolThreads, 0, s>>>(p);
    return launch_status();
}

// ---------------------------------------------------------------------------------------
// The sparse-attention decode step (dsa.cuh): indexer scores, top-k selection, core attention.
extern "C" hca_status_t hca_dsa_index(const void* q_idx, const float* w_idx, const void* k_idx, const int* seqlens,
                                      float* scores, int B, int HI, int dI, int Lmax, hca_stream_t stream) {
    using namespace hca;
    if (B < 0 || Lmax < 1 || HI < 1) return HCA_ERR_INVALID_ARG;
    if (dI != kDsaDI || HI % 16 || HI > kDsaMaxHI) return HCA_ERR_UNSUPPORTED;
    if (B == 0) return HCA_OK;
    if (!q_idx || !w_idx || !k_idx || !seqlens || !scores || !aligned16(q_idx) || !aligned16(k_idx) ||
        (reinterpret_cast<uintptr_t>(w_idx) & 3) || (reinterpret_cast<uintptr_t>(seqlens) & 3) ||
        (reinterpret_cast<uintptr_t>(scores) & 3))
        return HCA_ERR_INVALID_ARG;
    const int ns = num_sms();
    if (ns <= 0) return HCA_ERR_CUDA;
    CUtensorMap tq, tk;
    bool ok = make_tmap_4d(&tq, q_idx, kDsaDI, HI, B, 1, kDsaDI, (uint64_t)kDsaDI * HI, (uint64_t)kDsaDI * HI * B, 64, HI, 1, 1);
    ok &= make_tmap_4d(&tk, k_idx, kDsaDI, Lmax, B, 1, kDsaDI, (uint64_t)kDsaDI * Lmax, (uint64_t)kDsaDI * Lmax * B, 64, 128,
                       1, 1);
    if (!ok) return HCA_ERR_CUDA;
    if (!set_smem_attr_once(reinterpret_cast<const void*>(&dsa_index_kernel), (int)kIdxSmem, 10)) return HCA_ERR_CUDA;
    DsaIndexParams p;
    p.w = w_idx;
    p.seqlens = seqlens;
    p.scores = scores;
    p.B = B; p.HI = HI; p.Lmax = Lmax; p.ntile = (Lmax + 127) / 128;
    p.total = (long long)B * p.ntile;
    const long long grid = std::min<long long>(p.total, 2LL * ns);   // two CTAs per SM
    dsa_index_kernel<<<(unsigned)grid, kIdxThreads, kIdxSmem, reinterpret_cast<cudaStream_t>(stream)>>>(p, tq, tk);
    return launch_status();
}

extern "C" hca_status_t hca_dsa_topk(const float* scores, const int* seqlens, int* idx, int B, int Lmax, int k,
                                     hca_stream_t stream) {
    using namespace hca;
    if (B < 0 || Lmax < 1 || k < 1 || B > (1 << 28)) return HCA_ERR_INVALID_ARG;
    if (B == 0) return HCA_OK;
    if (!scores || !seqlens || !idx || (reinterpret_cast<uintptr_t>(scores) & 3) ||
        (reinterpret_cast<uintptr_t>(seqlens) & 3) || (reinterpret_cast<uintptr_t>(idx) & 3))
        return HCA_ERR_INVALID_ARG;
    DsaTopkParams p;
    p.scores = scores;
    p.seqlens = seqlens;
    p.idx = idx;
    p.B = B; p.Lmax = Lmax; p.k = k;
    // a cluster of kTopkCluster CTAs per sequence
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kTopkCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)((long long)kTopkCluster * B), 1, 1);
    cfg.blockDim = dim3(kTopkThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, dsa_topk_kernel, p) != cudaSuccess) {
        cudaGetLastError();
        return HCA_ERR_CUDA;
    }
    return HCA_OK;
}

extern "C" hca_status_t hca_dsa_attend(const void* q, const void* k, const void* v, const int* idx, const int* seqlens,
                                       float* out, int B, int Hq, int d, int Lmax, int kmax, float scale,
                                       hca_stream_t stream) {
    using namespace hca;
    if (B < 0 || Hq < 1 || Lmax < 1 || kmax < 1) return HCA_ERR_INVALID_ARG;
    if (d != kDsaD || Hq > kDsaHeads) return HCA_ERR_UNSUPPORTED;
    if (B > (1 << 30)) return HCA_ERR_INVALID_ARG;
    if (!(scale == scale)) return HCA_ERR_INVALID_ARG;
    if (B == 0) return HCA_OK;
    if (!q || !k || !v || !idx || !seqlens || !out || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
        (reinterpret_cast<uintptr_t>(idx) & 3) || (reinterpret_cast<uintptr_t>(seqlens) & 3) ||
        (reinterpret_cast<uintptr_t>(out) & 3))
        return HCA_ERR_INVALID_ARG;
    if (!set_smem_attr_once(reinterpret_cast<const void*>(&dsa_attend_kernel), (int)kAttSmem, 11)) return HCA_ERR_CUDA;
    // the key / value maps index rows with 32-bit coordinates, one past the last row meaning
    // "zeros": launch over groups of sequences whose rows stay below 2^31
    const long long forced = g_dsa_rows_limit.load();
    const long long limit = forced > 0 ? std::min<long long>(forced, INT32_MAX) : (long long)INT32_MAX;
    const long long per = std::max<long long>(1, std::min<long long>(B, limit / Lmax - 1));
    for (long long b0 = 0; b0 < B; b0 += per) {
        const int nb = (int)std::min<long long>(per, B - b0);
        const size_t row_off = (size_t)b0 * Lmax * kDsaD;
        const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(k) + row_off;
        const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(v) + row_off;
        const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q) + (size_t)b0 * Hq * kDsaD;
        CUtensorMap tq, tk, tv;
        if (!make_tmap_4d(&tq, qb, kDsaD, Hq, nb, 1, kDsaD, (uint64_t)kDsaD * Hq, (uint64_t)kDsaD * Hq * nb, 64, 64, 1, 1) ||
            !make_tmap_rows(&tk, kb, kDsaD, (uint64_t)nb * Lmax, 64) ||
            !make_tmap_rows(&tv, vb, kDsaD, (uint64_t)nb * Lmax, 64))
            return HCA_ERR_CUDA;
        DsaAttendParams p;
        p.k = kb;
        p.v = vb;
        p.idx = idx + (size_t)b0 * kmax;
        p.seqlens = seqlens + b0;
        p.out = out + (size_t)b0 * Hq * kDsaD;
        p.B = nb; p.Hq = Hq; p.Lmax = Lmax; p.kmax = kmax;
        p.rows = (int)((long long)nb * Lmax);
        p.scale_log2 = scale * 1.4426950408889634f;
        // a cluster of two CTAs per sequence (each takes half of the kept positions)
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3((unsigned)(2 * nb), 1, 1);
        cfg.blockDim = dim3(kAttThreads, 1, 1);
        cfg.dynamicSmemBytes = kAttSmem;
        cfg.stream = reinterpret_cast<cudaStream_t>(stream);
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, dsa_attend_kernel, p, tq, tk, tv) != cudaSuccess) {
            cudaGetLastError();
            return HCA_ERR_CUDA;
        }
    }
    return HCA_OK;
}
