/*
 * hca.h -- C ABI of libhca, a B200 (sm_100a) implementation of Heavily Compressed
 * Attention (HCA).
 *
 * The operation (web pages describing ERNIE 5.5 Flash Base):
 *  - "ERNIE 5.5 Flash Base . ERNIE" (official blog), section 2.1: an HCA layer
 *    compresses every 128 tokens into a single cached entry, then attends to all of
 *    these entries plus a short window of recent, uncompressed tokens; it still sees
 *    the whole sequence while caching only a small fraction of it.
 *  - Zhidx article "280B Total Parameters, 14B Activated ...", section
 *    "1. Latent-Gated Sparse Attention": 37 of 43 layers are HCA; attention is
 *    computed only over the compressed entries and a window of recent raw tokens.
 *  - Model-card page "ERNIE 5.5 Flash Base", architecture paragraph: HCA layers use
 *    512-dim heads, 64 attention heads; every attention layer uses QK normalization
 *    and a gated output (Low-Rank Gated Attention).
 *
 * Readings where the pages are silent (the same in the kernels and in the tests):
 *  - compression of block j (raw positions blk*j .. blk*j+blk-1) is a softmax-weighted
 *    pooling: alpha = softmax(w over the block), Kc[j] = sum alpha_i K[i], Vc[j] likewise;
 *    w == NULL means all-zero weights, i.e. the mean.  Only complete blocks are written.
 *  - a query at position t attends, in one softmax, to compressed entries
 *    j < n_c(t) = max(0, floor((t - W + 1) / blk)) and to raw tokens t-W+1 .. t.
 *  - logits are scale * q.k; query head h reads KV head h / (Hq / Hkv).
 *  - QK normalization (decode): per-head RMSNorm x / sqrt(mean(x^2) + eps) * g with gains
 *    g_q, g_k of length d shared by all heads, applied to q and to every key used.
 *  - output gate (decode): out *= sigmoid(gate), element-wise, gate logits [B,Hq,dv].
 *
 * Conventions for every entry point:
 *  - all tensor pointers are DEVICE pointers owned by the caller, dense row-major in the
 *    stated layout, 16-byte aligned; bf16 means IEEE bfloat16 bit patterns;
 *  - no call allocates device memory and none copies between host and device
 *    (hca_get_device_error excepted); the library's image holds one fixed 48 MiB device
 *    array per GPU, the scratch of hca_decode_noalloc; work is queued on `stream` and the
 *    call returns without waiting for it;
 *  - a call returns HCA_OK once the work is queued; HCA_ERR_INVALID_ARG for a NULL
 *    pointer, a misaligned pointer or a size out of range; HCA_ERR_UNSUPPORTED for a
 *    shape outside the supported set (nothing is launched in either case);
 *    HCA_ERR_CUDA if a launch failed (the CUDA error is consumed);
 *  - errors found on the device (a bounded wait that ran out, a sequence length or page
 *    index out of range) are recorded in a per-device error word read by
 *    hca_get_device_error; the affected outputs are then unspecified.
 *  - nothing is printed, nothing aborts, no C++ exception crosses the boundary.
 */
#ifndef HCA_H_
#define HCA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same handle as cudaStream_t / CUstream; NULL is the legacy default stream. */
typedef struct CUstream_st* hca_stream_t;

typedef enum {
    HCA_OK = 0,
    HCA_ERR_INVALID_ARG = 1,
    HCA_ERR_UNSUPPORTED = 2,
    HCA_ERR_CUDA = 3,
    HCA_ERR_TIMEOUT = 4,       /* a bounded device wait ran out (reported by hca_get_device_error) */
    HCA_ERR_DEVICE_INPUT = 5,  /* a device-resident input was out of range (seqlens, page table) */
    HCA_ERR_INTERNAL = 6       /* a kernel found its launch environment unusable (e.g. shared-memory alignment) */
} hca_status_t;

enum {
    HCA_QK_NORM = 1,    /* decode: RMSNorm q and k with gains gq, gk */
    HCA_OUT_GATE = 2,   /* decode: multiply the output by sigmoid(gate) */
    HCA_PAGED = 4,      /* decode: compressed cache is a page pool addressed by page_table */
    HCA_WRITE_LSE = 8,  /* prefill: also write the natural-log sum-exp of the logits */
    HCA_OUT_F32 = 16,   /* prefill: output in fp32 instead of bf16 */
    HCA_WINDOW_RING = 32 /* decode: the raw window is a ring, slot p % W holds position p */
};

/*
 * hca_compress -- build the compressed cache (official blog, section 2.1: every 128
 * tokens become one cached entry).
 *   k  [B,T,Hkv,d]  bf16     raw keys
 *   v  [B,T,Hkv,dv] bf16     raw values
 *   w  [B,T]        fp32     pooling weights, one per position, shared by K, V and all
 *                            KV heads; NULL = all zero (mean pooling)
 *   kc [B,Nc,Hkv,d]  bf16    output, Nc = floor(T / blk); a trailing partial block is
 *   vc [B,Nc,Hkv,dv] bf16    not written
 * Supported: d, dv in {64, 128, 256, 512}; 1 <= blk <= 128; B, T >= 0, Hkv >= 1.
 * Arithmetic: fp32 accumulation, one rounding to bf16 (nearest even) per output.
 */
hca_status_t hca_compress(const void* k, const void* v, const float* w,
                          void* kc, void* vc,
                          int B, int T, int Hkv, int d, int dv, int blk,
                          hca_stream_t stream);

/*
 * hca_prefill -- causal HCA attention for every position of B sequences of T tokens
 * (official blog, section 2.1; Zhidx article, section 1).
 *   q  [B,T,Hq,d]    bf16
 *   k  [B,T,Hkv,d]   bf16    raw keys (the window segment)
 *   v  [B,T,Hkv,dv]  bf16
 *   kc [B,Nc,Hkv,d]  bf16    compressed cache from hca_compress, Nc = floor(T / blk)
 *   vc [B,Nc,Hkv,dv] bf16
 *   out [B,T,Hq,dv]  bf16, or fp32 with HCA_OUT_F32
 *   lse [B,Hq,T]     fp32 natural-log sum-exp of the logits, written iff HCA_WRITE_LSE
 *                    (may be NULL otherwise)
 *   scale            logit scale (typically 1/sqrt(d))
 * Supported: d == dv in {64, 512}; Hq % Hkv == 0 with Hq / Hkv a power of two <= 128;
 * 1 <= blk <= 128; W >= 1; flags among HCA_WRITE_LSE | HCA_OUT_F32.
 */
hca_status_t hca_prefill(const void* q, const void* k, const void* v,
                         const void* kc, const void* vc,
                         void* out, float* lse,
                         int B, int T, int Hq, int Hkv, int d, int dv, int blk, int W,
                         float scale, unsigned flags, hca_stream_t stream);

/*
 * hca_prefill_backward_workspace_size -- bytes of device workspace hca_prefill_backward
 * needs: per-row softmax terms, the entries' gradients, and the bf16 P / dS tiles of one
 * segment of row tiles (at most about 2 GiB; the call walks the sequence segment by
 * segment).  Returns 0 for invalid or unsupported sizes.
 */
size_t hca_prefill_backward_workspace_size(int B, int T, int Hq, int Hkv, int dv, int blk, int W);

/*
 * hca_prefill_backward -- gradients of the HCA layer for training: the gradient of
 * sum(dout * out) with respect to q, the raw k and v (through the window and through the
 * pooling of official blog section 2.1) and the pooling weights w.  The forward is
 * hca_compress followed by hca_prefill; the stored bf16 cache is taken as it is (its
 * rounding has no gradient).
 *   q, k, v, w, kc, vc  the forward's inputs and compressed cache, as for hca_compress
 *                       and hca_prefill (w may be NULL: mean pooling)
 *   out  [B,T,Hq,dv]    the forward's output, bf16 or fp32 with HCA_OUT_F32
 *   lse  [B,Hq,T] fp32  the forward's log-sum-exp (hca_prefill with HCA_WRITE_LSE)
 *   dout [B,T,Hq,dv]    bf16 incoming gradient
 *   dq   [B,T,Hq,d]     fp32 output
 *   dk   [B,T,Hkv,d]    fp32 output (window path + pooling path; rows of a trailing
 *   dv   [B,T,Hkv,dv]   fp32 output  partial block get only the window path)
 *   dw   [B,T]          fp32 output, or NULL to skip (rows of a trailing partial block: 0)
 *   workspace           device memory of at least hca_prefill_backward_workspace_size
 *                       bytes, 256-byte aligned; its contents are overwritten
 * Supported: d == dv == 512; Hq % Hkv == 0 with Hq / Hkv a power of two <= 128;
 * 1 <= blk <= 128; W >= 1; flags 0 or HCA_OUT_F32.
 * Arithmetic: bf16 operands on the tensor cores with fp32 accumulation; the softmax
 * gradient dS = P * (dP - rowsum(dout * out)) is rounded once to bf16 before the dq and
 * dk contractions, P once before the dv contraction; dk and dv are accumulated with fp32
 * atomics, so their low bits depend on the order of the additions.
 */
hca_status_t hca_prefill_backward(const void* q, const void* k, const void* v, const float* w,
                                  const void* kc, const void* vc, const void* out, const float* lse,
                                  const void* dout, float* dq, float* dk, float* dv, float* dw,
                                  void* workspace, size_t workspace_bytes,
                                  int B, int T, int Hq, int Hkv, int d, int dv_dim, int blk, int W,
                                  float scale, unsigned flags, hca_stream_t stream);

/*
 * The sparse-attention layers' decode step, in three calls (Zhidx article, section
 * "1. Latent-Gated Sparse Attention", DSA paragraph: a lightweight indexer scores the past
 * positions of each query and core attention runs over the highest-scoring Top-K only; the
 * model card: those layers use 256-dim query, key and value).  Readings where the pages are
 * silent: H_I indexer heads of d_I dims and one d_I-dim indexer key per position, the score
 * I(s) = sum_j w_j * max(0, q_I[j] . k_I[s]); the k largest scores kept, equal scores in
 * increasing position order; core attention of Hq heads over one key and one value row per
 * kept position, shared by the heads.  One decode query per sequence, at position L_b - 1,
 * sees positions 0 .. L_b - 1.
 *
 * hca_dsa_index -- indexer scores.
 *   q_idx  [B,H_I,d_I] bf16, w_idx [B,H_I] fp32, k_idx [B,Lmax,d_I] bf16
 *   seqlens [B] int32 (device; clamped into [0, Lmax])
 *   scores [B,Lmax] fp32 output, -inf at positions >= L_b
 * Supported: d_I == 64, H_I a multiple of 16 up to 64.  bf16 products, fp32 sums.
 */
hca_status_t hca_dsa_index(const void* q_idx, const float* w_idx, const void* k_idx, const int* seqlens,
                           float* scores, int B, int HI, int dI, int Lmax, hca_stream_t stream);

/*
 * hca_dsa_topk -- the k positions of largest score of each sequence among 0 .. L_b - 1.
 *   scores [B,Lmax] fp32 (as hca_dsa_index writes them), seqlens [B] int32
 *   idx    [B,k] int32 output: kept positions in increasing order, then -1 where L_b < k
 * Equal scores are taken in increasing position order, so the result is unique (-0.0 and
 * +0.0 are equal scores; scores must not be NaN).
 */
hca_status_t hca_dsa_topk(const float* scores, const int* seqlens, int* idx, int B, int Lmax, int k,
                          hca_stream_t stream);

/*
 * hca_dsa_attend -- core attention of each sequence's Hq query heads over its kept positions.
 *   q    [B,Hq,d] bf16;  k, v [B,Lmax,d] bf16 (one row per position, shared by the heads)
 *   idx  [B,kmax] int32 from hca_dsa_topk (-1 entries and entries past min(kmax, L_b) unused;
 *        an entry >= Lmax is reported as HCA_ERR_DEVICE_INPUT and not read)
 *   seqlens [B] int32;  out [B,Hq,d] fp32;  scale: logit scale (typically 1/sqrt(d))
 * Supported: d == 256, Hq <= 64.  bf16 operands, fp32 accumulation, P rounded to bf16.
 * A sequence with L_b = 0 keeps no position: its output is NaN (a softmax over nothing).
 * Sequences are launched in groups whose B_group * Lmax stays below 2^31 (one launch at the
 * usual sizes).
 */
hca_status_t hca_dsa_attend(const void* q, const void* k, const void* v, const int* idx, const int* seqlens,
                            float* out, int B, int Hq, int d, int Lmax, int kmax, float scale,
                            hca_stream_t stream);

/*
 * hca_decode_workspace_size -- bytes of device workspace hca_decode needs for a batch
 * of B sequences on the CURRENT device (split-KV partial results).  Returns 0 for
 * invalid sizes.
 */
size_t hca_decode_workspace_size(int B, int Hq, int Hkv, int dv);

/*
 * hca_decode -- one new query per sequence over its compressed cache and raw window
 * (official blog, section 2.1), split over keys across the whole GPU and merged in a
 * second pass.
 *   q        [B,Hq,d] bf16        the query at position t = seqlens[b] - 1
 *   kc, vc   contiguous: [B,Nmax,Hkv,d|dv] bf16, entry j of sequence b at row (b, j);
 *            with HCA_PAGED: page pools [P,page_size,Hkv,d|dv], entry j of sequence b at
 *            pool[page_table[b*max_pages + j/page_size], j % page_size]
 *   page_table [B,max_pages] int32 (HCA_PAGED only, else NULL); num_pages = P, the
 *            number of pages in the pools (entries outside [0, P) are reported as
 *            HCA_ERR_DEVICE_INPUT and clamped into the pool; the output is then unspecified)
 *   kw, vw   [B,W,Hkv,d|dv] bf16  raw window: slot i holds position seqlens[b] - W + i;
 *            slots with a negative position are ignored.  With HCA_WINDOW_RING (the
 *            layout hca_append maintains) slot p % W holds position p instead; attention
 *            over the window does not depend on the order of its keys, so only which
 *            slots are valid changes (slots 0 .. L_b - 1 while L_b < W)
 *   seqlens  [B] int32            context length L_b >= 1 including the new token; the
 *            visible entry count n_c(L_b - 1) must not exceed Nmax (or the pages)
 *   gq, gk   [d] fp32 gains, eps  (HCA_QK_NORM only, else NULL)
 *   gate     [B,Hq,dv] bf16 logits (HCA_OUT_GATE only, else NULL)
 *   out      [B,Hq,dv] fp32
 *   workspace, ws_bytes           device scratch of at least
 *            hca_decode_workspace_size(B, Hq, Hkv, dv) bytes, owned by the caller; its
 *            contents need no initialisation and are overwritten
 * Supported: d == dv == 512; Hq % Hkv == 0 with Hq / Hkv <= 64; 1 <= blk <= 128; W >= 1;
 * page_size a multiple of 64 with HCA_PAGED.
 */
hca_status_t hca_decode(const void* q, const void* kc, const void* vc,
                        const int* page_table, int page_size, int max_pages, int num_pages,
                        const void* kw, const void* vw, const int* seqlens,
                        const float* gq, const float* gk, float eps,
                        const void* gate, float* out,
                        void* workspace, size_t ws_bytes,
                        int B, int Hq, int Hkv, int d, int dv, int blk, int W, int Nmax,
                        float scale, unsigned flags, hca_stream_t stream);

/*
 * hca_decode_vha -- hca_decode with Virtual Head Attention fused into its combine pass
 * (official blog, section 2.1, and the Zhidx article, section "1. Latent-Gated Sparse
 * Attention": a lightweight cross-head low-rank mixing with an identity skip, applied after the
 * attention).  The output is that of hca_decode (with the gate, when HCA_OUT_GATE is set) mixed
 * per sequence and channel over the Hq heads: out[b, :, c] <- (I + U V^T) out[b, :, c].
 *   vha_u, vha_v  [Hq, vha_rank] fp32 mixing factors (4-byte aligned), 1 <= vha_rank <= 32
 * The merge kernel already holds every head of a sequence on chip, so the mixing costs no extra
 * pass over the output (hca_vha on an hca_decode output gives the same result).  Other
 * arguments, layouts and errors: as hca_decode; Hkv must be 1 (one KV group holds all heads),
 * else HCA_ERR_UNSUPPORTED.
 */
hca_status_t hca_decode_vha(const void* q, const void* kc, const void* vc,
                            const int* page_table, int page_size, int max_pages, int num_pages,
                            const void* kw, const void* vw, const int* seqlens,
                            const float* gq, const float* gk, float eps,
                            const void* gate, const float* vha_u, const float* vha_v, int vha_rank,
                            float* out, void* workspace, size_t ws_bytes,
                            int B, int Hq, int Hkv, int d, int dv, int blk, int W, int Nmax,
                            float scale, unsigned flags, hca_stream_t stream);

/*
 * hca_decode_noalloc -- hca_decode without a workspace argument.  There is no counterpart
 * in the paper: this entry point exists for callers that cannot allocate device memory
 * when they decode -- an inference-engine plugin that must not allocate inside its
 * enqueue call, a latency-critical server that forbids allocation after warm-up, or host
 * code that only ever receives pre-allocated buffers -- and so cannot provide the
 * workspace hca_decode needs.
 *
 * Arguments, layouts, supported shapes and results are those of hca_decode.  The split
 * records live in a fixed array of HCA_DECODE_NOALLOC_MAX_BYTES inside the library's
 * device image, which every GPU that loads the library holds until the process exits.
 * The call allocates nothing (no cudaMalloc, no cudaFree, no allocating library routine).
 *  - Returns HCA_ERR_INVALID_ARG, before any launch, when the batch needs more scratch
 *    than the array holds, i.e. when hca_decode_workspace_size(B, Hq, Hkv, dv) exceeds
 *    HCA_DECODE_NOALLOC_MAX_BYTES (on a 148-SM B200 this allows up to 234
 *    (sequence, KV head) units).
 *  - The first call on a device looks up the array's device address on that device
 *    (once per device, with that device current); make that first call before any stream
 *    capture.  The address is cached per device ordinal for the primary context: after
 *    cudaDeviceReset, or when calling from a context other than the device's primary one,
 *    the cached address is no longer valid -- use hca_decode there.
 *  - Every call on a device shares the same array, and the array keeps the previous
 *    call's contents; nothing in it needs to start at zero.  Calls whose work overlaps
 *    on the GPU (for example on two streams at once) race on it: serialise them.
 */
#define HCA_DECODE_NOALLOC_MAX_BYTES (48u << 20)

hca_status_t hca_decode_noalloc(const void* q, const void* kc, const void* vc,
                                const int* page_table, int page_size, int max_pages, int num_pages,
                                const void* kw, const void* vw, const int* seqlens,
                                const float* gq, const float* gk, float eps,
                                const void* gate, float* out,
                                int B, int Hq, int Hkv, int d, int dv, int blk, int W, int Nmax,
                                float scale, unsigned flags, hca_stream_t stream);

/*
 * hca_vha -- Virtual Head Attention on an attention output, in place (official blog, section
 * 2.1, and the Zhidx article, section "1. Latent-Gated Sparse Attention": a lightweight
 * cross-head low-rank mixing with an identity skip after the attention).  Per token and per
 * channel c: out[:, c] <- (I + U V^T) out[:, c] over the token's Hq heads.
 *   out    [n,Hq,dv] bf16, or fp32 with HCA_OUT_F32, 16-byte aligned (a prefill output is
 *          n = B*T tokens, a decode output n = B); applied after the decode gate, to the final
 *          output
 *   U, V   [Hq,r] fp32 mixing factors (4-byte aligned)
 * Supported: Hq <= 64, 1 <= r <= 32, dv a multiple of 64; flags 0 or HCA_OUT_F32.  The
 * kernel reads and writes the output once; it computes in fp32 (the rank padded with zero
 * factors to 4, 8, 16 or 32) and rounds once to the output type.  Errors (nothing launched):
 * HCA_ERR_INVALID_ARG for null or misaligned pointers and negative sizes,
 * HCA_ERR_UNSUPPORTED outside the supported shapes or for other flags.
 */
hca_status_t hca_vha(void* out, const float* U, const float* V, long long n, int Hq, int dv, int r,
                     unsigned flags, hca_stream_t stream);

/*
 * hca_append_state_size -- bytes of pooling state hca_append keeps per batch:
 * B * Hkv * (4 + d + dv) floats.  Returns 0 for invalid sizes.
 */
size_t hca_append_state_size(int B, int Hkv, int d, int dv);

/*
 * hca_append -- one decode step's cache update: the newest token of every sequence enters
 * the raw window, and a block of blk tokens that it completes becomes one compressed entry
 * (official blog, section 2.1: every 128 tokens are compressed into a single cached entry).
 * The entry is the compressor's softmax-weighted mean of the block (hca_compress), computed
 * online: no raw token has to stay resident after it leaves the window.
 *   k_new, v_new [B,Hkv,d|dv] bf16  the newest token of each sequence, at position
 *                seqlens[b] - 1
 *   w_new    [B] fp32 pooling weight of that token (NULL = 0, i.e. the mean)
 *   seqlens  [B] int32 length L_b >= 1 INCLUDING the new token
 *   kw, vw   [B,W,Hkv,d|dv] bf16 window rings, written at slot (L_b - 1) % W; read them
 *            with hca_decode(..., HCA_WINDOW_RING)
 *   kc, vc   the compressed cache, laid out as for hca_decode (contiguous [B,Nmax,...], or
 *            page pools with HCA_PAGED); entry (L_b / blk) - 1 is written when
 *            L_b % blk == 0.  An entry outside the cache (or its pages) is reported as
 *            HCA_ERR_DEVICE_INPUT and not written
 *   state    hca_append_state_size(B, Hkv, d, dv) bytes of fp32 owned by the caller: the
 *            running pool of each (sequence, KV head)'s current block.  All zero means an
 *            empty block; set a sequence's state to zero before its first token (a call
 *            that completes a block leaves it zero).  Tokens must be appended in order,
 *            one call per position
 * Supported: d, dv in {64, 128, 256, 512}; 1 <= blk <= 128; W >= 1; flags 0 or HCA_PAGED
 * (page_size a multiple of 64).  One CTA per (sequence, KV head); the call only queues it.
 */
hca_status_t hca_append(const void* k_new, const void* v_new, const float* w_new, const int* seqlens,
                        void* kw, void* vw, void* kc, void* vc,
                        const int* page_table, int page_size, int max_pages, int num_pages,
                        void* state, int B, int Hkv, int d, int dv, int blk, int W, int Nmax,
                        unsigned flags, hca_stream_t stream);

/*
 * hca_gate_logits -- the gate projection of Low-Rank Gated Attention (Zhidx article, section
 * "1. Latent-Gated Sparse Attention": the output gate is computed from the attention layer's
 * query latent, a quarter of the hidden size, so the projection has 75% fewer weights than one
 * from the hidden state):  gate[i, h, c] = sum_k cq[i, k] * wg[k, h, c].
 *   cq    [n, rq] bf16       query latents of n tokens (decode: one per sequence)
 *   wg    [rq, Hq, dv] bf16  gate projection weights
 *   gate  [n, Hq, dv] bf16   output logits (fp32 accumulation, one rounding); pass them to
 *                            hca_decode / hca_decode_vha with HCA_OUT_GATE
 * Supported: rq a multiple of 64, Hq * dv a multiple of 256.  Tensor-core GEMM, bound by reading
 * wg once (64 MB at rq = 1024, Hq = 64, dv = 512).  Errors as for the other entry points.
 */
hca_status_t hca_gate_logits(const void* cq, const void* wg, void* gate, int n, int rq, int Hq, int dv,
                             hca_stream_t stream);

/* Static, NUL-terminated description of a status code. */
const char* hca_status_string(hca_status_t status);

/*
 * hca_get_device_error -- read and clear the current device's error word in one atomic
 * step on `stream` (a one-thread kernel), then wait for `stream`: HCA_OK if no kernel
 * recorded an error since the last call, HCA_ERR_TIMEOUT, HCA_ERR_DEVICE_INPUT or
 * HCA_ERR_INTERNAL otherwise, HCA_ERR_CUDA if the read failed.  An error recorded by work on
 * another stream is never lost: it is either returned or left for the next call.  The word
 * is per device and the read-out slot is shared, so make one such call at a time per device.
 * While the word holds HCA_ERR_TIMEOUT, hca_decode writes NaN to its outputs instead of
 * merging split records that a timed-out kernel may have left incomplete.
 */
hca_status_t hca_get_device_error(hca_stream_t stream);

/*
 * hca_debug_set_backward_segment -- test hook: hca_prefill_backward (and its workspace size)
 * processes at most `rows` row tiles per segment, so that short sequences exercise the
 * segment walk that long ones take; 0 restores the default (segments sized by a 2 GiB bound
 * on the P / dS records).  Process-wide; call it only while no backward is being enqueued.
 * HCA_ERR_INVALID_ARG for rows < 0.
 */
hca_status_t hca_debug_set_backward_segment(int rows);

/*
 * hca_debug_set_dsa_rows_limit -- test hook: hca_dsa_attend launches over groups of
 * sequences whose B_group * Lmax stays below `rows` instead of below 2^31, so that small
 * batches exercise the grouped launches that very large ones take; 0 restores the default.
 * Process-wide; call it only while no attention call is being enqueued.
 * HCA_ERR_INVALID_ARG for rows < 0.
 */
hca_status_t hca_debug_set_dsa_rows_limit(long long rows);

/*
 * Test hooks for the bounded waits (not part of the computation; the paper has no
 * counterpart).  Every wait inside the kernels gives up after a wall-clock limit, records
 * HCA_ERR_TIMEOUT and lets the kernel unwind (free its tensor memory, return) instead of
 * hanging the GPU.  These three calls let a test make that happen on purpose without any
 * bad address, trap or endless loop.  Each synchronises `stream`.
 *
 * hca_debug_set_wait_limit -- set the current device's wait limit in nanoseconds
 *   (0 restores the default of 1 s).  Affects every later launch on the device.
 * hca_debug_set_drop_slab -- on != 0: every later hca_decode launch on the device never
 *   requests the first key slab of each split CTA, so the wait for it runs out after the
 *   wait limit and the whole decode reports HCA_ERR_TIMEOUT (outputs NaN); 0 turns it off.
 * hca_debug_wait_probe -- queue one CTA that waits on a barrier that can never complete
 *   and so records HCA_ERR_TIMEOUT after the wait limit; nothing else is in flight.
 */
hca_status_t hca_debug_set_wait_limit(unsigned long long limit_ns, hca_stream_t stream);
hca_status_t hca_debug_set_drop_slab(int on, hca_stream_t stream);
hca_status_t hca_debug_wait_probe(hca_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HCA_H_ */
