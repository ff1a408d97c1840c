/*
 * hca_oracle.c -- plain, slow, fp64 CPU oracle for Heavily Compressed Attention (HCA).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file: only the test-suite, the smoke check and the benchmark's CPU-baseline
 * leg use it.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (sources are the web pages describing ERNIE 5.5 Flash Base):
 *
 *  - "ERNIE 5.5 Flash Base . ERNIE" (official blog), section 2.1, the HCA paragraph:
 *    every 128 tokens are compressed into one cached entry; each query attends to
 *    all of these entries plus a short window of recent uncompressed tokens, so the
 *    layer still sees the whole sequence while caching a small fraction of it.
 *  - Zhidx article "280B Total Parameters, 14B Activated ...", section
 *    "1. Latent-Gated Sparse Attention": attention runs only over the compressed
 *    entries and a window of a small number of recent uncompressed tokens.
 *  - Model-card page "ERNIE 5.5 Flash Base" (nlp.com.ai), architecture paragraph:
 *    HCA layers cache one entry per 128 tokens, use 512-dim heads, and every
 *    attention layer uses QK normalization and an output gate.
 *
 * The pages do not define the compressor, the window length, the boundary between
 * the two segments, the norm epsilon or the gate shape.  The readings used here:
 *  - compressor: per-position softmax-weighted pooling of the blk raw rows of a
 *    block, one fp32 weight per position shared by K and V and by all KV heads;
 *    all-zero weights give the plain mean;
 *  - only complete blocks are compressed: Nc = floor(T / blk);
 *  - a query at position t sees compressed entries j < n_c(t) with
 *    n_c(t) = max(0, floor((t - W + 1) / blk)) and raw tokens u in [t-W+1, t];
 *    tokens between the last visible block and the window are seen by neither;
 *  - one softmax over the union of both segments, logits scale * q.k;
 *  - QK normalization (decode only): per head RMSNorm over d,
 *    x / sqrt(mean(x^2) + eps) * g, applied to q and to every key at use time;
 *  - output gate (decode only): out *= 1 / (1 + exp(-gate)), element-wise.
 *
 * Every value is computed in fp64 from the exact values of the bf16/fp32 inputs.
 * The compressed cache is a stored bf16 tensor, so attention runs over the cache
 * rounded to bf16 (round to nearest even); oracle_round_bf16 does that rounding.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* exact widening of a bf16 bit pattern */
static double bf(uint16_t x) {
    uint32_t u = ((uint32_t)x) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Round a double to the nearest bf16 value, ties to even, in one step
 * (no intermediate float rounding). */
static uint16_t to_bf16(double x) {
    if (isnan(x)) return 0x7fc0;
    double ax = fabs(x);
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    if (ax == 0.0) return sign;
    int e;
    frexp(ax, &e);                  /* ax = m * 2^e, m in [0.5, 1) */
    int q = e - 8;                  /* 8 significant bits: quantum 2^(e-8) */
    if (q < -133) q = -133;         /* subnormal quantum of bf16 */
    double r = nearbyint(ldexp(ax, -q));   /* default rounding: nearest, ties even */
    double y = ldexp(r, q);
    if (y > 3.3895313892515355e38) return sign | 0x7f80;   /* overflow -> inf */
    float f = (float)y;             /* exact: y has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return sign | (uint16_t)(u >> 16);
}

void oracle_round_bf16(const double* x, uint16_t* y, int64_t n) {
    for (int64_t i = 0; i < n; ++i) y[i] = to_bf16(x[i]);
}

/* n_c(t): compressed entries visible to a query at position t. */
int64_t oracle_visible_entries(int64_t t, int64_t W, int64_t blk) {
    int64_t a = t - W + 1;
    if (a <= 0) return 0;
    return a / blk;
}

/*
 * Block compression.  k,v: [B,T,Hkv,d] / [B,T,Hkv,dv] bf16; w: [B,T] fp32 or NULL
 * (NULL means all-zero weights).  kc,vc: [B,T/blk,Hkv,d] / [.., dv] fp64.
 * Entry j of sequence b pools raw positions blk*j .. blk*j+blk-1 with
 * alpha = softmax over the block of w (max subtracted first).
 */
int oracle_compress(const uint16_t* k, const uint16_t* v, const float* w,
                    int64_t B, int64_t T, int64_t Hkv, int64_t d, int64_t dv, int64_t blk,
                    double* kc, double* vc) {
    if (B < 0 || T < 0 || Hkv <= 0 || d <= 0 || dv <= 0 || blk <= 0) return 1;
    int64_t Nc = T / blk;
    #pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t j = 0; j < Nc; ++j) {
            double* alpha = (double*)malloc(sizeof(double) * (size_t)blk);
            double m = -INFINITY;
            for (int64_t i = 0; i < blk; ++i) {
                double wi = w ? (double)w[b * T + blk * j + i] : 0.0;
                alpha[i] = wi;
                if (wi > m) m = wi;
            }
            double s = 0.0;
            for (int64_t i = 0; i < blk; ++i) { alpha[i] = exp(alpha[i] - m); s += alpha[i]; }
            for (int64_t i = 0; i < blk; ++i) alpha[i] /= s;
            for (int64_t g = 0; g < Hkv; ++g) {
                double* ko = kc + ((b * Nc + j) * Hkv + g) * d;
                double* vo = vc + ((b * Nc + j) * Hkv + g) * dv;
                for (int64_t c = 0; c < d; ++c) ko[c] = 0.0;
                for (int64_t c = 0; c < dv; ++c) vo[c] = 0.0;
                for (int64_t i = 0; i < blk; ++i) {
                    int64_t pos = blk * j + i;
                    const uint16_t* kr = k + ((b * T + pos) * Hkv + g) * d;
                    const uint16_t* vr = v + ((b * T + pos) * Hkv + g) * dv;
                    for (int64_t c = 0; c < d; ++c) ko[c] += alpha[i] * bf(kr[c]);
                    for (int64_t c = 0; c < dv; ++c) vo[c] += alpha[i] * bf(vr[c]);
                }
            }
            free(alpha);
        }
    }
    return 0;
}

/*
 * One softmax over a list of keys for one query head.
 *   z_i = scale * <qv, key_i>   (qv and the keys already normalised if asked)
 *   out = sum_i p_i val_i / sum_i p_i,  lse = max z + log(sum exp(z - max z))
 * keys/vals are given as fp64 rows gathered by the caller.
 */
static void attend(const double* qv, const double* keys, const double* vals, int64_t n,
                   int64_t d, int64_t dv, double scale, double* out, double* lse,
                   double* z /* scratch [n] */) {
    double m = -INFINITY;
    for (int64_t i = 0; i < n; ++i) {
        double s = 0.0;
        for (int64_t c = 0; c < d; ++c) s += qv[c] * keys[i * d + c];
        z[i] = scale * s;
        if (z[i] > m) m = z[i];
    }
    double l = 0.0;
    for (int64_t c = 0; c < dv; ++c) out[c] = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        double p = exp(z[i] - m);
        l += p;
        for (int64_t c = 0; c < dv; ++c) out[c] += p * vals[i * dv + c];
    }
    for (int64_t c = 0; c < dv; ++c) out[c] /= l;
    if (lse) *lse = m + log(l);
}

/*
 * Prefill rows.  q [B,T,Hq,d] (or, with q_rows != 0, [n_rows,Hq,d]: one query row per
 * requested (b, t)), k [B,T,Hkv,d], v [B,T,Hkv,dv] bf16;
 * kc [B,Nc,Hkv,d], vc [B,Nc,Hkv,dv] bf16 (the stored cache), Nc = T / blk.
 * rows: n_rows pairs (b, t).  out: [n_rows, Hq, dv] fp64; lse: [n_rows, Hq] or NULL.
 * Query head h reads KV head h / (Hq / Hkv).
 */
int oracle_prefill_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        const uint16_t* kc, const uint16_t* vc,
                        int64_t B, int64_t T, int64_t Hq, int64_t Hkv, int64_t d, int64_t dv,
                        int64_t blk, int64_t W, double scale,
                        const int64_t* rows, int64_t n_rows, int q_rows, double* out, double* lse) {
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv || blk <= 0 || W <= 0) return 1;
    for (int64_t r = 0; r < n_rows; ++r)     /* every requested row inside the batch */
        if (rows[2 * r] < 0 || rows[2 * r] >= B || rows[2 * r + 1] < 0 || rows[2 * r + 1] >= T) return 1;
    int64_t Nc = T / blk, grp = Hq / Hkv;
    #pragma omp parallel
    {
        double* keys = (double*)malloc(sizeof(double) * (size_t)((Nc + W) * d + 1));
        double* vals = (double*)malloc(sizeof(double) * (size_t)((Nc + W) * dv + 1));
        double* z = (double*)malloc(sizeof(double) * (size_t)(Nc + W + 1));
        double* qv = (double*)malloc(sizeof(double) * (size_t)d);
        #pragma omp for collapse(2) schedule(dynamic, 1)
        for (int64_t r = 0; r < n_rows; ++r) {
            for (int64_t g = 0; g < Hkv; ++g) {
                int64_t b = rows[2 * r], t = rows[2 * r + 1];
                int64_t nc = oracle_visible_entries(t, W, blk);
                int64_t lo = t - W + 1 < 0 ? 0 : t - W + 1;
                int64_t n = 0;
                for (int64_t j = 0; j < nc; ++j, ++n) {
                    for (int64_t c = 0; c < d; ++c) keys[n * d + c] = bf(kc[((b * Nc + j) * Hkv + g) * d + c]);
                    for (int64_t c = 0; c < dv; ++c) vals[n * dv + c] = bf(vc[((b * Nc + j) * Hkv + g) * dv + c]);
                }
                for (int64_t u = lo; u <= t; ++u, ++n) {
                    for (int64_t c = 0; c < d; ++c) keys[n * d + c] = bf(k[((b * T + u) * Hkv + g) * d + c]);
                    for (int64_t c = 0; c < dv; ++c) vals[n * dv + c] = bf(v[((b * T + u) * Hkv + g) * dv + c]);
                }
                for (int64_t h = g * grp; h < (g + 1) * grp; ++h) {
                    const uint16_t* qr = q_rows ? q + (r * Hq + h) * d : q + ((b * T + t) * Hq + h) * d;
                    for (int64_t c = 0; c < d; ++c) qv[c] = bf(qr[c]);
                    attend(qv, keys, vals, n, d, dv, scale, out + (r * Hq + h) * dv,
                           lse ? lse + r * Hq + h : NULL, z);
                }
            }
        }
        free(keys); free(vals); free(z); free(qv);
    }
    return 0;
}

/* RMSNorm of one head vector: x / sqrt(mean(x^2) + eps) * g */
static void rmsnorm(double* x, int64_t d, const float* g, double eps) {
    double ss = 0.0;
    for (int64_t c = 0; c < d; ++c) ss += x[c] * x[c];
    double inv = 1.0 / sqrt(ss / (double)d + eps);
    for (int64_t c = 0; c < d; ++c) x[c] = x[c] * inv * (double)g[c];
}

/*
 * Decode: one new query per sequence at position t = L_b - 1.
 *  q     [B,Hq,d] bf16
 *  cache contiguous kc/vc [B,Nmax,Hkv,d|dv] when page_table == NULL, else a pool
 *        [P,page_size,Hkv,d|dv] with entry j of sequence b at
 *        pool[page_table[b*max_pages + j/page_size], j % page_size]
 *  kw,vw [B,W,Hkv,d|dv] bf16: slot i holds raw position L_b - W + i (slots with a
 *        negative position are not part of the sequence)
 *  gq,gk [d] fp32 gains (both NULL: no QK normalization), eps
 *  gate  [B,Hq,dv] bf16 logits or NULL
 *  out   [B,Hq,dv] fp64; lse [B,Hq] or NULL
 */
int oracle_decode(const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                  const int32_t* page_table, int64_t page_size, int64_t max_pages,
                  const uint16_t* kw, const uint16_t* vw, const int32_t* seqlens,
                  const float* gq, const float* gk, double eps, const uint16_t* gate,
                  int64_t B, int64_t Hq, int64_t Hkv, int64_t d, int64_t dv,
                  int64_t blk, int64_t W, int64_t Nmax, double scale,
                  double* out, double* lse) {
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv || blk <= 0 || W <= 0) return 1;
    if ((gq == NULL) != (gk == NULL)) return 1;
    int64_t grp = Hq / Hkv;
    int64_t cap = page_table ? max_pages * page_size : Nmax;
    for (int64_t b = 0; b < B; ++b) {
        int64_t L = seqlens[b];
        if (L < 1) return 2;
        if (oracle_visible_entries(L - 1, W, blk) > cap) return 2;
    }
    int bad = 0;
    #pragma omp parallel
    {
        double* keys = (double*)malloc(sizeof(double) * (size_t)((cap + W) * d + 1));
        double* vals = (double*)malloc(sizeof(double) * (size_t)((cap + W) * dv + 1));
        double* z = (double*)malloc(sizeof(double) * (size_t)(cap + W + 1));
        double* qv = (double*)malloc(sizeof(double) * (size_t)d);
        #pragma omp for collapse(2) schedule(dynamic, 1)
        for (int64_t b = 0; b < B; ++b) {
            for (int64_t g = 0; g < Hkv; ++g) {
                int64_t L = seqlens[b], t = L - 1;
                int64_t nc = oracle_visible_entries(t, W, blk);
                int64_t n = 0;
                for (int64_t j = 0; j < nc; ++j, ++n) {
                    int64_t row;
                    if (page_table) {
                        int64_t pg = page_table[b * max_pages + j / page_size];
                        row = pg * page_size + j % page_size;
                    } else {
                        row = b * Nmax + j;
                    }
                    for (int64_t c = 0; c < d; ++c) keys[n * d + c] = bf(kc[(row * Hkv + g) * d + c]);
                    for (int64_t c = 0; c < dv; ++c) vals[n * dv + c] = bf(vc[(row * Hkv + g) * dv + c]);
                }
                for (int64_t i = 0; i < W; ++i) {
                    if (L - W + i < 0) continue;
                    for (int64_t c = 0; c < d; ++c) keys[n * d + c] = bf(kw[((b * W + i) * Hkv + g) * d + c]);
                    for (int64_t c = 0; c < dv; ++c) vals[n * dv + c] = bf(vw[((b * W + i) * Hkv + g) * dv + c]);
                    ++n;
                }
                if (gk)
                    for (int64_t i = 0; i < n; ++i) rmsnorm(keys + i * d, d, gk, eps);
                for (int64_t h = g * grp; h < (g + 1) * grp; ++h) {
                    for (int64_t c = 0; c < d; ++c) qv[c] = bf(q[(b * Hq + h) * d + c]);
                    if (gq) rmsnorm(qv, d, gq, eps);
                    double* o = out + (b * Hq + h) * dv;
                    attend(qv, keys, vals, n, d, dv, scale, o, lse ? lse + b * Hq + h : NULL, z);
                    if (gate)
                        for (int64_t c = 0; c < dv; ++c)
                            o[c] *= 1.0 / (1.0 + exp(-bf(gate[(b * Hq + h) * dv + c])));
                }
            }
        }
        free(keys); free(vals); free(z); free(qv);
    }
    return bad;
}
