/*
 * dsa_oracle.c -- plain, slow, fp64 CPU oracle for the indexed sparse
 * attention (DSA) hot path: Lightning Indexer scores -> per-row Top-K ->
 * sparse MLA attention over the selected latent KV rows, plus the FP8
 * index-key cache codec.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path links, loads or calls
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do. It shares no code, header, table or helper with the CUDA path.
 *
 * What it follows (sources are the five pages on Day-0 DSA inference; cited by
 * page title and section):
 *  - "Day-0 Inference Optimization for a New Sparse Attention Architecture",
 *    section 1 (Core Mechanisms): the Lightning Indexer scores the query
 *    against every historical position and keeps the Top-K; Sparse Flash
 *    Attention then attends only over the KV-cache rows those indices name,
 *    on top of multi-head latent attention (MLA).
 *  - "Optimizing Inference for New Model Architectures ...", section 3
 *    (Fusing Index and Attention): the indexer's three steps are relevance
 *    scoring, head-weight weighting and Top-K selection.
 *  - The score law, with its ReLU, is I[t,s] = sum_j w[t,j] * max(0,
 *    q_I[t,j,:] . k_I[s,:]) (the pages name the steps; this is the plain
 *    reading of "head-weighted summation" over per-head relevance scores).
 *  - "Day-0 Inference Adaptation and Performance Optimization for
 *    New-Architecture Large Language Models", Tiered Quantization (table and
 *    its pseudocode): per-group dynamic scale = max|group| / quant_max, then
 *    the 8-bit cast. quant_max = 448, the largest finite OCP E4M3 value.
 *
 * Every floating-point step runs in fp64 except the FP8 codec, whose scale
 * and quotient are fp32 by definition of the cache format (they decide an
 * integer code, so the oracle takes that decision in the kernel's precision).
 * No blocking, fusion or reordering beyond the definitions below.
 *
 * Parity pins for every function live in tests/test_oracle_*.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* OCP 8-bit floating point, E4M3 ("FN" variant: no infinities).             */
/* Layout: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.            */
/* Exponent field 0 encodes subnormals m/8 * 2^-6; field 1..15 encodes       */
/* (1 + m/8) * 2^(e-7), except S.1111.111 which is NaN. Max finite 448.      */
/* ------------------------------------------------------------------------ */

double oracle_e4m3_decode(uint8_t code)
{
    int sign = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Round-to-nearest-even onto the E4M3 grid, saturating finite values to
 * +-448 ("satfinite"). Inputs are finite. */
uint8_t oracle_e4m3_encode_satfinite(float xf)
{
    double x = (double)xf;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    if (a >= 448.0)
        return sign | 0x7E;
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: grid step 2^-9; n = 8 lands on the smallest normal,
         * whose code (0x08) follows the subnormal codes directly. */
        double n = nearbyint(a / ldexp(1.0, -9));   /* ties to even */
        return sign | (uint8_t)n;
    }
    int e = ilogb(a);                               /* floor(log2 a), -6..8 */
    double step = ldexp(1.0, e - 3);
    double n = nearbyint(a / step);                 /* 8..16, ties to even */
    if (n >= 16.0) {
        e += 1;
        n = 8.0;
    }
    return sign | (uint8_t)(((e + 7) << 3) | ((int)n - 8));
}

/* Index-key cache write (per-group dynamic FP8 quantisation).
 * k: [n, dim] values (bf16-exact fp32); per group of `group` elements:
 *   s = fl32(absmax / 448); s == 0 -> all codes 0;
 *   else code = e4m3_rn_satfinite(fl32(k / s)).
 * codes: [n, dim] uint8, scales: [n, dim/group] fp32. */
void oracle_quantize_keys(const float *k, int64_t n, int32_t dim, int32_t group,
                          uint8_t *codes, float *scales)
{
    int32_t ng = dim / group;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
        for (int32_t g = 0; g < ng; ++g) {
            const float *src = k + r * dim + (int64_t)g * group;
            uint8_t *dst = codes + r * dim + (int64_t)g * group;
            float amax = 0.0f;
            for (int32_t i = 0; i < group; ++i) {
                float v = fabsf(src[i]);
                if (v > amax)
                    amax = v;
            }
            volatile float s = amax / 448.0f;        /* fp32 division */
            scales[r * ng + g] = s;
            for (int32_t i = 0; i < group; ++i) {
                if (s == 0.0f) {
                    dst[i] = 0;
                } else {
                    volatile float qv = src[i] / s;  /* fp32 division */
                    dst[i] = oracle_e4m3_encode_satfinite(qv);
                }
            }
        }
    }
}

/* Dequantised value as fp32: fl32(decode(code) * s). The product is exact in
 * fp64 (4 x 24 significant bits), so this is a single correct rounding. */
void oracle_dequantize_keys(const uint8_t *codes, const float *scales, int64_t n, int32_t dim,
                            int32_t group, float *out)
{
    int32_t ng = dim / group;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r)
        for (int32_t d = 0; d < dim; ++d)
            out[r * dim + d] = (float)(oracle_e4m3_decode(codes[r * dim + d]) *
                                       (double)scales[r * ng + d / group]);
}

/* ------------------------------------------------------------------------ */
/* Lightning Indexer scores.                                                */
/* ------------------------------------------------------------------------ */

static int32_t seq_of_token(const int32_t *cu_q, int32_t B, int32_t t)
{
    int32_t b = 0;
    while (b + 1 < B && cu_q[b + 1] <= t)
        ++b;
    return b;
}

/* Key element (b, s, d) in fp64: either a bf16 value held in fp32, or the
 * dequantised FP8 value decode(code) * scale (exact in fp64). */
static inline double key_at(int32_t key_is_fp8, const float *kf, const uint8_t *k8,
                            const float *ks, int32_t group, int64_t row, int32_t dI, int32_t d)
{
    if (!key_is_fp8)
        return (double)kf[row * dI + d];
    return oracle_e4m3_decode(k8[row * dI + d]) * (double)ks[row * (dI / group) + d / group];
}

/* scores[r, s] for query token t = rows[r]:
 *   n_valid = min(q_pos[t] + 1, seq_lens[b])      (causal: s <= pos, s < len)
 *   s <  n_valid: sum_j w[t,j] * max(0, sum_d q_I[t,j,d] * k[b,s,d])
 *   s >= n_valid: -inf
 * q_I [T,HI,dI], w [T,HI], keys [B,Lmax,dI]; scores [n_rows, ld], ld >= Lmax. */
void oracle_indexer_scores(int32_t B, int32_t Lmax, const int32_t *cu_q, const int32_t *q_pos,
                           const int32_t *seq_lens, int32_t HI, int32_t dI, const float *q_idx,
                           const float *w, int32_t key_is_fp8, const float *k_f32,
                           const uint8_t *k_fp8, const float *k_scale, int32_t group,
                           int32_t n_rows, const int32_t *rows, double *scores, int64_t ld)
{
    /* every (row, position) is independent: spread them over the threads */
#pragma omp parallel for collapse(2) schedule(dynamic, 256)
    for (int32_t r = 0; r < n_rows; ++r) {
        for (int32_t s = 0; s < Lmax; ++s) {
            int32_t t = rows[r];
            int32_t b = seq_of_token(cu_q, B, t);
            int32_t nv = q_pos[t] + 1;
            if (nv > seq_lens[b])
                nv = seq_lens[b];
            double *out = scores + (int64_t)r * ld;
            if (s >= nv) {
                out[s] = -INFINITY;
                continue;
            }
            int64_t row = (int64_t)b * Lmax + s;
            double I = 0.0;
            for (int32_t j = 0; j < HI; ++j) {
                const float *qj = q_idx + ((int64_t)t * HI + j) * dI;
                double dot = 0.0;
                for (int32_t d = 0; d < dI; ++d)
                    dot += (double)qj[d] * key_at(key_is_fp8, k_f32, k_fp8, k_scale, group, row, dI, d);
                double relu = dot > 0.0 ? dot : 0.0;
                I += (double)w[(int64_t)t * HI + j] * relu;
            }
            out[s] = I;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Top-K with the tie rule: higher score first, then lower position.        */
/* ------------------------------------------------------------------------ */

typedef struct {
    double score;
    int32_t pos;
} cand_t;

static int cmp_rank(const void *pa, const void *pb)
{
    const cand_t *a = (const cand_t *)pa, *b = (const cand_t *)pb;
    if (a->score > b->score)
        return -1;
    if (a->score < b->score)
        return 1;
    return (a->pos < b->pos) ? -1 : (a->pos > b->pos);   /* -0 == +0 here */
}

static int cmp_int(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/* idx[r, :] = the min(K, n_valid[r]) best positions of scores[r, 0:n_valid[r]]
 * by a full sort on (score desc, position asc), emitted in ascending position
 * order and padded with -1. */
void oracle_topk(int32_t n_rows, const double *scores, int64_t ld, const int32_t *n_valid,
                 int32_t K, int32_t *idx)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int32_t r = 0; r < n_rows; ++r) {
        int32_t nv = n_valid[r];
        int32_t *out = idx + (int64_t)r * K;
        cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (size_t)(nv > 0 ? nv : 1));
        for (int32_t s = 0; s < nv; ++s) {
            c[s].score = scores[(int64_t)r * ld + s];
            c[s].pos = s;
        }
        qsort(c, (size_t)nv, sizeof(cand_t), cmp_rank);
        int32_t take = nv < K ? nv : K;
        for (int32_t i = 0; i < take; ++i)
            out[i] = c[i].pos;
        qsort(out, (size_t)take, sizeof(int32_t), cmp_int);
        for (int32_t i = take; i < K; ++i)
            out[i] = -1;
        free(c);
    }
}

/* ------------------------------------------------------------------------ */
/* Sparse MLA attention over the selected latent rows.                      */
/* ------------------------------------------------------------------------ */

/* For token t = rows[r] in sequence b and head h, with the selected rows
 * S = { idx[r,i] : 0 <= idx[r,i] < seq_lens[b] } (entries -1 are skipped):
 *   z_i = scale * sum_{d<D} q[t,h,d] * kv[b, s_i, d]
 *   m = max_i z_i;  p_i = exp(z_i - m) / sum_i exp(z_i - m)
 *   out[r,h,:] = sum_i p_i * kv[b, s_i, 0:dc]        (value = latent part)
 *   lse[r,h] = m + log(sum_i exp(z_i - m))
 * No selected row: out = 0, lse = -inf.
 * q [T,H,D] (bf16-exact fp32), kv [B,Lmax,D] fp64 (bf16 values, or FP8
 * codes times their tile scale, exact in fp64), idx [n_rows, K];
 * out [n_rows, H, dc], lse [n_rows, H] (fp64). */
void oracle_sparse_mla(int32_t B, int32_t Lmax, const int32_t *cu_q, const int32_t *seq_lens,
                       int32_t H, int32_t D, int32_t dc, double scale, const float *q,
                       const double *kv, int32_t n_rows, const int32_t *rows, const int32_t *idx,
                       int32_t K, double *out, double *lse)
{
#pragma omp parallel for collapse(2) schedule(dynamic, 4)
    for (int32_t r = 0; r < n_rows; ++r) {
        for (int32_t h = 0; h < H; ++h) {
            int32_t t = rows[r];
            int32_t b = seq_of_token(cu_q, B, t);
            const float *qh = q + ((int64_t)t * H + h) * D;
            const int32_t *sel = idx + (int64_t)r * K;
            double *o = out + ((int64_t)r * H + h) * dc;
            double *z = (double *)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
            int32_t *rowid = (int32_t *)malloc(sizeof(int32_t) * (size_t)(K > 0 ? K : 1));
            int32_t n = 0;
            for (int32_t i = 0; i < K; ++i) {
                int32_t s = sel[i];
                if (s < 0 || s >= seq_lens[b])
                    continue;
                const double *kr = kv + ((int64_t)b * Lmax + s) * D;
                double dot = 0.0;
                for (int32_t d = 0; d < D; ++d)
                    dot += (double)qh[d] * kr[d];
                z[n] = scale * dot;
                rowid[n] = s;
                ++n;
            }
            for (int32_t d = 0; d < dc; ++d)
                o[d] = 0.0;
            if (n == 0) {
                lse[(int64_t)r * H + h] = -INFINITY;
            } else {
                double m = z[0];
                for (int32_t i = 1; i < n; ++i)
                    if (z[i] > m)
                        m = z[i];
                double l = 0.0;
                for (int32_t i = 0; i < n; ++i)
                    l += exp(z[i] - m);
                for (int32_t i = 0; i < n; ++i) {
                    double p = exp(z[i] - m) / l;
                    const double *vr = kv + ((int64_t)b * Lmax + rowid[i]) * D;
                    for (int32_t d = 0; d < dc; ++d)
                        o[d] += p * vr[d];
                }
                lse[(int64_t)r * H + h] = m + log(l);
            }
            free(z);
            free(rowid);
        }
    }
}

/* Number of worker threads OpenMP would use (for reporting). */
int32_t oracle_num_threads(void)
{
#ifdef _OPENMP
    return (int32_t)omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int32_t n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}
