/*
 * dsa_oracle.c -- plain, slow, fp64 CPU oracle for the DSA decode/verify step.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code, header, table or
 * helper with the CUDA path, and the CUDA path never calls it.
 *
 * What is computed (NaiveAI research page, naive.ai/en/research):
 *   - "Technical Details > Model Architecture": a lightweight indexer scores the
 *     full history; the backbone attends only to a selected subset.
 *   - "Technical Details > Hybrid SWA-DSA Architecture": DSA selects the top
 *     2,048 tokens; GQA with four KV groups; the indexer has 16 query heads.
 *   - "AI-Centered R&D in Practice": results must be bitwise-deterministic,
 *     which fixes a unique tie rule for the selection.
 *   - "NaiveRT > Optimizing inside the kernel": eight query heads per GPU under
 *     TP8, i.e. 64 backbone query heads in total.
 * The pages do not print the indexer formula.  Reading taken (the standard
 * DeepSeek Sparse Attention indexer, which the page names):
 *     I[t,s] = sum_j w[t,j] * ReLU( q_idx[t,j,:] . k[s,:] ),  j < 16, dim 64,
 * with k[s,:] = scale[s] * k8[s,:] for FP8-E4M3 keys (scale = 1 for bf16 keys).
 * Selection: for query t at position pos[t], candidates are s in [0, pos[t]];
 * if there are at most topk of them all are taken, else the topk largest I
 * under the order (I descending, s ascending).  The result is listed in
 * ascending s, padded with -1.  Attention: softmax over the selected s of
 * (q[t,h,:] . K[s,g,:]) / sqrt(128), g = h / 16, weighting V[s,g,:].
 *
 * Every function below is pinned by tests against something other than
 * itself (library routines, closed forms, brute force, hand-worked fixtures).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { NH = 64, NG = 4, HD = 128, NHI = 16, DI = 64 };

/* bfloat16 is the upper 16 bits of an IEEE-754 binary32 value. */
double dsa_oracle_bf16(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP 8-bit floating point, E4M3: sign, 4 exponent bits (bias 7), 3 mantissa
 * bits; exponent field 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; there is
 * no infinity, so S.1111.110 = 448 is the largest magnitude. */
double dsa_oracle_e4m3(uint8_t code)
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

static double key_elem(const void *k, int k_fp8, int64_t ld, int64_t s, int d)
{
    if (k_fp8)
        return dsa_oracle_e4m3(((const uint8_t *)k)[s * ld + d]);
    return dsa_oracle_bf16(((const uint16_t *)k)[s * ld + d]);
}

/* Indexer scores, fp64, natural summation order.
 *   q_idx [T][16][64] bf16 bits, w [T][16] f32, k [L][ld] bf16 bits or E4M3
 *   codes, k_scale [L] f32 or NULL (= 1), pos [T].
 *   out [T][L]: I[t,s] for s <= pos[t]; -inf where s > pos[t] (not visible). */
void dsa_oracle_index_scores(int T, int64_t L, const uint16_t *q_idx, const float *w,
                             const void *k, int k_fp8, int64_t k_ld, const float *k_scale,
                             const int32_t *pos, double *out)
{
    for (int t = 0; t < T; ++t) {
        double q[NHI][DI], wt[NHI];
        for (int j = 0; j < NHI; ++j) {
            wt[j] = (double)w[t * NHI + j];
            for (int d = 0; d < DI; ++d)
                q[j][d] = dsa_oracle_bf16(q_idx[((int64_t)t * NHI + j) * DI + d]);
        }
#pragma omp parallel for schedule(static)
        for (int64_t s = 0; s < L; ++s) {
            if (s > pos[t]) {
                out[(int64_t)t * L + s] = -INFINITY;
                continue;
            }
            double scale = k_scale ? (double)k_scale[s] : 1.0;
            double key[DI];
            for (int d = 0; d < DI; ++d)
                key[d] = scale * key_elem(k, k_fp8, k_ld, s, d);
            double acc = 0.0;
            for (int j = 0; j < NHI; ++j) {
                double dot = 0.0;
                for (int d = 0; d < DI; ++d)
                    dot += q[j][d] * key[d];
                acc += wt[j] * (dot > 0.0 ? dot : 0.0);
            }
            out[(int64_t)t * L + s] = acc;
        }
    }
}

/* A-priori magnitude used by the tests' error band: for each visible (t,s),
 *   scale[s] * sum_j |w[t,j]| * sum_d |q_idx[t,j,d] * k8[s,d]|.
 * Any evaluation of the indexer sum in fp32 differs from the exact value by a
 * small multiple of 2^-24 times this quantity. */
void dsa_oracle_index_magnitude(int T, int64_t L, const uint16_t *q_idx, const float *w,
                                const void *k, int k_fp8, int64_t k_ld, const float *k_scale,
                                const int32_t *pos, double *out)
{
    for (int t = 0; t < T; ++t) {
#pragma omp parallel for schedule(static)
        for (int64_t s = 0; s < L; ++s) {
            if (s > pos[t]) {
                out[(int64_t)t * L + s] = 0.0;
                continue;
            }
            double scale = k_scale ? (double)k_scale[s] : 1.0;
            double acc = 0.0;
            for (int j = 0; j < NHI; ++j) {
                double sum = 0.0;
                for (int d = 0; d < DI; ++d)
                    sum += fabs(dsa_oracle_bf16(q_idx[((int64_t)t * NHI + j) * DI + d]) *
                                key_elem(k, k_fp8, k_ld, s, d));
                acc += fabs((double)w[t * NHI + j]) * sum;
            }
            out[(int64_t)t * L + s] = fabs(scale) * acc;
        }
    }
}

typedef struct {
    double v;
    int64_t s;
} scored_t;

/* Larger score first; equal scores: lower position first. */
static int by_score_then_pos(const void *a, const void *b)
{
    const scored_t *x = (const scored_t *)a, *y = (const scored_t *)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->s < y->s) ? -1 : (x->s > y->s);
}

static int by_pos(const void *a, const void *b)
{
    const scored_t *x = (const scored_t *)a, *y = (const scored_t *)b;
    return (x->s < y->s) ? -1 : (x->s > y->s);
}

/* Causal top-k.  scores [T][ld] (row t uses s in [0, pos[t]]), sel [T][topk].
 * Returns 0, or -1 if a visible score is NaN (invalid input). */
int dsa_oracle_topk(int T, int64_t L, const double *scores, int64_t ld, const int32_t *pos,
                    int topk, int32_t *sel)
{
    (void)L;
    for (int t = 0; t < T; ++t) {
        int64_t n = (int64_t)pos[t] + 1;
        int32_t *row = sel + (int64_t)t * topk;
        if (n <= topk) {
            for (int64_t i = 0; i < topk; ++i)
                row[i] = i < n ? (int32_t)i : -1;
            continue;
        }
        scored_t *c = (scored_t *)malloc((size_t)n * sizeof *c);
        if (!c) return -2;
        for (int64_t s = 0; s < n; ++s) {
            c[s].v = scores[(int64_t)t * ld + s];
            c[s].s = s;
            if (isnan(c[s].v)) {
                free(c);
                return -1;
            }
        }
        qsort(c, (size_t)n, sizeof *c, by_score_then_pos);
        qsort(c, (size_t)topk, sizeof *c, by_pos);
        for (int i = 0; i < topk; ++i)
            row[i] = (int32_t)c[i].s;
        free(c);
    }
    return 0;
}

/* Sparse GQA attention over the selected rows, fp64.
 *   q [T][64][128] bf16 bits; kv [L][kv_ld] bf16 bits, a row holds K for the 4
 *   groups (4 x 128) then V for the 4 groups; sel [T][topk], entries < 0 are
 *   padding; sink: NULL, or a per-head logit [64] that joins the softmax
 *   denominator only (a sink with no value row).  out [T][64][128] fp64.
 * Returns 0, or -1 if a selected index is outside [0, L). */
int dsa_oracle_sparse_attn(int T, int64_t L, const uint16_t *q, const uint16_t *kv, int64_t kv_ld,
                           const int32_t *sel, int topk, const float *sink, double *out)
{
    const double inv_sqrt_d = 1.0 / sqrt((double)HD);
    for (int t = 0; t < T; ++t)
        for (int i = 0; i < topk; ++i) {
            int32_t s = sel[(int64_t)t * topk + i];
            if (s >= L) return -1;
        }
#pragma omp parallel for collapse(2) schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int h = 0; h < NH; ++h) {
            const int g = h / (NH / NG);
            const int32_t *row = sel + (int64_t)t * topk;
            double qv[HD];
            for (int d = 0; d < HD; ++d)
                qv[d] = dsa_oracle_bf16(q[((int64_t)t * NH + h) * HD + d]);
            double *z = (double *)malloc((size_t)topk * sizeof *z);
            double zmax = -INFINITY;
            for (int i = 0; i < topk; ++i) {
                z[i] = -INFINITY;
                if (row[i] < 0) continue;
                const uint16_t *K = kv + (int64_t)row[i] * kv_ld + (int64_t)g * HD;
                double dot = 0.0;
                for (int d = 0; d < HD; ++d)
                    dot += qv[d] * dsa_oracle_bf16(K[d]);
                z[i] = dot * inv_sqrt_d;
                if (z[i] > zmax) zmax = z[i];
            }
            if (sink && (double)sink[h] > zmax) zmax = (double)sink[h];
            double denom = sink ? exp((double)sink[h] - zmax) : 0.0;
            double acc[HD];
            for (int d = 0; d < HD; ++d) acc[d] = 0.0;
            for (int i = 0; i < topk; ++i) {
                if (row[i] < 0) continue;
                double p = exp(z[i] - zmax);
                denom += p;
                const uint16_t *V = kv + (int64_t)row[i] * kv_ld + (int64_t)NG * HD + (int64_t)g * HD;
                for (int d = 0; d < HD; ++d)
                    acc[d] += p * dsa_oracle_bf16(V[d]);
            }
            for (int d = 0; d < HD; ++d)
                out[((int64_t)t * NH + h) * HD + d] = denom > 0.0 ? acc[d] / denom : 0.0;
            free(z);
        }
    }
    return 0;
}

/* The whole step: scores, selection, attention.  scores_out (may be NULL)
 * receives the [T][L] fp64 scores. */
int dsa_oracle_decode(int T, int64_t L, const uint16_t *q, const uint16_t *q_idx, const float *w,
                      const void *k, int k_fp8, int64_t k_ld, const float *k_scale,
                      const uint16_t *kv, int64_t kv_ld, const int32_t *pos, int topk,
                      double *out, int32_t *sel, double *scores_out)
{
    double *sc = scores_out ? scores_out : (double *)malloc((size_t)T * (size_t)L * sizeof(double));
    if (!sc) return -2;
    dsa_oracle_index_scores(T, L, q_idx, w, k, k_fp8, k_ld, k_scale, pos, sc);
    int rc = dsa_oracle_topk(T, L, sc, L, pos, topk, sel);
    if (rc == 0)
        rc = dsa_oracle_sparse_attn(T, L, q, kv, kv_ld, sel, topk, NULL, out);
    if (!scores_out) free(sc);
    return rc;
}

int dsa_oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void dsa_oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
