/*
 * CPU oracle for the DeepSeek Sparse Attention (DSA) forward path.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the package smoke check and
 * the benchmark's CPU-baseline leg may load this library. The product path
 * (the CUDA library and its Python binding) never calls it, and it shares no
 * code, header, table or helper with the CUDA sources.
 *
 * Plain, slow, obviously correct: one query row at a time, fp64 arithmetic,
 * no blocking, no fusion, no reordering beyond what the definitions state.
 * OpenMP only spreads independent query rows over host cores.
 *
 * Sources (page title, section, equation):
 *   "DeepSeek Sparse Attention: Learned Token Selection from Scratch"
 *     §2.1, boxed equation for I_{t,s}     -> oracle_indexer_rows
 *     §3.1, boxed equation for S_t         -> oracle_topk_rows
 *     §3.4, always including the current token -> oracle_topk_self_rows
 *     §3.3, equations for alpha and u_t;
 *     §10.1, the common attention form     -> oracle_attn_rows
 *     §4.1-4.2, one selected set shared by every head (MQA mode of MLA)
 *   "Sparse Attention LLM Design: Native Sparse Attention and DeepSeek Sparse
 *    Attention", section "Implemented on MLA's MQA mode" (one selection per
 *    token, read by every query head).
 *
 * Readings of points the pages leave open (each one is also listed in the
 * design notes of the repository):
 *   - candidates for query position t are the positions s <= t;
 *   - equal scores are ordered by position, the lower position first;
 *   - when t+1 <= k every candidate is kept (a consequence of taking the
 *     first min(t+1, k) entries of the sorted candidates);
 *   - the selected set is emitted in ascending position order, padded
 *     with -1 up to k entries;
 *   - scores are computed in fp64 and then rounded to fp32, and the
 *     selection compares those fp32 values (the precision the GPU path
 *     stores them in); -0.0 and +0.0 compare equal, as in C;
 *   - positions s > t are written as -inf in the score rows.
 *
 * Parity pins: the fp64 results are checked, independently of this file,
 * against the hand-traced t=10 example of "Learned Token Selection", brute-force
 * sorting, closed-form counts and library dense attention (see tests/).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1, ORACLE_E4M3 = 2 };

/* Value of an 8-bit e4m3 code (the FP8 format the pages suggest for the
 * indexer, "Learned Token Selection" §7.4): 1 sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits; exponent 0 holds the subnormals m/8 * 2^-6; the
 * one non-finite pattern per sign, exponent 15 with mantissa 7, is NaN (the
 * format has no infinities). */
static double e4m3_value(uint8_t code)
{
    const int sign = code >> 7;
    const int e = (code >> 3) & 15;
    const int m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Read element i of an array stored as fp32, as raw bf16 bits, or as e4m3
 * codes. A bf16 value is the top half of an fp32 bit pattern, so the widening
 * is exact; every e4m3 value is exact in a double. */
static double load_value(const void *base, size_t i, int dtype)
{
    if (dtype == ORACLE_F32) {
        return (double)((const float *)base)[i];
    }
    if (dtype == ORACLE_E4M3) {
        return e4m3_value(((const uint8_t *)base)[i]);
    }
    uint32_t bits = (uint32_t)((const uint16_t *)base)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* The decoded values of n e4m3 codes (for the pins of the decoding). */
void oracle_e4m3_decode(int n, const uint8_t *codes, double *out)
{
    for (int i = 0; i < n; ++i) out[i] = e4m3_value(codes[i]);
}

static void set_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Lightning-indexer scores, "Learned Token Selection" §2.1:
 *   I[t,s] = sum_{j=1..H} w[t,j] * ReLU( q[t,j] . k[s] )
 * for s = 0..t; s > t is not a candidate and is written as -inf.
 *
 * nrows query rows are evaluated. Row r belongs to batch entry row_b[r] and
 * sits at absolute position row_t[r].
 *   q_rows : [nrows, H, d]  indexer queries of those rows (dtype)
 *   w_rows : [nrows, H]     fp32 head weights of those rows
 *   k_cache: [B, L, d]      indexer keys, one per position (dtype)
 *   scores : [nrows, L]     fp32 output
 */
void oracle_indexer_rows(int nrows, const int32_t *row_b, const int32_t *row_t,
                         const void *q_rows, const float *w_rows,
                         const void *k_cache, int dtype, int L, int H, int d,
                         float *scores, int nthreads)
{
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        const int b = row_b[r];
        const int t = row_t[r];
        double *q = (double *)malloc(sizeof(double) * (size_t)H * d);
        double *key = (double *)malloc(sizeof(double) * (size_t)d);
        for (int j = 0; j < H; ++j)
            for (int e = 0; e < d; ++e)
                q[(size_t)j * d + e] = load_value(q_rows, ((size_t)r * H + j) * d + e, dtype);

        float *out = scores + (size_t)r * L;
        for (int s = 0; s < L; ++s) {
            if (s > t) {
                out[s] = -INFINITY;
                continue;
            }
            for (int e = 0; e < d; ++e)
                key[e] = load_value(k_cache, ((size_t)b * L + s) * d + e, dtype);
            double I = 0.0;
            for (int j = 0; j < H; ++j) {
                double dot = 0.0;
                for (int e = 0; e < d; ++e) dot += q[(size_t)j * d + e] * key[e];
                double relu = dot > 0.0 ? dot : 0.0;
                I += (double)w_rows[(size_t)r * H + j] * relu;
            }
            out[s] = (float)I;
        }
        free(key);
        free(q);
    }
}

typedef struct {
    float score;
    int32_t pos;
} candidate;

/* Descending score; equal scores keep the lower position first. This makes
 * the order total, so the sort below is equivalent to a stable sort of the
 * candidates by descending score. */
static int by_score_then_pos(const void *pa, const void *pb)
{
    const candidate *a = (const candidate *)pa;
    const candidate *b = (const candidate *)pb;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    return (a->pos > b->pos) - (a->pos < b->pos);
}

static int ascending_int(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/*
 * Top-k selection, "Learned Token Selection" §3.1: S_t holds the positions of the k largest
 * I[t,s] over the candidates s = 0..t. Brute force: sort every candidate by
 * (descending score, ascending position) and keep the first min(t+1, k).
 *   scores: [nrows, L] fp32 (only entries 0..row_t[r] are read)
 *   idx   : [nrows, k] int32, ascending positions, then -1 padding
 */
void oracle_topk_rows(int nrows, const int32_t *row_t, const float *scores,
                      int L, int k, int32_t *idx, int nthreads)
{
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        const int n = row_t[r] + 1;
        candidate *c = (candidate *)malloc(sizeof(candidate) * (size_t)n);
        for (int s = 0; s < n; ++s) {
            c[s].score = scores[(size_t)r * L + s];
            c[s].pos = s;
        }
        qsort(c, (size_t)n, sizeof(candidate), by_score_then_pos);
        const int keep = n < k ? n : k;
        int32_t *out = idx + (size_t)r * k;
        for (int j = 0; j < keep; ++j) out[j] = c[j].pos;
        qsort(out, (size_t)keep, sizeof(int32_t), ascending_int);
        for (int j = keep; j < k; ++j) out[j] = -1;
        free(c);
    }
}

/*
 * Top-k selection that always keeps the query's own position
 * ("Learned Token Selection" §3.4: a token whose own score does not reach
 * the top k is kept by always including the current token):
 *
 *   S_t = {t} united with the min(t, k-1) highest-scoring positions of 0..t-1
 *
 * with the same order and tie rule as oracle_topk_rows. When t+1 <= k this is
 * every candidate, as without the rule.
 */
void oracle_topk_self_rows(int nrows, const int32_t *row_t, const float *scores,
                           int L, int k, int32_t *idx, int nthreads)
{
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        const int t = row_t[r];
        /* the candidates other than t itself */
        candidate *c = (candidate *)malloc(sizeof(candidate) * (size_t)(t > 0 ? t : 1));
        for (int s = 0; s < t; ++s) {
            c[s].score = scores[(size_t)r * L + s];
            c[s].pos = s;
        }
        qsort(c, (size_t)t, sizeof(candidate), by_score_then_pos);
        const int others = t < k - 1 ? t : k - 1;
        int32_t *out = idx + (size_t)r * k;
        for (int j = 0; j < others; ++j) out[j] = c[j].pos;
        out[others] = t;
        qsort(out, (size_t)others + 1, sizeof(int32_t), ascending_int);
        for (int j = others + 1; j < k; ++j) out[j] = -1;
        free(c);
    }
}

/*
 * Attention restricted to the selected set, "Learned Token Selection" §3.3 and §10.1:
 *   alpha[t,h,s] = exp(q[t,h].k[s,g]*scale) / sum_{s' in S_t} exp(q[t,h].k[s',g]*scale)
 *   u[t,h]       = sum_{s in S_t} alpha[t,h,s] * v[s,g]
 * Every query head h uses the same S_t ("Learned Token Selection" §4.1-4.2); head h reads
 * KV head g = h / (Hq / Hkv). idx entries of -1 are padding and skipped.
 * The max is subtracted before exp (the result is unchanged).
 *   q_rows : [nrows, Hq, Dqk] (dtype)
 *   k_cache: element (b, s, g, e) at b*k_sb + s*k_ss + g*k_sh + e (dtype)
 *   v_cache: element (b, s, g, e) at b*v_sb + s*v_ss + g*v_sh + e (dtype)
 *   idx    : [nrows, k] int32
 *   out    : [nrows, Hq, Dv] fp64;  lse: [nrows, Hq] fp64 or NULL
 *            (lse = log sum_{s in S_t} exp(scale * q.k_s))
 */
void oracle_attn_rows(int nrows, const int32_t *row_b, const void *q_rows,
                      const void *k_cache, const void *v_cache, int dtype,
                      int64_t k_sb, int64_t k_ss, int64_t k_sh,
                      int64_t v_sb, int64_t v_ss, int64_t v_sh,
                      const int32_t *idx, int k, int Hq, int Hkv, int Dqk, int Dv,
                      double scale, double *out, double *lse, int nthreads)
{
    set_threads(nthreads);
    const int group = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        const int b = row_b[r];
        const int32_t *sel = idx + (size_t)r * k;
        double *z = (double *)malloc(sizeof(double) * (size_t)k);
        for (int h = 0; h < Hq; ++h) {
            const int g = h / group;
            double zmax = -INFINITY;
            for (int j = 0; j < k; ++j) {
                const int s = sel[j];
                if (s < 0) continue;
                double dot = 0.0;
                for (int e = 0; e < Dqk; ++e) {
                    double qv = load_value(q_rows, ((size_t)r * Hq + h) * Dqk + e, dtype);
                    double kv = load_value(k_cache, (size_t)(b * k_sb + s * k_ss + g * k_sh + e), dtype);
                    dot += qv * kv;
                }
                z[j] = dot * scale;
                if (z[j] > zmax) zmax = z[j];
            }
            double *u = out + ((size_t)r * Hq + h) * Dv;
            for (int e = 0; e < Dv; ++e) u[e] = 0.0;
            double denom = 0.0;
            for (int j = 0; j < k; ++j) {
                const int s = sel[j];
                if (s < 0) continue;
                const double p = exp(z[j] - zmax);
                denom += p;
                for (int e = 0; e < Dv; ++e)
                    u[e] += p * load_value(v_cache, (size_t)(b * v_sb + s * v_ss + g * v_sh + e), dtype);
            }
            if (denom > 0.0)
                for (int e = 0; e < Dv; ++e) u[e] /= denom;
            if (lse) lse[(size_t)r * Hq + h] = denom > 0.0 ? zmax + log(denom) : -INFINITY;
        }
        free(z);
    }
}
