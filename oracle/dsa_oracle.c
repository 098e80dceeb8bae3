/*
 * dsa_oracle.c -- plain, slow, fp64 CPU oracle for the GQA-adapted DeepSeek
 * Sparse Attention (DSA) layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or constant
 * with the CUDA library; the two meet only through the seeded input bytes.
 *
 * Sources (web pages on the Kwai Keye-VL-2.0 technical report):
 *   [REVIEW]  "Kwai Keye-VL-2.0 Technical Report" paper review
 *             (xllm-io.github.io), section 三 "技术架构", "核心公式":
 *             the lightning-indexer score, the top-k set Omega_t and the
 *             GQA sparse aggregation u_{t,g}.
 *   [REPORT]  "快手开源 Kwai Keye-VL-2.0-30B-A3B" (Chinese translation of the
 *             report), section 2.3.1 (MQA-style lightning indexer, one
 *             shared key head, FP8, ReLU scoring), section 2.3.2 (GQA sparse
 *             aggregation, one index set for all groups, k = 2048),
 *             section 5.1.2 (short-row rule: rows whose position is below k
 *             visit only the causally visible entries) and section 5.2.1
 *             (deterministic top-k).
 *
 * Everything is computed straight from the definitions, in double precision,
 * with no blocking, fusion or reordering.  OpenMP parallelises over query
 * rows only; each row is computed by one thread in a fixed order, so results
 * do not depend on the thread count.
 *
 * Readings of what the pages leave open (each repeated where it is used):
 *   - FP8 is OCP e4m3fn; a stored value means byte * per-token scale.
 *   - The causal range of query t is s in [0, t] (self included).
 *   - Top-k ties go to the lower key index; -0.0 and +0.0 are equal.
 *   - When t+1 <= k the set is all of [0, t].
 *   - GQA head h reads KV group g = h / (Hq / Hkv).
 *   - Attention is softmax(sm_scale * q.k) weighted sum of v.
 *   - Decode: the query sits at position seq_len-1 of its own cache.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------ */
/* Number formats                                                      */
/* ------------------------------------------------------------------ */

/* OCP 8-bit floating point, E4M3 "fn" variant: 1 sign bit, 4 exponent bits
 * with bias 7, 3 mantissa bits, no infinities, S.1111.111 is NaN.
 * Exponent field 0 holds subnormals m/8 * 2^(1-7). */
EXPORT double dsa_oracle_e4m3_to_double(uint8_t b)
{
    int sign = (b >> 7) & 1;
    int e = (b >> 3) & 0xF;
    int m = b & 0x7;
    double mag;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, 1 - 7);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* bfloat16 is the upper half of an IEEE binary32 pattern. */
EXPORT double dsa_oracle_bf16_to_double(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

EXPORT int dsa_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

EXPORT void dsa_oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------------ */
/* Lightning indexer ([REVIEW] 核心公式; [REPORT] 2.3.1)                */
/*   I[t,s] = sum_j w[t,j] * ReLU(qI[t,j] . kI[s]),  s <= t            */
/* qI[t,j,c] = e4m3(q8[t,j,c]) * sq[t];  kI[s,c] = e4m3(k8[s,c]) * sk[s] */
/* ------------------------------------------------------------------ */

static double indexer_pair(const uint8_t *q8_t, double sq_t, const float *w_t,
                           const uint8_t *k8_s, double sk_s, int HI, int dI)
{
    double I = 0.0;
    for (int j = 0; j < HI; ++j) {
        double dot = 0.0;
        for (int c = 0; c < dI; ++c) {
            double qv = dsa_oracle_e4m3_to_double(q8_t[(size_t)j * dI + c]) * sq_t;
            double kv = dsa_oracle_e4m3_to_double(k8_s[c]) * sk_s;
            dot += qv * kv;
        }
        double relu = dot > 0.0 ? dot : 0.0;
        I += (double)w_t[j] * relu;
    }
    return I;
}

/* Scores of query rows t in [row_begin, row_begin + n_rows) against every key
 * s in [0, t].  out[r*ld + s]; entries with s > t are set to -inf.
 * Needs ld >= row_begin + n_rows.  Returns 0, or -1 on bad arguments. */
EXPORT int dsa_oracle_indexer(const uint8_t *q8, const float *sq, const float *w,
                              const uint8_t *k8, const float *sk,
                              int L, int HI, int dI, int row_begin, int n_rows,
                              double *out, int64_t ld)
{
    if (L < 1 || HI < 1 || dI < 1 || row_begin < 0 || n_rows < 0 ||
        row_begin + n_rows > L || ld < row_begin + n_rows)
        return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < n_rows; ++r) {
        int t = row_begin + r;
        const uint8_t *q8_t = q8 + (size_t)t * HI * dI;
        double *row = out + (size_t)r * ld;
        for (int s = 0; s < row_begin + n_rows; ++s) {
            if (s > t) { row[s] = -INFINITY; continue; }
            row[s] = indexer_pair(q8_t, sq[t], w + (size_t)t * HI,
                                  k8 + (size_t)s * dI, sk[s], HI, dI);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Causal top-k ([REVIEW] Omega_t; [REPORT] 2.3.1, 5.1.2, 5.2.1)       */
/* ------------------------------------------------------------------ */

typedef struct { double v; int32_t s; } scored_t;

/* Descending score; equal scores (including -0.0 == +0.0) by ascending key
 * index.  The order is total, so the selection is deterministic. */
static int cmp_desc_then_index(const void *a, const void *b)
{
    const scored_t *x = (const scored_t *)a, *y = (const scored_t *)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->s > y->s) - (x->s < y->s);
}

static int cmp_int32(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* Row r holds n = row_len[r] candidate scores scores[r*ld + 0 .. n-1].
 * Writes idx[r*k + 0 .. k-1]: the selected key indices in ascending order,
 * padded with -1.  If n <= k every index 0..n-1 is selected. */
EXPORT int dsa_oracle_topk(const double *scores, int64_t ld, const int32_t *row_len,
                           int n_rows, int k, int32_t *idx)
{
    if (n_rows < 0 || k < 1) return -1;
    for (int r = 0; r < n_rows; ++r)
        if (row_len[r] < 0 || row_len[r] > ld) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < n_rows; ++r) {
        int n = row_len[r];
        int32_t *out = idx + (size_t)r * k;
        int take = n < k ? n : k;
        if (n <= k) {
            for (int i = 0; i < n; ++i) out[i] = i;
        } else {
            scored_t *tmp = (scored_t *)malloc(sizeof(scored_t) * (size_t)n);
            for (int s = 0; s < n; ++s) {
                tmp[s].v = scores[(size_t)r * ld + s];
                tmp[s].s = s;
            }
            qsort(tmp, (size_t)n, sizeof(scored_t), cmp_desc_then_index);
            for (int i = 0; i < k; ++i) out[i] = tmp[i].s;
            free(tmp);
            qsort(out, (size_t)k, sizeof(int32_t), cmp_int32);
        }
        for (int i = take; i < k; ++i) out[i] = -1;
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* GQA sparse aggregation ([REVIEW] u_{t,g}; [REPORT] 2.3.2)           */
/*   O[t,h] = sum_{s in Omega_t} softmax_s(sm * Q[t,h].K[s,g]) V[s,g]  */
/*   g = h / (Hq/Hkv); the same Omega_t for every group g.             */
/* ------------------------------------------------------------------ */

/* One query row, one head: krows[i] / vrows[i] point at the D values of the
 * i-th selected key and value row (already resolved to the head's group). */
static void attend_one(const uint16_t *q_h, int D, double sm_scale,
                       const uint16_t *const *krows, const uint16_t *const *vrows, int n,
                       double *o_h, double *lse_h)
{
    if (n == 0) {
        for (int d = 0; d < D; ++d) o_h[d] = 0.0;
        if (lse_h) *lse_h = -INFINITY;
        return;
    }
    double *logit = (double *)malloc(sizeof(double) * (size_t)n);
    double m = -INFINITY;
    for (int i = 0; i < n; ++i) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += dsa_oracle_bf16_to_double(q_h[d]) * dsa_oracle_bf16_to_double(krows[i][d]);
        logit[i] = sm_scale * dot;
        if (logit[i] > m) m = logit[i];
    }
    double denom = 0.0;
    for (int d = 0; d < D; ++d) o_h[d] = 0.0;
    for (int i = 0; i < n; ++i) {
        double p = exp(logit[i] - m);
        denom += p;
        for (int d = 0; d < D; ++d) o_h[d] += p * dsa_oracle_bf16_to_double(vrows[i][d]);
    }
    for (int d = 0; d < D; ++d) o_h[d] /= denom;
    if (lse_h) *lse_h = m + log(denom);
    free(logit);
}

/* Prefill.  Query rows t in [row_begin, row_begin + n_rows).
 * Q is [n_rows, Hq, D] (row 0 is query t = row_begin), K and V are
 * [>= row_begin + n_rows, Hkv, D], all bf16 bit patterns.  idx is
 * [n_rows, k]; entries outside [0, t] (the -1 padding) are not part of
 * Omega_t.  O is [n_rows, Hq, D], lse (nullable) is [n_rows, Hq]. */
EXPORT int dsa_oracle_sparse_attention(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                                       const int32_t *idx, int row_begin, int n_rows,
                                       int Hq, int Hkv, int D, int k, double sm_scale,
                                       double *O, double *lse)
{
    if (n_rows < 0 || row_begin < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv || D < 1 || k < 1)
        return -1;
    int G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < n_rows; ++r) {
        int t = row_begin + r;
        const uint16_t **kr = (const uint16_t **)malloc(sizeof(void *) * (size_t)k);
        const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * (size_t)k);
        for (int h = 0; h < Hq; ++h) {
            int g = h / G;
            int n = 0;
            for (int i = 0; i < k; ++i) {
                int32_t s = idx[(size_t)r * k + i];
                if (s < 0 || s > t) continue;
                kr[n] = K + ((size_t)s * Hkv + g) * D;
                vr[n] = V + ((size_t)s * Hkv + g) * D;
                ++n;
            }
            attend_one(Q + ((size_t)r * Hq + h) * D, D, sm_scale, kr, vr, n,
                       O + ((size_t)r * Hq + h) * D, lse ? lse + (size_t)r * Hq + h : NULL);
        }
        free(kr);
        free(vr);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Decode over a paged cache.  A sequence's logical token s lives in   */
/* page block_table[b, s / page] at slot s % page.                      */
/* ------------------------------------------------------------------ */

/* Indexer for one query per sequence (position seq_len-1) against every
 * cached key s in [0, seq_len).  q8 [B,HI,dI], sq [B], w [B,HI];
 * k8_cache [P,page,dI], sk_cache [P,page]; out[b*ld + s], -inf past seq_len. */
EXPORT int dsa_oracle_decode_indexer(const uint8_t *q8, const float *sq, const float *w,
                                     const uint8_t *k8_cache, const float *sk_cache,
                                     const int32_t *block_table, int max_pages, int page, int num_pages,
                                     const int32_t *seq_lens, int B, int HI, int dI,
                                     double *out, int64_t ld)
{
    if (B < 0 || HI < 1 || dI < 1 || page < 1 || max_pages < 1 || num_pages < 1) return -1;
    for (int b = 0; b < B; ++b)
        if (seq_lens[b] < 0 || seq_lens[b] > ld || seq_lens[b] > (int64_t)max_pages * page) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        for (int64_t s = 0; s < ld; ++s) {
            if (s >= seq_lens[b]) { out[(size_t)b * ld + s] = -INFINITY; continue; }
            int32_t p = block_table[(size_t)b * max_pages + s / page];
            /* library convention (not from the papers): a token whose page id
             * is not a cache page has no key and scores -inf */
            if (p < 0 || p >= num_pages) { out[(size_t)b * ld + s] = -INFINITY; continue; }
            size_t slot = (size_t)p * page + (size_t)(s % page);
            out[(size_t)b * ld + s] = indexer_pair(q8 + (size_t)b * HI * dI, sq[b], w + (size_t)b * HI,
                                                   k8_cache + slot * dI, sk_cache[slot], HI, dI);
        }
    }
    return 0;
}

/* Attention for one query per sequence over the selected cached rows.
 * q [B,Hq,D]; k_cache, v_cache [P,page,Hkv,D]; idx [B,k] (entries outside
 * [0, seq_len) or on a page id outside [0, num_pages) are ignored);
 * out [B,Hq,D]; lse nullable [B,Hq]. */
EXPORT int dsa_oracle_decode_attention(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                                       const int32_t *block_table, int max_pages, int page, int num_pages,
                                       const int32_t *seq_lens, const int32_t *idx,
                                       int B, int Hq, int Hkv, int D, int k, double sm_scale,
                                       double *out, double *lse)
{
    if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv || D < 1 || k < 1 || page < 1 || num_pages < 1) return -1;
    int G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        const uint16_t **kr = (const uint16_t **)malloc(sizeof(void *) * (size_t)k);
        const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * (size_t)k);
        for (int h = 0; h < Hq; ++h) {
            int g = h / G;
            int n = 0;
            for (int i = 0; i < k; ++i) {
                int32_t s = idx[(size_t)b * k + i];
                if (s < 0 || s >= seq_lens[b]) continue;
                int32_t p = block_table[(size_t)b * max_pages + s / page];
                if (p < 0 || p >= num_pages) continue; /* unmapped page: no key, skipped */
                size_t slot = (size_t)p * page + (size_t)(s % page);
                kr[n] = k_cache + (slot * Hkv + g) * D;
                vr[n] = v_cache + (slot * Hkv + g) * D;
                ++n;
            }
            attend_one(q + ((size_t)b * Hq + h) * D, D, sm_scale, kr, vr, n,
                       out + ((size_t)b * Hq + h) * D, lse ? lse + (size_t)b * Hq + h : NULL);
        }
        free(kr);
        free(vr);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Indexer distillation losses                                         */
/* ------------------------------------------------------------------ */

/* [REVIEW] 核心公式, dense warm-up and sparse adaptation losses of the
 * indexer; [REPORT] 2.3.3 (the target of group g is the group's aggregated
 * dense attention, normalised; in the sparse stage it is truncated to the
 * selected set S_t and renormalised, and the softmax of the indexer scores is
 * taken over S_t only):
 *   dense:  L = sum_t sum_g KL( p[t,:,g]   || Softmax(I[t,:])   )
 *   sparse: L = sum_t sum_g KL( p[t,S_t,g] || Softmax(I[t,S_t]) )
 * KL(a || b) = sum_s a_s log(a_s / b_s), with 0 log 0 = 0.
 *
 * Row r is query t = row_begin + r.  I [n_rows, ld_I]: scores of keys
 * 0..t.  p [n_rows, G, ld_p]: non-negative target weights of keys 0..t
 * (normalised here over the set, so a scaled target gives the same loss).
 * idx NULL: S_t = [0, t] (dense); otherwise S_t = the entries of idx row r
 * that lie in [0, t] (k of them at most, -1 padded, distinct).
 * Readings: the causal range [0, t] is the one the indexer scores; a group
 * whose target has no mass on S_t contributes 0.
 * loss [n_rows] receives sum_g KL for each row, *total their sum. */
EXPORT int dsa_oracle_indexer_kl(const double *I, int64_t ld_I, int row_begin, int n_rows,
                                 const double *p, int G, int64_t ld_p, const int32_t *idx, int k,
                                 double *loss, double *total)
{
    if (row_begin < 0 || n_rows < 0 || G < 1 || (idx && k < 1)) return -1;
    if (ld_I < row_begin + n_rows || ld_p < row_begin + n_rows) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < n_rows; ++r) {
        int t = row_begin + r;
        /* the set S_t */
        int n = idx ? 0 : t + 1;
        int32_t *S = (int32_t *)malloc(sizeof(int32_t) * (size_t)(idx ? k : t + 1));
        if (idx) {
            for (int i = 0; i < k; ++i) {
                int32_t s = idx[(size_t)r * k + i];
                if (s >= 0 && s <= t) S[n++] = s;
            }
        } else {
            for (int s = 0; s <= t; ++s) S[s] = s;
        }
        const double *Ir = I + (size_t)r * ld_I;
        /* Softmax(I[t, S]) as log-probabilities: log q_s = I_s - log sum_u exp(I_u) */
        double mx = -INFINITY;
        for (int i = 0; i < n; ++i) if (Ir[S[i]] > mx) mx = Ir[S[i]];
        double z = 0.0;
        for (int i = 0; i < n; ++i) z += exp(Ir[S[i]] - mx);
        double logz = mx + log(z);
        double row_loss = 0.0;
        for (int g = 0; g < G; ++g) {
            const double *pr = p + ((size_t)r * G + g) * ld_p;
            double mass = 0.0;
            for (int i = 0; i < n; ++i) mass += pr[S[i]];
            if (!(mass > 0.0)) continue;
            double kl = 0.0;
            for (int i = 0; i < n; ++i) {
                double a = pr[S[i]] / mass;
                if (a > 0.0) kl += a * (log(a) - (Ir[S[i]] - logz));
            }
            row_loss += kl;
        }
        loss[r] = row_loss;
        free(S);
    }
    double sum = 0.0;
    for (int r = 0; r < n_rows; ++r) sum += loss[r];
    *total = sum;
    return 0;
}
