/*
 * tri_oracle.c -- plain fp64 CPU definition of TriAttention's KV-cache
 * scoring-and-pruning pass.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or calls
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do. It shares no code, header, table or helper with the CUDA library.
 *
 * Pages cited (titles; sections as headed on each page):
 *   [Deep-dive]  "TriAttention深度解析：用三角函数革命性压缩KV Cache，让长推理从「显存地狱」中脱困"
 *                (chenxutan.com/d/2624)
 *   [Stage]      "旋转舞台上的追光者——TriAttention如何用三角函数破解长文本推理的内存困局"
 *                (zhichai.net/topic/177169654)
 *   [10100]      the 10100.com article 127765992 on TriAttention (untitled extract)
 *   [Summary]    "TriAttention：面向长文本推理的高效KV缓存压缩，2.5倍吞吐提升与10.7倍内存缩减"
 *                (watermelonwater.tech)
 *
 * What is computed, per unit (one sequence, layer and KV head; N cached keys):
 *   1. RoPE frequencies omega_f = base^(-2f/d), f < F = d/2 ([Deep-dive] §4.4
 *      apply_rope; [Stage] §RoPE回顾). A band is a complex number made of two
 *      dims: (f, f+F) in the "half" layout, (2f, 2f+1) in the "interleaved" one.
 *   2. Each stored (post-RoPE) key band is un-rotated by its position,
 *      k_f = k~_f * e^{-i omega_f p}, giving the pre-RoPE key band.
 *   3. Trigonometric-series score ([Stage] §TriAttention：把理论变成算法 item 1):
 *        S_trig(k, Delta) = sum_f |qbar_f| |k_f| cos(omega_f Delta + phi_f),
 *      with phi_f = arg qbar_f - arg k_f and Delta = (t + delta) - p, averaged
 *      over the future offsets delta in D ([Deep-dive] §3.3 gives the
 *      geometric set D = {1, 2, 4, ..., 2^16}; its code takes the max over
 *      delta, the average is the reading adopted here because it is the one
 *      that the pass being checked computes).
 *   4. Norm score ([Stage] item 2), weighted per band by (1 - R_f) and added
 *      to S_trig as [10100] §TriAttention方法 describes:
 *        S_norm(k) = sum_f (1 - R_f) E|q_f| |k_f|.
 *   5. s_h = mean_delta S_trig + S_norm for each query head h of the group.
 *   6. GQA aggregation ([10100] §TriAttention方法, last paragraph; [Summary]
 *      §方案设计 item 4): z-score each head's scores over the unit's keys
 *      (population standard deviation; a head whose scores are all equal gets
 *      z = 0), then take the max over the group's heads.
 *   7. Keep the B keys with the largest max-z, ties to the lower slot (the
 *      lower position, since positions ascend within a unit), and restore the
 *      original order ([Deep-dive] §4 prune_kv_cache: top-k then sort).
 *   8. Gather K, V and position rows at the kept slots into slots 0..M-1.
 *
 * Nothing is folded, blocked or reordered beyond hoisting per-key and
 * per-head quantities out of the offset loop; the cosine series is summed
 * literally over every delta and every band.
 *
 * The calibration statistics the pass consumes (tri_oracle_calibrate) are the
 * means over T calibration tokens of the pre-RoPE query bands ([Deep-dive]
 * §3.4 offline calibration; [Stage] §TriAttention：把理论变成算法 items 1-2):
 * the complex centre E[q_f], the mean modulus E|q_f|, and the concentration
 * R_f = |E[q_f]| / E|q_f| of [Stage] §破局之道, taken per band.
 *
 * The consumer of the pruned cache (tri_oracle_decode_attention) is the standard scaled
 * dot-product attention of each query head over the unit's kept rows: softmax of
 * q.k / sqrt(d) over the keys, applied to the values, as the page "TriAttention 深度解析：
 * MIT韩松团队如何用三角函数让单卡4090跑出百万Token上下文" writes it out in its section 二.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define TRI_ORACLE_HALF 0
#define TRI_ORACLE_INTERLEAVED 1

/* A bf16 value is, by definition, the fp32 value whose upper 16 bits are its
 * bits and whose lower 16 bits are zero. */
static double bf16_value(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Dims (re, im) that make up band f. */
static void band_dims(int d, int layout, int f, int *re, int *im)
{
    if (layout == TRI_ORACLE_HALF) {
        *re = f;
        *im = f + d / 2;
    } else {
        *re = 2 * f;
        *im = 2 * f + 1;
    }
}

int tri_oracle_version(void) { return 1; }

/*
 * Scores of one unit.
 *   K       [N][d] bf16 bits of the stored (post-RoPE) keys
 *   pos     [N] positions of the keys
 *   t       query position; future queries sit at t + delta
 *   q_mean  [G][d] pre-RoPE query centres, same dim layout as the keys
 *   q_norm  [G][F] E|q_f|;   R [G][F] concentration R_f
 *   offsets [n_off] the set D
 * Outputs s [G][N] (and optionally the two terms separately).
 * Returns 0, or -1 on bad arguments.
 */
#define TRI_ORACLE_MEAN_OVER_DELTA 0
#define TRI_ORACLE_MAX_OVER_DELTA 1

static int unit_scores(int combine, int d, int G, int layout, double base,
                       const int64_t *offsets, int n_off, int64_t t,
                       const float *q_mean, const float *q_norm, const float *R,
                       const uint16_t *K, const int32_t *pos, int N,
                       double *s_out, double *trig_out, double *norm_out)
{
    if (d < 2 || (d & 1) || G < 1 || N < 0 || n_off < 1 || !offsets || !s_out)
        return -1;
    const int F = d / 2;
    double *omega = (double *)malloc(sizeof(double) * F);
    double *qmag = (double *)malloc(sizeof(double) * G * F);
    double *qarg = (double *)malloc(sizeof(double) * G * F);
    double *kmag = (double *)malloc(sizeof(double) * F);
    double *karg = (double *)malloc(sizeof(double) * F);
    if (!omega || !qmag || !qarg || !kmag || !karg) {
        free(omega); free(qmag); free(qarg); free(kmag); free(karg);
        return -1;
    }
    for (int f = 0; f < F; ++f)
        omega[f] = pow(base, -2.0 * (double)f / (double)d);
    for (int h = 0; h < G; ++h) {
        for (int f = 0; f < F; ++f) {
            int re, im;
            band_dims(d, layout, f, &re, &im);
            double a = q_mean[(size_t)h * d + re];
            double b = q_mean[(size_t)h * d + im];
            qmag[h * F + f] = sqrt(a * a + b * b);
            qarg[h * F + f] = atan2(b, a);
        }
    }
    for (int i = 0; i < N; ++i) {
        const double p = (double)pos[i];
        for (int f = 0; f < F; ++f) {
            int re, im;
            band_dims(d, layout, f, &re, &im);
            double xr = bf16_value(K[(size_t)i * d + re]);
            double xi = bf16_value(K[(size_t)i * d + im]);
            /* k_f = k~_f * e^{-i omega_f p} */
            double c = cos(omega[f] * p), sn = sin(omega[f] * p);
            double pr = xr * c + xi * sn;
            double pi = -xr * sn + xi * c;
            kmag[f] = sqrt(pr * pr + pi * pi);
            karg[f] = atan2(pi, pr);
        }
        for (int h = 0; h < G; ++h) {
            double trig = 0.0, best = 0.0;
            for (int j = 0; j < n_off; ++j) {
                const double delta = (double)((int64_t)t + offsets[j]) - p;
                double series = 0.0;
                for (int f = 0; f < F; ++f) {
                    const double phi = qarg[h * F + f] - karg[f];
                    series += qmag[h * F + f] * kmag[f] * cos(omega[f] * delta + phi);
                }
                trig += series;
                if (j == 0 || series > best) best = series;
            }
            trig /= (double)n_off;
            if (combine == TRI_ORACLE_MAX_OVER_DELTA) trig = best;
            double norm = 0.0;
            for (int f = 0; f < F; ++f)
                norm += (1.0 - (double)R[h * F + f]) * (double)q_norm[h * F + f] * kmag[f];
            s_out[(size_t)h * N + i] = trig + norm;
            if (trig_out) trig_out[(size_t)h * N + i] = trig;
            if (norm_out) norm_out[(size_t)h * N + i] = norm;
        }
    }
    free(omega); free(qmag); free(qarg); free(kmag); free(karg);
    return 0;
}

int tri_oracle_unit_scores(int d, int G, int layout, double base,
                           const int64_t *offsets, int n_off, int64_t t,
                           const float *q_mean, const float *q_norm, const float *R,
                           const uint16_t *K, const int32_t *pos, int N,
                           double *s_out, double *trig_out, double *norm_out)
{
    return unit_scores(TRI_ORACLE_MEAN_OVER_DELTA, d, G, layout, base, offsets, n_off, t, q_mean, q_norm, R,
                       K, pos, N, s_out, trig_out, norm_out);
}

/*
 * The same scores with the offsets combined by the maximum instead of the mean: the
 * trigonometric term is max over delta of S_trig(k, t + delta - p), the reading of
 * [Deep-dive] §3.3 and of the listing of its §4.2 (where the norm score is then added).
 * The pass built on the GPU uses the mean; this mode is the definition for a variant.
 */
int tri_oracle_unit_scores_max(int d, int G, int layout, double base,
                               const int64_t *offsets, int n_off, int64_t t,
                               const float *q_mean, const float *q_norm, const float *R,
                               const uint16_t *K, const int32_t *pos, int N,
                               double *s_out, double *trig_out, double *norm_out)
{
    return unit_scores(TRI_ORACLE_MAX_OVER_DELTA, d, G, layout, base, offsets, n_off, t, q_mean, q_norm, R,
                       K, pos, N, s_out, trig_out, norm_out);
}

/*
 * z-score per head over the N keys (population std, two passes), then the
 * max over the G heads. A head whose scores are all equal (its standard
 * deviation is zero) contributes z = 0 for every key.
 */
int tri_oracle_zmax(int G, int N, const double *s, double *z_out, double *zmax_out)
{
    if (G < 1 || N < 0 || !s || !zmax_out)
        return -1;
    for (int i = 0; i < N; ++i)
        zmax_out[i] = -INFINITY;
    for (int h = 0; h < G; ++h) {
        const double *sh = s + (size_t)h * N;
        double lo = INFINITY, hi = -INFINITY, sum = 0.0;
        for (int i = 0; i < N; ++i) {
            sum += sh[i];
            if (sh[i] < lo) lo = sh[i];
            if (sh[i] > hi) hi = sh[i];
        }
        const double mu = N > 0 ? sum / (double)N : 0.0;
        double m2 = 0.0;
        for (int i = 0; i < N; ++i)
            m2 += (sh[i] - mu) * (sh[i] - mu);
        const double sigma = N > 0 ? sqrt(m2 / (double)N) : 0.0;
        const int flat = !(hi > lo);
        for (int i = 0; i < N; ++i) {
            double z = flat ? 0.0 : (sh[i] - mu) / sigma;
            if (z_out) z_out[(size_t)h * N + i] = z;
            if (z > zmax_out[i]) zmax_out[i] = z;
        }
    }
    return 0;
}

typedef struct { double z; int32_t i; } ranked;

/* Larger z first; among equal z, the lower slot first. */
static int rank_cmp(const void *pa, const void *pb)
{
    const ranked *a = (const ranked *)pa, *b = (const ranked *)pb;
    if (a->z > b->z) return -1;
    if (a->z < b->z) return 1;
    return (a->i > b->i) - (a->i < b->i);
}

static int idx_cmp(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/* Top-B slots by zmax (ties to the lower slot), returned in ascending slot
 * order. Returns the kept count min(N, B), or -1 on bad arguments. */
int tri_oracle_select(int N, int B, const double *zmax, int32_t *kept_out)
{
    if (N < 0 || B < 1 || (N > 0 && (!zmax || !kept_out)))
        return -1;
    const int M = N < B ? N : B;
    if (M == 0) return 0;
    ranked *r = (ranked *)malloc(sizeof(ranked) * (size_t)N);
    if (!r) return -1;
    for (int i = 0; i < N; ++i) { r[i].z = zmax[i]; r[i].i = i; }
    qsort(r, (size_t)N, sizeof(ranked), rank_cmp);
    for (int j = 0; j < M; ++j) kept_out[j] = r[j].i;
    free(r);
    qsort(kept_out, (size_t)M, sizeof(int32_t), idx_cmp);
    return M;
}

/* Same selection on fp32 values (used where a test feeds fp32 inputs). */
int tri_oracle_select_f32(int N, int B, const float *zmax, int32_t *kept_out)
{
    if (N < 0 || B < 1 || (N > 0 && (!zmax || !kept_out)))
        return -1;
    double *z = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
    if (!z) return -1;
    for (int i = 0; i < N; ++i) z[i] = (double)zmax[i];
    int m = tri_oracle_select(N, B, z, kept_out);
    free(z);
    return m;
}

/* Gather rows at the kept slots (bit copies) into slots 0..M-1. */
int tri_oracle_compact(int d, int M, const int32_t *kept,
                       const uint16_t *K, const uint16_t *V, const int32_t *pos,
                       uint16_t *K_out, uint16_t *V_out, int32_t *pos_out)
{
    if (d < 1 || M < 0)
        return -1;
    for (int j = 0; j < M; ++j) {
        const int32_t i = kept[j];
        memcpy(K_out + (size_t)j * d, K + (size_t)i * d, sizeof(uint16_t) * d);
        memcpy(V_out + (size_t)j * d, V + (size_t)i * d, sizeof(uint16_t) * d);
        pos_out[j] = pos[i];
    }
    return 0;
}

/*
 * The whole pass over a batch of units, units spread over threads.
 *   K [n_units][stride][d], pos [n_units][stride], lens [n_units] (<= stride),
 *   t [n_units], q_mean [n_units][G][d], q_norm / R [n_units][G][F].
 * Outputs (optional where marked): s [n_units][G][stride] per-head scores (NULL ok),
 * zmax [n_units][stride] (NULL ok), kept [n_units][B], n_kept [n_units].
 * Returns 0, or -1 on a bad argument.
 */
static int prune_batch(int combine, int n_units, int stride, int B, int d, int G, int layout, double base,
                       const int64_t *offsets, int n_off, const int64_t *t,
                       const float *q_mean, const float *q_norm, const float *R,
                       const uint16_t *K, const int32_t *pos, const int32_t *lens,
                       double *s_out, double *zmax_out, int32_t *kept_out, int32_t *n_kept_out,
                       int n_threads)
{
    if (n_units < 0 || stride < 0 || B < 1 || d < 2 || G < 1)
        return -1;
    const int F = d / 2;
    int bad = 0;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(|: bad)
#endif
    for (int u = 0; u < n_units; ++u) {
        const int N = lens[u];
        if (N < 0 || N > stride) { bad |= 1; continue; }
        double *s = (double *)malloc(sizeof(double) * (size_t)G * (N > 0 ? N : 1));
        double *zm = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
        if (!s || !zm) { free(s); free(zm); bad |= 1; continue; }
        int rc = unit_scores(combine, d, G, layout, base, offsets, n_off, t[u],
                             q_mean + (size_t)u * G * d, q_norm + (size_t)u * G * F,
                             R + (size_t)u * G * F, K + (size_t)u * stride * d,
                             pos + (size_t)u * stride, N, s, NULL, NULL);
        if (rc == 0) rc = tri_oracle_zmax(G, N, s, NULL, zm);
        if (rc == 0) {
            if (s_out)
                for (int h = 0; h < G; ++h)
                    memcpy(s_out + ((size_t)u * G + h) * stride, s + (size_t)h * N, sizeof(double) * N);
            if (zmax_out) memcpy(zmax_out + (size_t)u * stride, zm, sizeof(double) * N);
            int m = tri_oracle_select(N, B, zm, kept_out + (size_t)u * B);
            n_kept_out[u] = m;
            if (m < 0) rc = -1;
        }
        if (rc != 0) bad |= 1;
        free(s); free(zm);
    }
    return bad ? -1 : 0;
}

int tri_oracle_prune_batch(int n_units, int stride, int B, int d, int G, int layout, double base,
                           const int64_t *offsets, int n_off, const int64_t *t,
                           const float *q_mean, const float *q_norm, const float *R,
                           const uint16_t *K, const int32_t *pos, const int32_t *lens,
                           double *s_out, double *zmax_out, int32_t *kept_out, int32_t *n_kept_out,
                           int n_threads)
{
    return prune_batch(TRI_ORACLE_MEAN_OVER_DELTA, n_units, stride, B, d, G, layout, base, offsets, n_off, t,
                       q_mean, q_norm, R, K, pos, lens, s_out, zmax_out, kept_out, n_kept_out, n_threads);
}

/* The same selection with the offsets combined by the maximum (tri_oracle_unit_scores_max). */
int tri_oracle_prune_batch_max(int n_units, int stride, int B, int d, int G, int layout, double base,
                               const int64_t *offsets, int n_off, const int64_t *t,
                               const float *q_mean, const float *q_norm, const float *R,
                               const uint16_t *K, const int32_t *pos, const int32_t *lens,
                               double *s_out, double *zmax_out, int32_t *kept_out, int32_t *n_kept_out,
                               int n_threads)
{
    return prune_batch(TRI_ORACLE_MAX_OVER_DELTA, n_units, stride, B, d, G, layout, base, offsets, n_off, t,
                       q_mean, q_norm, R, K, pos, lens, s_out, zmax_out, kept_out, n_kept_out, n_threads);
}

/*
 * Calibration statistics from T pre-RoPE query samples.
 *   Q            [L][T][Hq][d] bf16 bits of the pre-RoPE queries, in the keys' dim layout
 *   q_mean       [L][Hq][d] out: E[q_f], its real part at band f's first dim and its
 *                imaginary part at the second (the same layout as the queries)
 *   q_norm_mean  [L][Hq][F] out: E|q_f|
 *   R            [L][Hq][F] out: |E[q_f]| / E|q_f|; 0 for a band whose samples are all 0
 *                (then E[q_f] = 0 and E|q_f| = 0 as well, so no score uses the value)
 * Every mean is a plain average over the T tokens. Returns 0, or -1 on bad arguments.
 */
int tri_oracle_calibrate(const uint16_t *Q, int L, int T, int Hq, int d, int layout,
                         double *q_mean, double *q_norm_mean, double *R)
{
    if (!Q || L < 1 || T < 1 || Hq < 1 || d < 2 || d % 2 || !q_mean || !q_norm_mean || !R) return -1;
    const int F = d / 2;
#pragma omp parallel for collapse(2) schedule(static)
    for (int l = 0; l < L; ++l) {
        for (int h = 0; h < Hq; ++h) {
            for (int f = 0; f < F; ++f) {
                int dr, di;
                band_dims(d, layout, f, &dr, &di);
                double sr = 0.0, si = 0.0, sm = 0.0;
                for (int t = 0; t < T; ++t) {
                    const uint16_t *q = Q + (((size_t)l * T + t) * Hq + h) * (size_t)d;
                    const double re = bf16_value(q[dr]);
                    const double im = bf16_value(q[di]);
                    sr += re;
                    si += im;
                    sm += sqrt(re * re + im * im);
                }
                const double mr = sr / (double)T, mi = si / (double)T, mm = sm / (double)T;
                double *qm = q_mean + ((size_t)l * Hq + h) * (size_t)d;
                qm[dr] = mr;
                qm[di] = mi;
                q_norm_mean[((size_t)l * Hq + h) * F + f] = mm;
                R[((size_t)l * Hq + h) * F + f] = mm > 0.0 ? sqrt(mr * mr + mi * mi) / mm : 0.0;
            }
        }
    }
    return 0;
}

/*
 * Decode attention over one pruned unit: the consumer of the compacted cache. For every
 * query head h of the group, the standard scaled dot-product attention that the
 * "TriAttention 深度解析：MIT韩松团队如何用三角函数让单卡4090跑出百万Token上下文" page writes out
 * in its section 二 (logits q.k / sqrt(d), softmax over the cached keys, weights applied to
 * the values), evaluated on the M rows that the prune kept. The query is post-RoPE (rotated
 * at its own position t) like the stored keys, so each logit already depends on t - p only
 * and the kept keys' scattered positions need no other treatment.
 *   q     [G][d] bf16 bits of the post-RoPE queries of the group
 *   K, V  [M][d] bf16 bits of the kept (post-RoPE) keys and their values
 *   out   [G][d] fp64 attention outputs
 * The largest logit is subtracted before the exponentials (the same softmax, written so that
 * no exponential overflows). Returns 0, or -1 on bad arguments (M < 1 has no softmax).
 */
int tri_oracle_decode_attention(int d, int G, int M, const uint16_t *q, const uint16_t *K, const uint16_t *V,
                                double *out)
{
    if (d < 1 || G < 1 || M < 1 || !q || !K || !V || !out) return -1;
    const double scale = 1.0 / sqrt((double)d);
    double *logit = (double *)malloc(sizeof(double) * (size_t)M);
    if (!logit) return -1;
    for (int h = 0; h < G; ++h) {
        double top = -INFINITY;
        for (int j = 0; j < M; ++j) {
            double dot = 0.0;
            for (int i = 0; i < d; ++i)
                dot += bf16_value(q[(size_t)h * d + i]) * bf16_value(K[(size_t)j * d + i]);
            logit[j] = dot * scale;
            if (logit[j] > top) top = logit[j];
        }
        double denom = 0.0;
        for (int j = 0; j < M; ++j) {
            logit[j] = exp(logit[j] - top);
            denom += logit[j];
        }
        for (int i = 0; i < d; ++i) {
            double acc = 0.0;
            for (int j = 0; j < M; ++j) acc += logit[j] * bf16_value(V[(size_t)j * d + i]);
            out[(size_t)h * d + i] = acc / denom;
        }
    }
    free(logit);
    return 0;
}
