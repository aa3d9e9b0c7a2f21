/*
 * Double-precision CPU oracle for grouped-query scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  It shares no code, header or constant with the
 * CUDA library; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark call it.
 *
 * What it computes is the plain definition, written out with no blocking,
 * fusion or reordering:
 *   - query head hq reads KV head hq / (Hq / Hkv): contiguous groups
 *     (TT Lab "キー・バリューヘッドだけ減らしてみる", step 1: group = head // (h // g));
 *   - score s_j = scale * sum_c q_c k_jc, scale = 1/sqrt(d) by default
 *     (same lab, step 4; course "Неделя 7. Внимание", step 1, A = QK^T/sqrt(H));
 *   - with the causal mask, s_j = -inf for j > i + (Tkv - Tq) before the
 *     softmax (course step 1: the mask goes in before the softmax);
 *   - softmax with the row max subtracted, then the weighted mean of V
 *     (lab step 4).
 * lse = m + ln(sum_j exp(s_j - m)) is reported beside each row; a row with no
 * visible key gives o = 0 and lse = -inf.
 *
 * Inputs are float32 arrays holding the exact values the GPU sees (bf16 and
 * fp32 both widen to float32 exactly); all arithmetic is in double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Contiguous grouping: h heads in g groups, head -> head / (h / g). */
static long kv_head_of(long hq, long Hq, long Hkv) { return hq / (Hq / Hkv); }

/*
 * One query row against n_keys keys.  Key j is visible when j < n_vis (the
 * causal limit) and, with a sliding window, when j >= lo or j < sinks (the
 * window's first key and the always-visible sink keys); hidden keys get score
 * -inf before the softmax.  lo = 0, sinks = 0 means no window.
 */
static void attend_row_win(const float *qrow, const float *k0, const float *v0,
                           long key_stride, long n_keys, long n_vis, long lo, long sinks,
                           long d, double scale, double *s, double *orow, double *lse)
{
    double m = -INFINITY;
    for (long j = 0; j < n_keys; ++j) {
        if (j >= n_vis || (j < lo && j >= sinks)) { s[j] = -INFINITY; continue; }
        const float *kj = k0 + j * key_stride;
        double dot = 0.0;
        for (long c = 0; c < d; ++c) dot += (double)qrow[c] * (double)kj[c];
        s[j] = scale * dot;
        if (s[j] > m) m = s[j];
    }
    for (long c = 0; c < d; ++c) orow[c] = 0.0;
    if (m == -INFINITY) { *lse = -INFINITY; return; }   /* no visible key */
    double l = 0.0;
    for (long j = 0; j < n_keys; ++j) {
        if (s[j] == -INFINITY) continue;                   /* exp(-inf) = 0 */
        double p = exp(s[j] - m);
        l += p;
        const float *vj = v0 + j * key_stride;
        for (long c = 0; c < d; ++c) orow[c] += p * (double)vj[c];
    }
    for (long c = 0; c < d; ++c) orow[c] /= l;
    *lse = m + log(l);
}

static void attend_row(const float *qrow, const float *k0, const float *v0,
                       long key_stride, long n_keys, long n_vis, long d,
                       double scale, double *s, double *orow, double *lse)
{
    attend_row_win(qrow, k0, v0, key_stride, n_keys, n_vis, 0, 0, d, scale, s, orow, lse);
}

static int check_shape(long B, long Tq, long Tkv, long Hq, long Hkv, long d)
{
    if (B < 0 || Tq < 0 || Tkv < 0 || Hq <= 0 || Hkv <= 0 || d <= 0) return 1;
    if (Hq % Hkv != 0) return 1;                  /* the lab's ValueError */
    return 0;
}

static void set_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Number of keys query row i may see. */
static long visible_keys(long i, long Tq, long Tkv, int causal)
{
    if (!causal) return Tkv;
    long n = i + (Tkv - Tq) + 1;          /* keys j <= i + Tkv - Tq */
    if (n < 0) n = 0;
    if (n > Tkv) n = Tkv;
    return n;
}

/*
 * Full forward.  q:[B,Tq,Hq,d]  k,v:[B,Tkv,Hkv,d]  o:[B,Tq,Hq,d]  lse:[B,Hq,Tq]
 * (lse may be NULL).  Returns 0, or 1 for an invalid shape.
 */
int oracle_attn_fwd(const float *q, const float *k, const float *v,
                    double *o, double *lse,
                    long B, long Tq, long Tkv, long Hq, long Hkv, long d,
                    int causal, double scale, int nthreads)
{
    if (check_shape(B, Tq, Tkv, Hq, Hkv, d)) return 1;
    set_threads(nthreads);
    long n_rows = B * Hq * Tq;
    #pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Tkv > 0 ? Tkv : 1));
        #pragma omp for schedule(dynamic, 8)
        for (long r = 0; r < n_rows; ++r) {
            long i = r % Tq, bh = r / Tq, hq = bh % Hq, b = bh / Hq;
            long kvh = kv_head_of(hq, Hq, Hkv);
            const float *qrow = q + ((b * Tq + i) * Hq + hq) * d;
            const float *k0 = k + (b * Tkv * Hkv + kvh) * d;
            const float *v0 = v + (b * Tkv * Hkv + kvh) * d;
            double l_row;
            attend_row(qrow, k0, v0, Hkv * d, Tkv, visible_keys(i, Tq, Tkv, causal),
                       d, scale, s, o + ((b * Tq + i) * Hq + hq) * d, &l_row);
            if (lse) lse[(b * Hq + hq) * Tq + i] = l_row;
        }
        free(s);
    }
    return 0;
}

/*
 * Selected rows only.  rows[r] = (b * Hq + hq) * Tq + i; o:[n_rows,d],
 * lse:[n_rows] (may be NULL).  Same arithmetic as oracle_attn_fwd.
 */
int oracle_attn_fwd_rows(const float *q, const float *k, const float *v,
                         const int64_t *rows, long n_rows, double *o, double *lse,
                         long B, long Tq, long Tkv, long Hq, long Hkv, long d,
                         int causal, double scale, int nthreads)
{
    if (check_shape(B, Tq, Tkv, Hq, Hkv, d)) return 1;
    for (long r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= B * Hq * Tq) return 1;
    set_threads(nthreads);
    #pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Tkv > 0 ? Tkv : 1));
        #pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < n_rows; ++r) {
            long idx = (long)rows[r];
            long i = idx % Tq, bh = idx / Tq, hq = bh % Hq, b = bh / Hq;
            long kvh = kv_head_of(hq, Hq, Hkv);
            double l_row;
            attend_row(q + ((b * Tq + i) * Hq + hq) * d,
                       k + (b * Tkv * Hkv + kvh) * d, v + (b * Tkv * Hkv + kvh) * d,
                       Hkv * d, Tkv, visible_keys(i, Tq, Tkv, causal), d, scale, s,
                       o + r * d, &l_row);
            if (lse) lse[r] = l_row;
        }
        free(s);
    }
    return 0;
}

/*
 * Decode: one query token per sequence against the first seqlens[b] rows of
 * a KV cache (the causal mask leaves every cached key visible to the newest
 * token).  q:[B,Hq,d]  k_cache,v_cache:[B,Lmax,Hkv,d]  o:[B,Hq,d]  lse:[B,Hq].
 */
int oracle_decode(const float *q, const float *kc, const float *vc,
                  const int32_t *seqlens, double *o, double *lse,
                  long B, long Hq, long Hkv, long d, long Lmax,
                  double scale, int nthreads)
{
    if (check_shape(B, 1, Lmax, Hq, Hkv, d)) return 1;
    for (long b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > Lmax) return 1;
    set_threads(nthreads);
    #pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Lmax > 0 ? Lmax : 1));
        #pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < B * Hq; ++r) {
            long hq = r % Hq, b = r / Hq, kvh = kv_head_of(hq, Hq, Hkv);
            long L = seqlens[b];
            double l_row;
            attend_row(q + r * d, kc + (b * Lmax * Hkv + kvh) * d,
                       vc + (b * Lmax * Hkv + kvh) * d, Hkv * d, L, L, d, scale, s,
                       o + r * d, &l_row);
            if (lse) lse[r] = l_row;
        }
        free(s);
    }
    return 0;
}

/*
 * Decode computed split by split and merged with the log-sum-exp identity:
 * split s covers keys [s*chunk, min((s+1)*chunk, L)); its partial output O_s
 * and lse_s are merged as O = sum_s e^(lse_s - M) O_s / sum_s e^(lse_s - M),
 * M = max_s lse_s.  This is the same number as oracle_decode in exact
 * arithmetic, which is what pins the merge.
 */
int oracle_decode_split(const float *q, const float *kc, const float *vc,
                        const int32_t *seqlens, double *o, double *lse,
                        long B, long Hq, long Hkv, long d, long Lmax,
                        double scale, long chunk, int nthreads)
{
    if (check_shape(B, 1, Lmax, Hq, Hkv, d) || chunk <= 0) return 1;
    for (long b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > Lmax) return 1;
    set_threads(nthreads);
    #pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)chunk);
        double *part = (double *)malloc(sizeof(double) * (size_t)d);
        #pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < B * Hq; ++r) {
            long hq = r % Hq, b = r / Hq, kvh = kv_head_of(hq, Hq, Hkv);
            long L = seqlens[b];
            long n_split = (L + chunk - 1) / chunk;
            double *orow = o + r * d;
            for (long c = 0; c < d; ++c) orow[c] = 0.0;
            if (n_split == 0) { if (lse) lse[r] = -INFINITY; continue; }
            /* first pass: the largest split lse */
            double M = -INFINITY;
            for (long sp = 0; sp < n_split; ++sp) {
                long j0 = sp * chunk, n = (L - j0 < chunk) ? L - j0 : chunk;
                double l_sp;
                attend_row(q + r * d, kc + ((b * Lmax + j0) * Hkv + kvh) * d,
                           vc + ((b * Lmax + j0) * Hkv + kvh) * d, Hkv * d, n, n, d,
                           scale, s, part, &l_sp);
                if (l_sp > M) M = l_sp;
            }
            /* second pass: weighted sum of the split outputs */
            double wsum = 0.0;
            for (long sp = 0; sp < n_split; ++sp) {
                long j0 = sp * chunk, n = (L - j0 < chunk) ? L - j0 : chunk;
                double l_sp;
                attend_row(q + r * d, kc + ((b * Lmax + j0) * Hkv + kvh) * d,
                           vc + ((b * Lmax + j0) * Hkv + kvh) * d, Hkv * d, n, n, d,
                           scale, s, part, &l_sp);
                double w = exp(l_sp - M);
                wsum += w;
                for (long c = 0; c < d; ++c) orow[c] += w * part[c];
            }
            for (long c = 0; c < d; ++c) orow[c] /= wsum;
            if (lse) lse[r] = M + log(wsum);
        }
        free(part);
        free(s);
    }
    return 0;
}

/*
 * Causal forward with a sliding window of `window` keys (window >= 1) and
 * `sinks` always-visible leading keys: row i (key position p = i + Tkv - Tq)
 * sees key j iff j <= p and (j > p - window or j < sinks).  Course "Неделя 7.
 * Внимание", step 3 ("Sliding window, attention sinks").  Layouts as
 * oracle_attn_fwd.
 */
int oracle_attn_fwd_window(const float *q, const float *k, const float *v,
                           double *o, double *lse,
                           long B, long Tq, long Tkv, long Hq, long Hkv, long d,
                           long window, long sinks, double scale, int nthreads)
{
    if (check_shape(B, Tq, Tkv, Hq, Hkv, d) || window < 1 || sinks < 0) return 1;
    set_threads(nthreads);
    long n_rows = B * Hq * Tq;
    #pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Tkv > 0 ? Tkv : 1));
        #pragma omp for schedule(dynamic, 8)
        for (long r = 0; r < n_rows; ++r) {
            long i = r % Tq, bh = r / Tq, hq = bh % Hq, b = bh / Hq;
            long kvh = kv_head_of(hq, Hq, Hkv);
            long p = i + (Tkv - Tq);
            double l_row;
            attend_row_win(q + ((b * Tq + i) * Hq + hq) * d,
                           k + (b * Tkv * Hkv + kvh) * d, v + (b * Tkv * Hkv + kvh) * d,
                           Hkv * d, Tkv, visible_keys(i, Tq, Tkv, 1), p - window + 1, sinks,
                           d, scale, s, o + ((b * Tq + i) * Hq + hq) * d, &l_row);
            if (lse) lse[(b * Hq + hq) * Tq + i] = l_row;
        }
        free(s);
    }
    return 0;
}

/*
 * Decode with a sliding window: the newest token of sequence b (position
 * L - 1, L = seqlens[b]) sees cache rows j >= L - window plus rows j < sinks.
 */
int oracle_decode_window(const float *q, const float *kc, const float *vc,
                         const int32_t *seqlens, double *o, double *lse,
                         long B, long Hq, long Hkv, long d, long Lmax,
                         long window, long sinks, double scale, int nthreads)
{
    if (check_shape(B, 1, Lmax, Hq, Hkv, d) || window < 1 || sinks < 0) return 1;
    for (long b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > Lmax) return 1;
    set_threads(nthreads);
    #pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Lmax > 0 ? Lmax : 1));
        #pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < B * Hq; ++r) {
            long hq = r % Hq, b = r / Hq, kvh = kv_head_of(hq, Hq, Hkv);
            long L = seqlens[b];
            double l_row;
            attend_row_win(q + r * d, kc + (b * Lmax * Hkv + kvh) * d,
                           vc + (b * Lmax * Hkv + kvh) * d, Hkv * d, L, L, L - window, sinks,
                           d, scale, s, o + r * d, &l_row);
            if (lse) lse[r] = l_row;
        }
        free(s);
    }
    return 0;
}
