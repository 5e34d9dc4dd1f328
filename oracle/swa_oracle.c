/*
 * Plain fp64 CPU oracle for causal sliding-window softmax attention with
 * attention sinks.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and
 * the benchmark's CPU-baseline / reference legs call it; the CUDA library
 * never does, and the two share no code.
 *
 * What it computes (the definition, written out, with no blocking, no
 * fusion and no online rescaling):
 *
 *   Visible set.  "Sliding-window beats linear attention", section 1 (Key
 *   Terms): a query attends only to a fixed-size window of preceding tokens,
 *   and the first few tokens of the sequence (attention sinks) must stay
 *   visible; section 3 keeps 4 sinks.  With window w (the query's own
 *   position included) and n_sink = s, the keys visible from position t are
 *       S(t) = { j : j <= t  and  ( j >= t - w + 1  or  j < s ) }.
 *   A key that is both in the window and a sink is counted once.  Positions
 *   are relative to the start of the sequence.
 *
 *   Grouped-query heads ("Rethinking Attention Output Projection", section 1
 *   names MQA/GQA): G = Hq / Hkv consecutive query heads share one KV head,
 *   kvh = hq / G.
 *
 *   Softmax attention for one query row t and query head h:
 *       z_j  = scale * sum_c q[t,h,c] * k[j,kvh,c]       for j in S(t)
 *       m    = max_j z_j
 *       l    = sum_j exp(z_j - m)
 *       out  = sum_j exp(z_j - m) * v[j,kvh,:] / l
 *       lse  = m + ln(l)                                  (natural log)
 *   computed as an exact two-pass softmax in double precision.
 *
 * Every function here is parity-pinned by the pytest cases marked "not gpu"
 * (closed forms, a library causal-attention routine, brute-force masks and
 * hand-derived golden values); none of those cases retypes this code.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Lower end of the window: the first position j >= t - w + 1 (clamped at 0). */
static int64_t window_lo(int64_t t, int64_t w) {
    int64_t lo = t - w + 1;
    return lo < 0 ? 0 : lo;
}

/*
 * The visible set of row t as two disjoint ranges, [0, sink_end) and [lo, t]:
 * j < s and j < lo are the sinks left of the window, lo..t is the window.
 * This is S(t) rewritten; the tests compare it with the literal predicate.
 */
static void visible_ranges(int64_t t, int64_t w, int64_t s, int64_t* sink_end, int64_t* lo) {
    *lo = window_lo(t, w);
    int64_t se = s < *lo ? s : *lo;
    *sink_end = se < 0 ? 0 : se;
}

int64_t oracle_visible_count(int64_t t, int64_t w, int64_t s) {
    int64_t se, lo;
    visible_ranges(t, w, s, &se, &lo);
    return se + (t - lo + 1);
}

static int set_threads(int n_threads) {
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
    return omp_get_max_threads();
#else
    (void)n_threads;
    return 1;
#endif
}

/*
 * One sequence, a list of query rows.
 *   q     [n_rows][Hq][d]     query vectors of the rows
 *   t_row [n_rows]            position of each row in the sequence (0 <= t < L)
 *   k, v  [L][Hkv][d]         keys and values of the sequence (positions 0..L-1)
 *   out   [n_rows][Hq][d]
 *   lse   [n_rows][Hq]        (may be NULL)
 * Returns 0, or -1 on bad arguments.
 */
int oracle_swa_rows(const double* q, const int64_t* t_row, int64_t n_rows,
                    const double* k, const double* v, int64_t L,
                    int Hq, int Hkv, int d, int64_t window, int64_t n_sink, double scale,
                    double* out, double* lse, int n_threads) {
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || window < 1 || n_sink < 0 || n_rows < 0)
        return -1;
    for (int64_t r = 0; r < n_rows; ++r)
        if (t_row[r] < 0 || t_row[r] >= L) return -1;
    const int G = Hq / Hkv;
    const int64_t zmax = (window < L ? window : L) + n_sink + 1;
    set_threads(n_threads);
    int bad = 0;
#pragma omp parallel
    {
        double* z = (double*)malloc(sizeof(double) * (size_t)zmax);
        int64_t* key = (int64_t*)malloc(sizeof(int64_t) * (size_t)zmax);
        double* acc = (double*)malloc(sizeof(double) * (size_t)d);
        if (!z || !key || !acc) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t rh = 0; rh < n_rows * Hq; ++rh) {
                const int64_t r = rh / Hq;
                const int h = (int)(rh % Hq);
                const int kvh = h / G;
                const int64_t t = t_row[r];
                const double* qv = q + ((size_t)r * Hq + h) * d;
                int64_t se, lo;
                visible_ranges(t, window, n_sink, &se, &lo);
                int64_t n = 0;
                for (int64_t j = 0; j < se; ++j) key[n++] = j;
                for (int64_t j = lo; j <= t; ++j) key[n++] = j;
                /* pass 1: scores and their maximum */
                double m = -INFINITY;
                for (int64_t i = 0; i < n; ++i) {
                    const double* kj = k + ((size_t)key[i] * Hkv + kvh) * d;
                    double dot = 0.0;
                    for (int c = 0; c < d; ++c) dot += qv[c] * kj[c];
                    z[i] = scale * dot;
                    if (z[i] > m) m = z[i];
                }
                /* pass 2: normaliser and weighted sum of values */
                double l = 0.0;
                for (int c = 0; c < d; ++c) acc[c] = 0.0;
                for (int64_t i = 0; i < n; ++i) {
                    const double p = exp(z[i] - m);
                    l += p;
                    const double* vj = v + ((size_t)key[i] * Hkv + kvh) * d;
                    for (int c = 0; c < d; ++c) acc[c] += p * vj[c];
                }
                double* o = out + ((size_t)r * Hq + h) * d;
                for (int c = 0; c < d; ++c) o[c] = acc[c] / l;
                if (lse) lse[(size_t)r * Hq + h] = m + log(l);
            }
        }
        free(z);
        free(key);
        free(acc);
    }
    return bad ? -1 : 0;
}

/*
 * Explicit attention weights of one (row t, query head h): w[j] for j = 0..L-1,
 * zero for keys outside S(t).  Same arithmetic as oracle_swa_rows.
 */
int oracle_swa_weights(const double* qrow /* [Hq][d] */, int64_t t, const double* k, int64_t L,
                       int Hq, int Hkv, int d, int h, int64_t window, int64_t n_sink,
                       double scale, double* wout /* [L] */) {
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || h < 0 || h >= Hq || t < 0 || t >= L || window < 1)
        return -1;
    const int kvh = h / (Hq / Hkv);
    const double* qv = qrow + (size_t)h * d;
    int64_t se, lo;
    visible_ranges(t, window, n_sink, &se, &lo);
    for (int64_t j = 0; j < L; ++j) wout[j] = 0.0;
    double m = -INFINITY;
    for (int pass = 0; pass < 2; ++pass) {
        for (int64_t j = 0; j <= t; ++j) {
            if (!(j < se || j >= lo)) continue;
            const double* kj = k + ((size_t)j * Hkv + kvh) * d;
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += qv[c] * kj[c];
            const double zj = scale * dot;
            if (pass == 0) { if (zj > m) m = zj; }
            else wout[j] = exp(zj - m);
        }
    }
    double l = 0.0;
    for (int64_t j = 0; j < L; ++j) l += wout[j];
    for (int64_t j = 0; j < L; ++j) wout[j] /= l;
    return 0;
}

/*
 * Whole prefill of a batch of equal-length sequences.
 *   q [B][L][Hq][d], k/v [B][L][Hkv][d], out [B][L][Hq][d], lse [B][Hq][L] (may be NULL).
 */
int oracle_swa_fwd(const double* q, const double* k, const double* v, double* out, double* lse,
                   int B, int Hq, int Hkv, int64_t L, int d, int64_t window, int64_t n_sink,
                   double scale, int n_threads) {
    if (B < 0 || L < 0) return -1;
    int64_t* t_row = (int64_t*)malloc(sizeof(int64_t) * (size_t)(L > 0 ? L : 1));
    double* lrow = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * (size_t)Hq);
    if (!t_row || !lrow) { free(t_row); free(lrow); return -1; }
    for (int64_t t = 0; t < L; ++t) t_row[t] = t;
    int rc = 0;
    for (int b = 0; b < B && rc == 0; ++b) {
        const size_t qo = (size_t)b * L * Hq * d, ko = (size_t)b * L * Hkv * d;
        rc = oracle_swa_rows(q + qo, t_row, L, k + ko, v + ko, L, Hq, Hkv, d, window, n_sink,
                             scale, out + qo, lrow, n_threads);
        if (lse && rc == 0)
            for (int64_t t = 0; t < L; ++t)
                for (int h = 0; h < Hq; ++h)
                    lse[((size_t)b * Hq + h) * L + t] = lrow[(size_t)t * Hq + h];
    }
    free(t_row);
    free(lrow);
    return rc;
}

/*
 * Packed variable-length prefill: sequence i owns tokens cu[i]..cu[i+1]-1 and its
 * window and sinks are relative to its own start.
 *   q [T][Hq][d], k/v [T][Hkv][d], out [T][Hq][d], lse [Hq][T] (may be NULL).
 */
int oracle_swa_fwd_varlen(const double* q, const double* k, const double* v, double* out,
                          double* lse, const int64_t* cu, int n_seq, int Hq, int Hkv, int d,
                          int64_t window, int64_t n_sink, double scale, int n_threads) {
    if (n_seq < 0) return -1;
    const int64_t T = cu[n_seq];
    int rc = 0;
    for (int i = 0; i < n_seq && rc == 0; ++i) {
        const int64_t a = cu[i], L = cu[i + 1] - cu[i];
        if (L < 0) return -1;
        if (L == 0) continue;
        int64_t* t_row = (int64_t*)malloc(sizeof(int64_t) * (size_t)L);
        double* lrow = (double*)malloc(sizeof(double) * (size_t)L * (size_t)Hq);
        if (!t_row || !lrow) { free(t_row); free(lrow); return -1; }
        for (int64_t t = 0; t < L; ++t) t_row[t] = t;
        rc = oracle_swa_rows(q + (size_t)a * Hq * d, t_row, L, k + (size_t)a * Hkv * d,
                             v + (size_t)a * Hkv * d, L, Hq, Hkv, d, window, n_sink, scale,
                             out + (size_t)a * Hq * d, lrow, n_threads);
        if (lse && rc == 0)
            for (int64_t t = 0; t < L; ++t)
                for (int h = 0; h < Hq; ++h)
                    lse[(size_t)h * T + a + t] = lrow[(size_t)t * Hq + h];
        free(t_row);
        free(lrow);
    }
    return rc;
}

int oracle_num_threads(int n_threads) { return set_threads(n_threads); }
