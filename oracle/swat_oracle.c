/*
 * swat_oracle.c — plain, slow, fp64 CPU oracle for SWAT sliding-window attention.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product library links, includes or
 * calls this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark load it. It shares no header, helper or table with the CUDA
 * sources.
 *
 * What it computes (sources are cited per function):
 *   - the key set of a query (causal sliding window plus attention sinks),
 *   - RoPE rotation (RoFormer convention, adjacent pairs),
 *   - the SWAT forward: sigmoid of (rotated q . rotated k)/sqrt(d) plus a
 *     per-head ALiBi term slope*(m-n), summed against v, no normalisation,
 *   - the softmax-with-sinks SWA(w, s) forward, with the log-sum-exp per row,
 *   - the analytic backward of both (derived by calculus from the forward),
 *   - the ring-buffer KV cache and one decode step over it.
 *
 * Inputs arrive as float (every bf16 value is exact in float) and are upcast
 * to double element by element; all arithmetic is double. There is no tiling,
 * fusion or reordering: each output is the literal sum over its key set.
 *
 * Layout: q [B,N,H,d], k and v [B,N,Hkv,d], o [B,N,H,d], lse [B,H,N], all
 * row-major ("BSHD"). Query head h reads KV head h / (H/Hkv).
 *
 * Parity status: the RoPE pairing/frequency convention and the slope
 * magnitudes for H != 16 are not printed on the pages; they follow the
 * RoFormer paper and the stated geometric rule, and are "parity unpinned"
 * beyond that convention. Everything else is pinned by tests/test_oracle_*.py.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#include <stdint.h>

#define MODE_SIGMOID 0
#define MODE_SOFTMAX 1

/* ------------------------------------------------------------------------ */
/* Key set.
 * "Sliding Window Attention" glossary (Ultralytics), section "How the window
 * grows with depth": with offset = i - j, a query attends iff
 * 0 <= offset < window (itself plus window-1 predecessors).
 * "SWAT: Sliding Window Attention Training", Symbol Map: m - n < omega, and
 * the attention equation sums n from m-omega+1 to m.
 * "Sliding-window beats linear attention", key idea / technical approach:
 * SWA(w, s) keeps the first s (sink) tokens besides the recent w tokens.
 * A sink already inside the window is counted once (union of the two sets).
 */
int oracle_in_keyset(long long i, long long j, long long window, long long n_sink)
{
    if (j < 0 || j > i) return 0;
    if (i - j < window) return 1;
    if (j < n_sink) return 1;
    return 0;
}

/* Number of keys of query i in a sequence (used by closed-form pins). */
long long oracle_keyset_size(long long i, long long window, long long n_sink)
{
    long long c = 0;
    for (long long j = 0; j <= i; ++j) c += oracle_in_keyset(i, j, window, n_sink);
    return c;
}

/* ------------------------------------------------------------------------ */
/* RoPE. "SWAT" page, section "RoPE: Stabilizing Sigmoid Attention Training"
 * and the Symbol Map entry R^d_{Theta,m}; the convention is the cited RoFormer
 * paper: pair (2t, 2t+1) is rotated by the angle m * theta_t with
 * theta_t = base^(-2t/d). A base <= 0 means "no rotation". */
void oracle_rope_rotate(double *x, int d, long long pos, double rope_base)
{
    if (!(rope_base > 0.0)) return;
    for (int t = 0; t < d / 2; ++t) {
        double theta = pow(rope_base, -2.0 * (double)t / (double)d);
        double a = (double)pos * theta;
        double c = cos(a), s = sin(a);
        double x0 = x[2 * t], x1 = x[2 * t + 1];
        x[2 * t]     = x0 * c - x1 * s;
        x[2 * t + 1] = x0 * s + x1 * c;
    }
}

/* Transposed rotation R^T (used to map gradients back from rotated space). */
void oracle_rope_rotate_inv(double *x, int d, long long pos, double rope_base)
{
    if (!(rope_base > 0.0)) return;
    for (int t = 0; t < d / 2; ++t) {
        double theta = pow(rope_base, -2.0 * (double)t / (double)d);
        double a = (double)pos * theta;
        double c = cos(a), s = sin(a);
        double x0 = x[2 * t], x1 = x[2 * t + 1];
        x[2 * t]     =  x0 * c + x1 * s;
        x[2 * t + 1] = -x0 * s + x1 * c;
    }
}

/* Table of cos/sin(pos * theta_t) for pos in [0, n_pos), t in [0, d/2):
 * the same numbers oracle_rope_rotate computes, cached so that a key's
 * rotation is not recomputed with trigonometry for every query. */
typedef struct { double *c, *s; int half; long long n_pos; int on; } rope_table;

static rope_table rope_table_make(long long n_pos, int d, double rope_base)
{
    rope_table tb;
    tb.half = d / 2; tb.n_pos = n_pos; tb.on = rope_base > 0.0;
    tb.c = NULL; tb.s = NULL;
    if (!tb.on) return tb;
    tb.c = (double *)malloc(sizeof(double) * (size_t)n_pos * tb.half);
    tb.s = (double *)malloc(sizeof(double) * (size_t)n_pos * tb.half);
    for (long long p = 0; p < n_pos; ++p)
        for (int t = 0; t < tb.half; ++t) {
            double theta = pow(rope_base, -2.0 * (double)t / (double)d);
            double a = (double)p * theta;
            tb.c[p * tb.half + t] = cos(a);
            tb.s[p * tb.half + t] = sin(a);
        }
    return tb;
}

static void rope_table_free(rope_table *tb) { free(tb->c); free(tb->s); }

/* out = R_pos * in (float input upcast to double). */
static void rope_apply(const rope_table *tb, const float *in, double *out, int d, long long pos)
{
    for (int c = 0; c < d; ++c) out[c] = (double)in[c];
    if (!tb->on) return;
    for (int t = 0; t < d / 2; ++t) {
        double c = tb->c[pos * tb->half + t], s = tb->s[pos * tb->half + t];
        double x0 = out[2 * t], x1 = out[2 * t + 1];
        out[2 * t]     = x0 * c - x1 * s;
        out[2 * t + 1] = x0 * s + x1 * c;
    }
}

/* out = R_pos^T * in (double). */
static void rope_apply_inv(const rope_table *tb, const double *in, double *out, int d, long long pos)
{
    for (int c = 0; c < d; ++c) out[c] = in[c];
    if (!tb->on) return;
    for (int t = 0; t < d / 2; ++t) {
        double c = tb->c[pos * tb->half + t], s = tb->s[pos * tb->half + t];
        double x0 = out[2 * t], x1 = out[2 * t + 1];
        out[2 * t]     =  x0 * c + x1 * s;
        out[2 * t + 1] = -x0 * s + x1 * c;
    }
}

/* ------------------------------------------------------------------------ */
/* Activation. "SWAT" page, section "Sigmoid: Dense Attention Without
 * Suppression": sigma(x) = 1/(1+e^-x), element-wise, no row normalisation. */
double oracle_sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

static size_t idx_q(int b, long long i, int h, int N, int H, int d)
{ return (((size_t)b * N + (size_t)i) * H + h) * (size_t)d; }

/* Score list of one query row: keys[] and s[] (length returned).
 * Score per the attention equation of the "SWAT" page, section "Balanced
 * ALiBi": (R_m q_m)^T (R_n k_n) / sqrt(d_k) + s_h * (m - n). */
static long long row_scores(const float *q, const float *k, const rope_table *tb,
                            int b, int h, long long i, int H, int Hkv, int N, int d,
                            int window, int n_sink, double slope,
                            long long *keys, double *s, double *qr, double *kr)
{
    int G = H / Hkv, kvh = h / G;
    double scale = 1.0 / sqrt((double)d);
    rope_apply(tb, q + idx_q(b, i, h, N, H, d), qr, d, i);
    long long n = 0;
    for (long long j = 0; j <= i; ++j) {
        if (!oracle_in_keyset(i, j, window, n_sink)) continue;
        rope_apply(tb, k + idx_q(b, j, kvh, N, Hkv, d), kr, d, j);
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += qr[c] * kr[c];
        keys[n] = j;
        s[n] = dot * scale + slope * (double)(i - j);
        ++n;
    }
    return n;
}

/* Turns scores into weights p (sigmoid or softmax); returns lse (softmax) or 0.
 * Softmax: "SWAT" page, section "Why This Exists" (exponential
 * sparsification example) and the SWA(w, s) page (softmax attention with sinks). */
static double row_weights(const double *s, double *p, long long n, int mode)
{
    if (mode == MODE_SIGMOID) {
        for (long long a = 0; a < n; ++a) p[a] = oracle_sigmoid(s[a]);
        return 0.0;
    }
    double m = -INFINITY;
    for (long long a = 0; a < n; ++a) if (s[a] > m) m = s[a];
    double l = 0.0;
    for (long long a = 0; a < n; ++a) { p[a] = exp(s[a] - m); l += p[a]; }
    for (long long a = 0; a < n; ++a) p[a] /= l;
    return m + log(l);
}

/* ------------------------------------------------------------------------ */
/* Forward for an explicit list of rows: rows[3*r + {0,1,2}] = (b, h, i).
 * o_rows [n_rows, d]; lse_rows [n_rows] (softmax mode, may be NULL). */
void oracle_swat_fwd_rows(const float *q, const float *k, const float *v,
                          int B, int H, int Hkv, int N, int d, int window, int n_sink,
                          int mode, const float *slopes, double rope_base,
                          long long n_rows, const long long *rows,
                          double *o_rows, double *lse_rows)
{
    (void)B;
    rope_table tb = rope_table_make(N, d, rope_base);
    int G = H / Hkv;
    #pragma omp parallel
    {
        long long *keys = (long long *)malloc(sizeof(long long) * (size_t)N);
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        double *p = (double *)malloc(sizeof(double) * (size_t)N);
        double *qr = (double *)malloc(sizeof(double) * (size_t)d);
        double *kr = (double *)malloc(sizeof(double) * (size_t)d);
        #pragma omp for schedule(dynamic, 4)
        for (long long r = 0; r < n_rows; ++r) {
            int b = (int)rows[3 * r], h = (int)rows[3 * r + 1];
            long long i = rows[3 * r + 2];
            double slope = slopes ? (double)slopes[h] : 0.0;
            long long n = row_scores(q, k, &tb, b, h, i, H, Hkv, N, d, window, n_sink,
                                     slope, keys, s, qr, kr);
            double lse = row_weights(s, p, n, mode);
            double *o = o_rows + (size_t)r * d;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            for (long long a = 0; a < n; ++a) {
                const float *vj = v + idx_q(b, keys[a], h / G, N, Hkv, d);
                for (int c = 0; c < d; ++c) o[c] += p[a] * (double)vj[c];
            }
            if (lse_rows) lse_rows[r] = (mode == MODE_SOFTMAX) ? lse : 0.0;
        }
        free(keys); free(s); free(p); free(qr); free(kr);
    }
    rope_table_free(&tb);
}

/* Full forward: o [B,N,H,d]; lse [B,H,N] (may be NULL). */
void oracle_swat_fwd(const float *q, const float *k, const float *v, double *o, double *lse,
                     int B, int H, int Hkv, int N, int d, int window, int n_sink, int mode,
                     const float *slopes, double rope_base)
{
    long long n_rows = (long long)B * H * N;
    long long *rows = (long long *)malloc(sizeof(long long) * 3 * (size_t)n_rows);
    double *orow = (double *)malloc(sizeof(double) * (size_t)n_rows * d);
    double *lrow = (double *)malloc(sizeof(double) * (size_t)n_rows);
    long long r = 0;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (long long i = 0; i < N; ++i, ++r) {
                rows[3 * r] = b; rows[3 * r + 1] = h; rows[3 * r + 2] = i;
            }
    oracle_swat_fwd_rows(q, k, v, B, H, Hkv, N, d, window, n_sink, mode, slopes, rope_base,
                         n_rows, rows, orow, lrow);
    r = 0;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (long long i = 0; i < N; ++i, ++r) {
                memcpy(o + idx_q(b, i, h, N, H, d), orow + (size_t)r * d, sizeof(double) * d);
                if (lse) lse[((size_t)b * H + h) * N + i] = lrow[r];
            }
    free(rows); free(orow); free(lrow);
}

/* ------------------------------------------------------------------------ */
/* Backward (derived by calculus from the "SWAT" attention equation; the pages
 * print no backward, but SWAT is trained from scratch, so it exists).
 * With p = act(s), s = q'.k'/sqrt(d) + slope*(i-j), o_i = sum_j p_ij v_j:
 *   dv_j  = sum_i p_ij dO_i
 *   dP_ij = dO_i . v_j
 *   sigmoid: dS_ij = dP_ij p_ij (1 - p_ij)
 *   softmax: dS_ij = p_ij (dP_ij - D_i),  D_i = sum_j p_ij dP_ij
 *   dq'_i = sum_j dS_ij k'_j / sqrt(d),   dk'_j = sum_i dS_ij q'_i / sqrt(d)
 *   dq_i = R_i^T dq'_i,  dk_j = R_j^T dk'_j
 * For grouped KV heads the query heads of a group add into one dk/dv. */
void oracle_swat_bwd(const float *q, const float *k, const float *v, const float *dout,
                     double *dq, double *dk, double *dv,
                     int B, int H, int Hkv, int N, int d, int window, int n_sink, int mode,
                     const float *slopes, double rope_base)
{
    rope_table tb = rope_table_make(N, d, rope_base);
    int G = H / Hkv;
    double scale = 1.0 / sqrt((double)d);
    memset(dq, 0, sizeof(double) * (size_t)B * N * H * d);
    memset(dk, 0, sizeof(double) * (size_t)B * N * Hkv * d);
    memset(dv, 0, sizeof(double) * (size_t)B * N * Hkv * d);
    /* one (b, kv head) per task: it owns its dk/dv rows and the dq rows of its group */
    #pragma omp parallel
    {
        long long *keys = (long long *)malloc(sizeof(long long) * (size_t)N);
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        double *p = (double *)malloc(sizeof(double) * (size_t)N);
        double *dP = (double *)malloc(sizeof(double) * (size_t)N);
        double *qr = (double *)malloc(sizeof(double) * (size_t)d);
        double *kr = (double *)malloc(sizeof(double) * (size_t)d);
        double *dqr = (double *)malloc(sizeof(double) * (size_t)d);
        double *tmp = (double *)malloc(sizeof(double) * (size_t)d);
        double *dkr = (double *)malloc(sizeof(double) * (size_t)N * d);  /* rotated-space dk of this (b,kvh) */
        #pragma omp for schedule(dynamic, 1)
        for (long long task = 0; task < (long long)B * Hkv; ++task) {
            int b = (int)(task / Hkv), kvh = (int)(task % Hkv);
            memset(dkr, 0, sizeof(double) * (size_t)N * d);
            for (int g = 0; g < G; ++g) {
                int h = kvh * G + g;
                double slope = slopes ? (double)slopes[h] : 0.0;
                for (long long i = 0; i < N; ++i) {
                    long long n = row_scores(q, k, &tb, b, h, i, H, Hkv, N, d, window, n_sink,
                                             slope, keys, s, qr, kr);
                    row_weights(s, p, n, mode);
                    const float *dOi = dout + idx_q(b, i, h, N, H, d);
                    double D = 0.0;
                    for (long long a = 0; a < n; ++a) {
                        const float *vj = v + idx_q(b, keys[a], kvh, N, Hkv, d);
                        double acc = 0.0;
                        for (int c = 0; c < d; ++c) acc += (double)dOi[c] * (double)vj[c];
                        dP[a] = acc;
                        D += p[a] * acc;
                    }
                    for (int c = 0; c < d; ++c) dqr[c] = 0.0;
                    for (long long a = 0; a < n; ++a) {
                        long long j = keys[a];
                        double dS = (mode == MODE_SIGMOID) ? dP[a] * p[a] * (1.0 - p[a])
                                                           : p[a] * (dP[a] - D);
                        rope_apply(&tb, k + idx_q(b, j, kvh, N, Hkv, d), kr, d, j);
                        double *dvj = dv + idx_q(b, j, kvh, N, Hkv, d);
                        double *dkj = dkr + (size_t)j * d;
                        for (int c = 0; c < d; ++c) {
                            dqr[c] += dS * kr[c] * scale;
                            dkj[c] += dS * qr[c] * scale;
                            dvj[c] += p[a] * (double)dOi[c];
                        }
                    }
                    rope_apply_inv(&tb, dqr, tmp, d, i);
                    memcpy(dq + idx_q(b, i, h, N, H, d), tmp, sizeof(double) * d);
                }
            }
            for (long long j = 0; j < N; ++j) {
                rope_apply_inv(&tb, dkr + (size_t)j * d, tmp, d, j);
                memcpy(dk + idx_q(b, j, kvh, N, Hkv, d), tmp, sizeof(double) * d);
            }
        }
        free(keys); free(s); free(p); free(dP); free(qr); free(kr); free(dqr); free(tmp); free(dkr);
    }
    rope_table_free(&tb);
}

/* Backward for sampled rows, same formulas as oracle_swat_bwd.
 * dq rows: qrows[3r..] = (b, h, i)  -> dq_rows [n_q, d]
 * dk/dv rows: krows[3r..] = (b, kvh, j) -> dk_rows, dv_rows [n_k, d]
 * A key row needs p_ij of every query i that sees it; each such row's weights
 * are recomputed from its full score list. */
void oracle_swat_bwd_rows(const float *q, const float *k, const float *v, const float *dout,
                          int B, int H, int Hkv, int N, int d, int window, int n_sink, int mode,
                          const float *slopes, double rope_base,
                          long long n_q, const long long *qrows, double *dq_rows,
                          long long n_k, const long long *krows, double *dk_rows, double *dv_rows)
{
    (void)B;
    rope_table tb = rope_table_make(N, d, rope_base);
    int G = H / Hkv;
    double scale = 1.0 / sqrt((double)d);
    #pragma omp parallel
    {
        long long *keys = (long long *)malloc(sizeof(long long) * (size_t)N);
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        double *p = (double *)malloc(sizeof(double) * (size_t)N);
        double *qr = (double *)malloc(sizeof(double) * (size_t)d);
        double *kr = (double *)malloc(sizeof(double) * (size_t)d);
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
        #pragma omp for schedule(dynamic, 1)
        for (long long r = 0; r < n_q; ++r) {
            int b = (int)qrows[3 * r], h = (int)qrows[3 * r + 1];
            long long i = qrows[3 * r + 2];
            int kvh = h / G;
            double slope = slopes ? (double)slopes[h] : 0.0;
            long long n = row_scores(q, k, &tb, b, h, i, H, Hkv, N, d, window, n_sink,
                                     slope, keys, s, qr, kr);
            row_weights(s, p, n, mode);
            const float *dOi = dout + idx_q(b, i, h, N, H, d);
            double D = 0.0;
            double *dP = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
            for (long long a = 0; a < n; ++a) {
                const float *vj = v + idx_q(b, keys[a], kvh, N, Hkv, d);
                double t = 0.0;
                for (int c = 0; c < d; ++c) t += (double)dOi[c] * (double)vj[c];
                dP[a] = t; D += p[a] * t;
            }
            for (int c = 0; c < d; ++c) acc[c] = 0.0;
            for (long long a = 0; a < n; ++a) {
                double dS = (mode == MODE_SIGMOID) ? dP[a] * p[a] * (1.0 - p[a]) : p[a] * (dP[a] - D);
                rope_apply(&tb, k + idx_q(b, keys[a], kvh, N, Hkv, d), kr, d, keys[a]);
                for (int c = 0; c < d; ++c) acc[c] += dS * kr[c] * scale;
            }
            free(dP);
            rope_apply_inv(&tb, acc, dq_rows + (size_t)r * d, d, i);
        }
        double *dkacc = (double *)malloc(sizeof(double) * (size_t)d);
        #pragma omp for schedule(dynamic, 1)
        for (long long r = 0; r < n_k; ++r) {
            int b = (int)krows[3 * r], kvh = (int)krows[3 * r + 1];
            long long j = krows[3 * r + 2];
            double *dvj = dv_rows + (size_t)r * d;
            for (int c = 0; c < d; ++c) { dkacc[c] = 0.0; dvj[c] = 0.0; }
            for (int g = 0; g < G; ++g) {
                int h = kvh * G + g;
                double slope = slopes ? (double)slopes[h] : 0.0;
                for (long long i = j; i < N; ++i) {
                    if (!oracle_in_keyset(i, j, window, n_sink)) continue;
                    long long n = row_scores(q, k, &tb, b, h, i, H, Hkv, N, d, window, n_sink,
                                             slope, keys, s, qr, kr);
                    row_weights(s, p, n, mode);
                    const float *dOi = dout + idx_q(b, i, h, N, H, d);
                    double D = 0.0, pj = 0.0, dPj = 0.0;
                    for (long long a = 0; a < n; ++a) {
                        const float *va = v + idx_q(b, keys[a], kvh, N, Hkv, d);
                        double t = 0.0;
                        for (int c = 0; c < d; ++c) t += (double)dOi[c] * (double)va[c];
                        D += p[a] * t;
                        if (keys[a] == j) { pj = p[a]; dPj = t; }
                    }
                    double dS = (mode == MODE_SIGMOID) ? dPj * pj * (1.0 - pj) : pj * (dPj - D);
                    /* qr holds the rotated q_i from row_scores */
                    for (int c = 0; c < d; ++c) {
                        dkacc[c] += dS * qr[c] * scale;
                        dvj[c] += pj * (double)dOi[c];
                    }
                }
            }
            rope_apply_inv(&tb, dkacc, dk_rows + (size_t)r * d, d, j);
        }
        free(dkacc);
        free(keys); free(s); free(p); free(qr); free(kr); free(acc);
    }
    rope_table_free(&tb);
}

/* ------------------------------------------------------------------------ */
/* Ring-buffer KV cache and decode.
 * "Sliding Window Attention" glossary, ring-buffer paragraph: the cache holds
 * w slots; position i is written to slot i mod w, overwriting the oldest
 * entry. "Attention sink" entry: the first tokens are kept beside the window
 * (StreamingLLM). The cache stores rotated keys at their absolute positions.
 *
 * State (all double): kc, vc [B, Hkv, window, d]; ks, vs [B, Hkv, n_sink, d].
 * Slot contents are defined by the caller having written every position
 * 0..pos-1 of each sequence (or an equivalent fill). */

/* Write one token (raw k, v; k is rotated here) at position pos of sequence b. */
static void ring_write(double *kc, double *vc, double *ks, double *vs,
                       const float *k_tok, const float *v_tok, int b, int Hkv, int d,
                       int window, int n_sink, long long pos, double rope_base)
{
    double *kr = (double *)malloc(sizeof(double) * (size_t)d);
    long long slot = pos % window;
    for (int kvh = 0; kvh < Hkv; ++kvh) {
        for (int c = 0; c < d; ++c) kr[c] = (double)k_tok[(size_t)kvh * d + c];
        oracle_rope_rotate(kr, d, pos, rope_base);
        size_t base = (((size_t)b * Hkv + kvh) * window + (size_t)slot) * d;
        for (int c = 0; c < d; ++c) {
            kc[base + c] = kr[c];
            vc[base + c] = (double)v_tok[(size_t)kvh * d + c];
        }
        if (pos < n_sink) {
            size_t sb = (((size_t)b * Hkv + kvh) * n_sink + (size_t)pos) * d;
            for (int c = 0; c < d; ++c) {
                ks[sb + c] = kr[c];
                vs[sb + c] = (double)v_tok[(size_t)kvh * d + c];
            }
        }
    }
    free(kr);
}

/* Fill the cache of every sequence from a prefill: k, v [B, n_tok, Hkv, d]
 * hold positions p0 .. p0+n_tok-1. Tokens are written in order, so later
 * positions overwrite earlier ones in the ring, exactly as decode would. */
void oracle_cache_fill(double *kc, double *vc, double *ks, double *vs,
                       const float *k, const float *v, int B, int Hkv, int d,
                       int window, int n_sink, long long p0, long long n_tok, double rope_base)
{
    for (int b = 0; b < B; ++b)
        for (long long t = 0; t < n_tok; ++t) {
            size_t off = (((size_t)b * n_tok + (size_t)t) * Hkv) * d;
            ring_write(kc, vc, ks, vs, k + off, v + off, b, Hkv, d, window, n_sink,
                       p0 + t, rope_base);
        }
}

/* One decode step: q [B,H,d], k_new, v_new [B,Hkv,d], pos [B]. Writes the new
 * token first (it attends to itself), then attends over the ring slots whose
 * position pos - delta (delta = (pos - slot) mod window) is >= 0, plus the
 * sinks j < n_sink that lie before the window (j < pos - window + 1).
 * o [B,H,d]. */
void oracle_decode_step(double *kc, double *vc, double *ks, double *vs,
                        const float *q, const float *k_new, const float *v_new,
                        const long long *pos, double *o,
                        int B, int H, int Hkv, int d, int window, int n_sink, int mode,
                        const float *slopes, double rope_base)
{
    int G = H / Hkv;
    double scale = 1.0 / sqrt((double)d);
    for (int b = 0; b < B; ++b)
        ring_write(kc, vc, ks, vs, k_new + (size_t)b * Hkv * d, v_new + (size_t)b * Hkv * d,
                   b, Hkv, d, window, n_sink, pos[b], rope_base);
    #pragma omp parallel
    {
        double *qr = (double *)malloc(sizeof(double) * (size_t)d);
        double *s = (double *)malloc(sizeof(double) * (size_t)(window + n_sink));
        const double **kp = (const double **)malloc(sizeof(double *) * (size_t)(window + n_sink));
        const double **vp = (const double **)malloc(sizeof(double *) * (size_t)(window + n_sink));
        #pragma omp for schedule(dynamic, 1)
        for (long long task = 0; task < (long long)B * H; ++task) {
            int b = (int)(task / H), h = (int)(task % H), kvh = h / G;
            long long P = pos[b];
            double slope = slopes ? (double)slopes[h] : 0.0;
            for (int c = 0; c < d; ++c) qr[c] = (double)q[((size_t)b * H + h) * d + c];
            oracle_rope_rotate(qr, d, P, rope_base);
            int n = 0;
            for (int slot = 0; slot < window; ++slot) {
                long long delta = ((P - slot) % window + window) % window;
                if (P - delta < 0) continue;
                size_t base = (((size_t)b * Hkv + kvh) * window + (size_t)slot) * d;
                double dot = 0.0;
                for (int c = 0; c < d; ++c) dot += qr[c] * kc[base + c];
                s[n] = dot * scale + slope * (double)delta;
                kp[n] = kc + base; vp[n] = vc + base; ++n;
            }
            for (int j = 0; j < n_sink; ++j) {
                if (!(j < P - window + 1)) continue;
                size_t sb = (((size_t)b * Hkv + kvh) * n_sink + (size_t)j) * d;
                double dot = 0.0;
                for (int c = 0; c < d; ++c) dot += qr[c] * ks[sb + c];
                s[n] = dot * scale + slope * (double)(P - j);
                kp[n] = ks + sb; vp[n] = vs + sb; ++n;
            }
            double m = -INFINITY, l = 0.0;
            if (mode == MODE_SOFTMAX) {
                for (int a = 0; a < n; ++a) if (s[a] > m) m = s[a];
                for (int a = 0; a < n; ++a) l += exp(s[a] - m);
            }
            double *ob = o + ((size_t)b * H + h) * d;
            for (int c = 0; c < d; ++c) ob[c] = 0.0;
            for (int a = 0; a < n; ++a) {
                double pa = (mode == MODE_SIGMOID) ? oracle_sigmoid(s[a]) : exp(s[a] - m) / l;
                for (int c = 0; c < d; ++c) ob[c] += pa * vp[a][c];
            }
        }
        free(qr); free(s); free(kp); free(vp);
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
