/*
 * Exact scaled dot-product attention, fp64, on the CPU.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the oracle that the CUDA library is
 * checked against. Only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark may load it; the product path never does. It shares no
 * code, header, table or constant with the CUDA sources.
 *
 * What it computes, per (batch*head bh, query row i), follows the three steps
 * of the standard attention computation as the pages describe them
 * ("The Computational Steps of Standard Self-Attention", grasp.study lesson;
 * and the boundary-crossing walk-through on "Attention Is Memory-Bound, and
 * Nobody Noticed for Five Years", anylearn.cc):
 *
 *   1. scores      s_j = scale * sum_k q[i,k] * K[j,k]          for j in J(i)
 *   2. softmax     p_j = exp(s_j - m) / l,  m = max_j s_j,  l = sum_j exp(s_j - m)
 *   3. output      o[i,:] = sum_j p_j * V[j,:]
 *
 * plus the per-row log-sum-exp lse_i = m + ln(l) (natural logarithm).
 *
 * J(i) = {0..N-1}, or {0..i} when causal (key j allowed iff j <= i). Masked
 * keys are excluded from the softmax, which is what setting their logit to
 * -inf before the softmax means. A causal row always has key j = i, so no row
 * is empty; if a row were empty anyway the oracle writes o = 0, lse = -inf.
 *
 * With fewer queries than keys (Nq <= Nk, the shape of generating new tokens
 * against a long context) the Nq queries are the last Nq positions of the
 * sequence: causally, query i may see keys j <= i + (Nk - Nq); for Nq = Nk
 * that is the rule above.
 *
 * The anylearn.cc page ("FlashAttention computes exactly the same function as
 * standard attention ... to within floating point reassociation") is why the
 * plain definition is the oracle for the fused kernel.
 *
 * Inputs are either bf16 bit patterns (converted exactly to double) or
 * doubles. All arithmetic is IEEE double with libm exp/log; no reassociation,
 * no fused multiply-add (built with -ffp-contract=off).
 *
 * Rows to evaluate are given as (bh, i) pairs so that a seeded sample of rows
 * can be checked on large shapes; rows are grouped by head, each head's K and
 * V are converted to double once, and the head's rows are split over threads.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

enum { IN_BF16 = 0, IN_F64 = 1, IN_E4M3 = 2 };

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
static double bf16_bits_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP 8-bit floating point E4M3 (the "fn" variant: finite values and NaN
 * only): sign bit, 4 exponent bits with bias 7, 3 mantissa bits. Exponent
 * field 0 encodes subnormals m * 2^-9; exponent 15 with mantissa 7 is NaN
 * (there is no infinity), so the largest value is 1.75 * 2^8 = 448. */
double oracle_e4m3_to_double(uint8_t bits) {
    int sign = (bits >> 7) & 1;
    int e = (bits >> 3) & 0xF;
    int m = bits & 0x7;
    double mag;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m, -9);
    else
        mag = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -mag : mag;
}

static double load_elem(const void *base, int kind, int64_t idx) {
    if (kind == IN_F64) return ((const double *)base)[idx];
    if (kind == IN_E4M3) return oracle_e4m3_to_double(((const uint8_t *)base)[idx]);
    return bf16_bits_to_double(((const uint16_t *)base)[idx]);
}

/* Step 1: the scores of query q (length d, sequence position pos) against
 * keys j0..j1-1: s[j - j0] = scale * q.K[j] - slope * |pos - j| (the second
 * term is the linear distance bias; slope = 0 leaves the plain score). */
static void scores_row(const double *q, const double *K, int j0, int j1, int d,
                       double scale, double slope, int64_t pos, double *s) {
    for (int j = j0; j < j1; ++j) {
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += q[c] * K[(int64_t)j * d + c];
        s[j - j0] = scale * dot;
        if (slope != 0.0) s[j - j0] -= slope * fabs((double)(pos - j));
    }
}

/* Step 2: softmax of s[0..n-1] in place; returns m and l through pointers. */
static void softmax_row(double *s, int n, double *m_out, double *l_out) {
    double m = -INFINITY;
    for (int j = 0; j < n; ++j)
        if (s[j] > m) m = s[j];
    double l = 0.0;
    for (int j = 0; j < n; ++j) {
        s[j] = exp(s[j] - m);
        l += s[j];
    }
    for (int j = 0; j < n; ++j) s[j] /= l;
    *m_out = m;
    *l_out = l;
}

/* Step 3: o = sum_j p_j * V[j,:] over keys j0..j1-1 (p indexed from j0). */
static void output_row(const double *p, const double *V, int j0, int j1, int d,
                       double *o) {
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (int j = j0; j < j1; ++j)
        for (int c = 0; c < d; ++c) o[c] += p[j - j0] * V[(int64_t)j * d + c];
}

/* One query row of one head: steps 1-3 and the log-sum-exp over the allowed
 * keys j0..j1-1. */
static void attend_row(const double *q, const double *K, const double *V, int j0,
                       int j1, int d, double scale, double slope, int64_t pos,
                       double *s_buf, double *o, double *lse) {
    if (j1 <= j0) {
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        *lse = -INFINITY;
        return;
    }
    double m, l;
    scores_row(q, K, j0, j1, d, scale, slope, pos, s_buf);
    softmax_row(s_buf, j1 - j0, &m, &l);
    output_row(s_buf, V, j0, j1, d, o);
    *lse = m + log(l);
}

/* Allowed keys of query i, as the range j0..j1-1. Query i is sequence
 * position pos = i + (Nk - Nq). Key j is allowed iff j < Nk, and j <= pos when
 * causal, and j >= pos - wl when wl >= 0, and j <= pos + wr when wr >= 0
 * (a window of wl keys before the query's position and wr after it; a
 * negative bound means unbounded on that side). */
static void key_range(int i, int Nq, int Nk, int causal, int wl, int wr, int *j0,
                      int *j1) {
    int64_t pos = (int64_t)i + (Nk - Nq);
    int64_t hi = Nk - 1;
    if (causal && pos < hi) hi = pos;
    if (wr >= 0 && pos + wr < hi) hi = pos + wr;
    int64_t lo = 0;
    if (wl >= 0 && pos - wl > lo) lo = pos - wl;
    if (hi < lo - 1) hi = lo - 1;
    *j0 = (int)lo;
    *j1 = (int)(hi + 1);
}

typedef struct {
    const void *q;
    int kind;
    const double *K, *V; /* this head, converted */
    int64_t bh;
    int N, d, causal;
    double scale;
    const int64_t *rows;  /* all (bh, i) pairs */
    const int64_t *mine;  /* indices into rows[] for this head */
    int64_t nmine;
    int Nq;               /* query rows per head (N is the key count) */
    int wl, wr;           /* window bounds, negative = unbounded */
    double slope;         /* distance-bias slope of this head (0 = none) */
    int tid, nthreads;
    double *o, *lse;
    int ok;        /* set to 1 by run_job when its rows are done */
    int joinable;  /* 1 if run on its own pthread */
} job_t;

static void *run_job(void *arg) {
    job_t *jb = (job_t *)arg;
    double *s = (double *)malloc(sizeof(double) * (size_t)jb->N);
    double *qrow = (double *)malloc(sizeof(double) * (size_t)jb->d);
    if (!s || !qrow) {
        jb->ok = 0;
        free(s);
        free(qrow);
        return NULL;
    }
    for (int64_t t = jb->tid; t < jb->nmine; t += jb->nthreads) {
        int64_t r = jb->mine[t];
        int i = (int)jb->rows[2 * r + 1];
        int64_t qoff = (jb->bh * jb->Nq + i) * (int64_t)jb->d;
        for (int c = 0; c < jb->d; ++c) qrow[c] = load_elem(jb->q, jb->kind, qoff + c);
        int j0, j1;
        key_range(i, jb->Nq, jb->N, jb->causal, jb->wl, jb->wr, &j0, &j1);
        attend_row(qrow, jb->K, jb->V, j0, j1, jb->d, jb->scale, jb->slope,
                   (int64_t)i + (jb->N - jb->Nq), s, jb->o + r * (int64_t)jb->d,
                   jb->lse + r);
    }
    free(s);
    free(qrow);
    jb->ok = 1;
    return NULL;
}

int oracle_default_threads(void) {
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

static int attend(const void *q, const void *k, const void *v, int kind, int B,
                  int H, int Nq, int N, int d, double scale, int causal, int wl,
                  int wr, const double *slopes, const int64_t *rows, int64_t nrows,
                  double *o, double *lse, int nthreads) {
    if (!q || !k || !v || !rows || !o || !lse) return -1;
    if (B <= 0 || H <= 0 || Nq <= 0 || N <= 0 || d <= 0 || nrows < 0) return -2;
    if (causal && Nq > N) return -2;
    if (!isfinite(scale)) return -3;
    if (slopes)
        for (int h = 0; h < H; ++h)
            if (!isfinite(slopes[h])) return -3;
    if (nthreads <= 0) nthreads = oracle_default_threads();
    int64_t BH = (int64_t)B * H;
    for (int64_t r = 0; r < nrows; ++r) {
        if (rows[2 * r] < 0 || rows[2 * r] >= BH) return -4;
        if (rows[2 * r + 1] < 0 || rows[2 * r + 1] >= Nq) return -4;
    }
    int64_t head_elems = (int64_t)N * d;
    double *K = (double *)malloc(sizeof(double) * (size_t)head_elems);
    double *V = (double *)malloc(sizeof(double) * (size_t)head_elems);
    int64_t *mine = (int64_t *)malloc(sizeof(int64_t) * (size_t)(nrows > 0 ? nrows : 1));
    job_t *jobs = (job_t *)calloc((size_t)nthreads, sizeof(job_t));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    int status = 0;
    if (!K || !V || !mine || !jobs || !th) status = -5;

    for (int64_t bh = 0; bh < BH && status == 0; ++bh) {
        int64_t nmine = 0;
        for (int64_t r = 0; r < nrows; ++r)
            if (rows[2 * r] == bh) mine[nmine++] = r;
        if (nmine == 0) continue;
        int64_t base = bh * head_elems;
        for (int64_t e = 0; e < head_elems; ++e) {
            K[e] = load_elem(k, kind, base + e);
            V[e] = load_elem(v, kind, base + e);
        }
        int nt = nmine < nthreads ? (int)nmine : nthreads;
        for (int t = 0; t < nt; ++t) {
            double slope = slopes ? slopes[bh % H] : 0.0;
            job_t jb = {q, kind, K, V, bh, N, d, causal, scale, rows, mine, nmine, Nq,
                        wl, wr, slope, t, nt, o, lse, 0, 0};
            jobs[t] = jb;
        }
        /* A thread that cannot be created runs its share inline. */
        for (int t = 1; t < nt; ++t) {
            if (pthread_create(&th[t], NULL, run_job, &jobs[t]) == 0)
                jobs[t].joinable = 1;
            else
                run_job(&jobs[t]);
        }
        run_job(&jobs[0]);
        for (int t = 1; t < nt; ++t)
            if (jobs[t].joinable) pthread_join(th[t], NULL);
        for (int t = 0; t < nt; ++t)
            if (!jobs[t].ok) status = -5;
    }
    free(K);
    free(V);
    free(mine);
    free(jobs);
    free(th);
    return status;
}

/* q, k, v: bf16 bit patterns, [B, H, N, d] contiguous. rows: nrows (bh, i)
 * pairs. o: [nrows, d] doubles; lse: [nrows] doubles. nthreads <= 0 means all
 * online cores. Returns 0 on success, negative on bad arguments or failure. */
int oracle_attn_bf16(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     int B, int H, int N, int d, double scale, int causal,
                     const int64_t *rows, int64_t nrows, double *o, double *lse,
                     int nthreads) {
    return attend(q, k, v, IN_BF16, B, H, N, N, d, scale, causal, -1, -1, NULL, rows,
                  nrows, o, lse, nthreads);
}

/* Same as oracle_attn_bf16 with double inputs (values need not be bf16). */
int oracle_attn_f64(const double *q, const double *k, const double *v, int B,
                    int H, int N, int d, double scale, int causal,
                    const int64_t *rows, int64_t nrows, double *o, double *lse,
                    int nthreads) {
    return attend(q, k, v, IN_F64, B, H, N, N, d, scale, causal, -1, -1, NULL, rows,
                  nrows, o, lse, nthreads);
}

/* Nq queries against Nk keys per head: q is [B, H, Nq, d], k and v are
 * [B, H, Nk, d] (bf16 bit patterns); rows are (bh, i) with i < Nq; causal
 * requires Nq <= Nk (the queries are the last Nq positions). */
int oracle_attn_kv_bf16(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        int B, int H, int Nq, int Nk, int d, double scale,
                        int causal, const int64_t *rows, int64_t nrows, double *o,
                        double *lse, int nthreads) {
    return attend(q, k, v, IN_BF16, B, H, Nq, Nk, d, scale, causal, -1, -1, NULL, rows,
                  nrows, o, lse, nthreads);
}

/* Same with double inputs. */
int oracle_attn_kv_f64(const double *q, const double *k, const double *v, int B,
                       int H, int Nq, int Nk, int d, double scale, int causal,
                       const int64_t *rows, int64_t nrows, double *o, double *lse,
                       int nthreads) {
    return attend(q, k, v, IN_F64, B, H, Nq, Nk, d, scale, causal, -1, -1, NULL, rows,
                  nrows, o, lse, nthreads);
}

/* Masked and position-biased variants (the bespoke biases, masks and
 * position encodings that, per the anylearn.cc page, a fused library's fast
 * path does not cover): keys limited to the window
 * [pos - wl, pos + wr] (negative bound = unbounded) on top of the causal
 * rule, and, when slopes is not NULL, the score of key j for a query at
 * position pos lowered by slopes[h] * |pos - j| (a linear distance bias per
 * head h). wl = wr = -1 with slopes = NULL is oracle_attn_kv_*. */
int oracle_attn_ext_bf16(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         int B, int H, int Nq, int Nk, int d, double scale,
                         int causal, int wl, int wr, const double *slopes,
                         const int64_t *rows, int64_t nrows, double *o, double *lse,
                         int nthreads) {
    return attend(q, k, v, IN_BF16, B, H, Nq, Nk, d, scale, causal, wl, wr, slopes,
                  rows, nrows, o, lse, nthreads);
}

/* Same with double inputs. */
int oracle_attn_ext_f64(const double *q, const double *k, const double *v, int B,
                        int H, int Nq, int Nk, int d, double scale, int causal, int wl,
                        int wr, const double *slopes, const int64_t *rows,
                        int64_t nrows, double *o, double *lse, int nthreads) {
    return attend(q, k, v, IN_F64, B, H, Nq, Nk, d, scale, causal, wl, wr, slopes, rows,
                  nrows, o, lse, nthreads);
}

/* FP8 inputs: q, k, v hold E4M3 codes [B, H, N, d]; the values attended are
 * q_descale * Q, k_descale * K, v_descale * V (decoded exactly, scaled in
 * double), i.e. attention of the dequantized tensors. */
int oracle_attn_e4m3(const uint8_t *q, const uint8_t *k, const uint8_t *v, int B, int H,
                     int N, int d, double scale, double q_descale, double k_descale,
                     double v_descale, int causal, const int64_t *rows, int64_t nrows,
                     double *o, double *lse, int nthreads) {
    if (!isfinite(q_descale) || !isfinite(k_descale) || !isfinite(v_descale)) return -3;
    /* scores scale * (qd Q).(kd K) = (scale qd kd) Q.K; output vd * (P V) */
    int st = attend(q, k, v, IN_E4M3, B, H, N, N, d, scale * q_descale * k_descale, causal, -1,
                    -1, NULL, rows, nrows, o, lse, nthreads);
    if (st != 0) return st;
    for (int64_t r = 0; r < nrows * (int64_t)d; ++r) o[r] *= v_descale;
    return 0;
}

/* The probability row p[0..N-1] of query i for a single head (q: [N, d],
 * k: [N, d] doubles); masked keys get p = 0. Steps 1-2 only. */
int oracle_probs_f64(const double *q, const double *k, int N, int d,
                     double scale, int causal, int i, double *p) {
    if (!q || !k || !p || N <= 0 || d <= 0 || i < 0 || i >= N) return -1;
    int j0, j1;
    key_range(i, N, N, causal, -1, -1, &j0, &j1);
    double m, l;
    for (int j = 0; j < N; ++j) p[j] = 0.0;
    scores_row(q + (int64_t)i * d, k, j0, j1, d, scale, 0.0, i, p + j0);
    softmax_row(p + j0, j1 - j0, &m, &l);
    return 0;
}

/* The elementwise chain of the anylearn.cc page ("multiply a tensor by a
 * scalar, add a bias, apply an activation"): y[r, c] = act(alpha * x[r, c] +
 * b[c]) for bf16 x [rows, cols] and b [cols], in double. act 0: max(z, 0);
 * 1: z * (1 + erf(z / sqrt(2))) / 2 (GELU with the exact normal CDF);
 * 2: z / (1 + exp(-z)) (SiLU); 3: z * (1 + tanh(sqrt(2/pi) * (z + 0.044715 z^3))) / 2
 * (GELU, tanh form). Returns 0, or -1 on bad arguments. */
int oracle_chain_bf16(const uint16_t *x, const uint16_t *b, int64_t rows, int cols,
                      double alpha, int act, double *y) {
    if (!x || !b || !y || rows < 1 || cols < 1 || act < 0 || act > 3) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        for (int c = 0; c < cols; ++c) {
            double z = alpha * bf16_bits_to_double(x[r * cols + c]) + bf16_bits_to_double(b[c]);
            double out;
            if (act == 0)
                out = z > 0.0 ? z : 0.0;
            else if (act == 1)
                out = 0.5 * z * (1.0 + erf(z / sqrt(2.0)));
            else if (act == 2)
                out = z / (1.0 + exp(-z));
            else
                out = 0.5 * z * (1.0 + tanh(sqrt(2.0 / acos(-1.0)) * (z + 0.044715 * z * z * z)));
            y[r * cols + c] = out;
        }
    }
    return 0;
}
