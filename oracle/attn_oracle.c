/*
 * attn_oracle.c -- CPU reference for exact softmax attention, in fp64.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
 * call this file; only the tests, the package's smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or constant with
 * the CUDA library.
 *
 * What it computes (FlashAttention teaching pages, all three):
 *   - "GPU 学习日报 Day 21", section 3.1 (the standard three-step computation):
 *         S = Q K^T / sqrt(d);  P = softmax(S);  O = P V
 *     generalised to a caller-given scale and an optional causal mask (key j is
 *     excluded from query row i when j > i; section 6 table, "非因果计算浪费" row).
 *   - Same page, section 5.1: the numerically safe softmax is two passes over the
 *     row -- first the maximum m, then the sum of e^{x - m} and the division.
 *   - The saved statistic for the backward pass (airsota "science-depth-m4-047",
 *     section 3, point (c)) is read as the natural-log log-sum-exp of the scaled,
 *     masked score row:  LSE_i = m_i + ln(sum_j e^{s_ij - m_i}).
 *   - "GPU 学习日报 Day 21", sections 5.2 and 5.3: the one-pass online recurrence
 *         m_new = max(m_old, m_block)
 *         l_new = e^{m_old - m_new} l_old + sum_block e^{x - m_new}
 *         O_acc = e^{m_old - m_new} O_acc + e^{S_block - m_new} V_block
 *         O     = O_acc / l   (once, after the last block)
 *     is provided as a second, independent function so that the tests can pin
 *     the two against each other (the pages claim exact equality up to
 *     floating-point order: "GPU 学习日报 Day 21" FAQ Q1; "science-depth-m4-047" section 3).
 *   - The backward pass ("science-depth-m4-047", section 3, point (c): gradients recomputed
 *     from the saved statistics) is checked against the gradients of the same
 *     definition, written out in fp64 with every N x N matrix materialised:
 *         dV = P^T dO,  dP = dO V^T,  dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik),
 *         dQ = scale dS K,  dK = scale dS^T Q
 *     (the Jacobian of the row softmax applied to dP, and the chain rule
 *     through S = scale Q K^T).
 *
 * Every function materialises what the definition materialises (a full score
 * row), loops in the plain order of the formula and uses no blocking, fusion or
 * reordering beyond what the formula states.  Inputs are fp64 arrays; the
 * callers pass bf16 values widened exactly to fp64, so the oracle sees the very
 * numbers the GPU sees.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Softmax of one vector, two passes ("GPU 学习日报 Day 21", section 5.1).                  */
/* ------------------------------------------------------------------------ */
int oracle_softmax_two_pass(const double* x, int64_t n, double* p) {
    if (n <= 0 || !x || !p) return -1;
    double m = -INFINITY;
    for (int64_t i = 0; i < n; ++i) if (x[i] > m) m = x[i];          /* pass 1: max  */
    double l = 0.0;
    for (int64_t i = 0; i < n; ++i) { p[i] = exp(x[i] - m); l += p[i]; } /* pass 2: sum */
    for (int64_t i = 0; i < n; ++i) p[i] /= l;
    return 0;
}

/*
 * Softmax of one vector with the online recurrence, block by block
 * ("GPU 学习日报 Day 21", section 5.2 and its practice exercise 2).  After block b the
 * statistics (m, l) describe x[0 .. end of block b]; the outputs written so far
 * are rescaled by the correction factor e^{m_old - m_new}.  The correction
 * factor of every block is written to factors[b] when factors is non-null
 * (block 0 has m_old = -inf, factor 0).  Final m and l go to *m_out, *l_out.
 */
int oracle_online_softmax(const double* x, int64_t n, int64_t block, double* p,
                          double* m_out, double* l_out, double* factors) {
    if (n <= 0 || block <= 0 || !x || !p) return -1;
    double m = -INFINITY, l = 0.0;
    int64_t b = 0;
    for (int64_t start = 0; start < n; start += block, ++b) {
        int64_t end = start + block < n ? start + block : n;
        double m_block = -INFINITY;
        for (int64_t i = start; i < end; ++i) if (x[i] > m_block) m_block = x[i];
        double m_new = m > m_block ? m : m_block;
        double corr = exp(m - m_new);                 /* e^{m_old - m_new} */
        double psum = 0.0;
        for (int64_t i = start; i < end; ++i) { p[i] = exp(x[i] - m_new); psum += p[i]; }
        l = corr * l + psum;
        for (int64_t i = 0; i < start; ++i) p[i] *= corr; /* rescale earlier outputs */
        if (factors) factors[b] = corr;
        m = m_new;
    }
    for (int64_t i = 0; i < n; ++i) p[i] /= l;
    if (m_out) *m_out = m;
    if (l_out) *l_out = l;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Attention, standard three steps, one query row at a time.                 */
/* ------------------------------------------------------------------------ */

/* Number of keys query row i may attend to: all N, or 0..i when causal. */
static int64_t allowed_keys(int64_t i, int64_t N, int causal) {
    return causal ? (i + 1 < N ? i + 1 : N) : N;
}

/*
 * One row of the textbook computation.  s is scratch of length >= N.
 * Writes O_i (d values) and LSE_i; when p_out is non-null also writes the
 * probability row P_i (length N, zero for masked keys).
 */
static void attention_row_three_step(const double* qi, const double* K, const double* V,
                                     int64_t N, int64_t d, int64_t i, int causal, double scale,
                                     double* s, double* o_i, double* lse_i, double* p_out) {
    const int64_t n = allowed_keys(i, N, causal);
    /* step 1: the score row S_i = scale * q_i . k_j for every allowed key j */
    for (int64_t j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int64_t c = 0; c < d; ++c) acc += qi[c] * K[j * d + c];
        s[j] = scale * acc;
    }
    /* step 2: safe softmax in two passes -> probability row P_i */
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j) if (s[j] > m) m = s[j];
    double l = 0.0;
    for (int64_t j = 0; j < n; ++j) { s[j] = exp(s[j] - m); l += s[j]; }
    for (int64_t j = 0; j < n; ++j) s[j] /= l;
    /* step 3: O_i = P_i V */
    for (int64_t c = 0; c < d; ++c) o_i[c] = 0.0;
    for (int64_t j = 0; j < n; ++j)
        for (int64_t c = 0; c < d; ++c) o_i[c] += s[j] * V[j * d + c];
    *lse_i = m + log(l);
    if (p_out) {
        for (int64_t j = 0; j < n; ++j) p_out[j] = s[j];
        for (int64_t j = n; j < N; ++j) p_out[j] = 0.0;
    }
}

/*
 * One row of the online (FlashAttention) recurrence with key blocks of size
 * `block` ("GPU 学习日报 Day 21", section 5.3).  Every key block: scores, block max,
 * correction factor, rescale of l and O_acc, accumulate e^{s - m_new} V.
 * Normalise once at the end.
 */
static void attention_row_online(const double* qi, const double* K, const double* V,
                                 int64_t N, int64_t d, int64_t i, int causal, double scale,
                                 int64_t block, double* s, double* o_i, double* lse_i) {
    const int64_t n = allowed_keys(i, N, causal);
    double m = -INFINITY, l = 0.0;
    for (int64_t c = 0; c < d; ++c) o_i[c] = 0.0;
    for (int64_t start = 0; start < n; start += block) {
        int64_t end = start + block < n ? start + block : n;
        double m_block = -INFINITY;
        for (int64_t j = start; j < end; ++j) {
            double acc = 0.0;
            for (int64_t c = 0; c < d; ++c) acc += qi[c] * K[j * d + c];
            s[j - start] = scale * acc;
            if (s[j - start] > m_block) m_block = s[j - start];
        }
        double m_new = m > m_block ? m : m_block;
        double corr = exp(m - m_new);
        double psum = 0.0;
        for (int64_t c = 0; c < d; ++c) o_i[c] *= corr;
        for (int64_t j = start; j < end; ++j) {
            double pj = exp(s[j - start] - m_new);
            psum += pj;
            for (int64_t c = 0; c < d; ++c) o_i[c] += pj * V[j * d + c];
        }
        l = corr * l + psum;
        m = m_new;
    }
    for (int64_t c = 0; c < d; ++c) o_i[c] /= l;
    *lse_i = m + log(l);
}

/* ------------------------------------------------------------------------ */
/* Row-parallel drivers (threads over the requested (head, row) pairs).     */
/* ------------------------------------------------------------------------ */
typedef struct {
    const double *q, *k, *v;
    int64_t Nq, N, d;   /* query rows and key rows per head */
    int causal;
    double scale;
    int64_t block;          /* 0 = three-step definition, > 0 = online recurrence */
    const int64_t *bh_idx, *row_idx;
    int64_t nrows, first, stride;
    double *o_out, *lse_out;
    int status;
} job_t;

static void* run_rows(void* arg) {
    job_t* jb = (job_t*)arg;
    double* s = (double*)malloc(sizeof(double) * (size_t)(jb->N > 0 ? jb->N : 1));
    if (!s) { jb->status = -2; return NULL; }
    const int64_t head = jb->N * jb->d;
    const int64_t head_q = jb->Nq * jb->d;
    for (int64_t r = jb->first; r < jb->nrows; r += jb->stride) {
        const int64_t bh = jb->bh_idx[r], i = jb->row_idx[r];
        const double* qi = jb->q + bh * head_q + i * jb->d;
        const double* K = jb->k + bh * head;
        const double* V = jb->v + bh * head;
        if (jb->block > 0)
            attention_row_online(qi, K, V, jb->N, jb->d, i, jb->causal, jb->scale, jb->block,
                                 s, jb->o_out + r * jb->d, jb->lse_out + r);
        else
            attention_row_three_step(qi, K, V, jb->N, jb->d, i, jb->causal, jb->scale,
                                     s, jb->o_out + r * jb->d, jb->lse_out + r, NULL);
    }
    free(s);
    return NULL;
}

static int run_parallel(const double* q, const double* k, const double* v, int64_t BH,
                        int64_t Nq, int64_t N, int64_t d, int causal, double scale, int64_t block,
                        const int64_t* bh_idx, const int64_t* row_idx, int64_t nrows,
                        double* o_out, double* lse_out, int nthreads) {
    if (!q || !k || !v || !bh_idx || !row_idx || !o_out || !lse_out) return -1;
    if (BH <= 0 || Nq <= 0 || N <= 0 || d <= 0 || nrows < 0) return -1;
    if (causal && Nq != N) return -1;   /* causal is defined for square attention only */
    for (int64_t r = 0; r < nrows; ++r)
        if (bh_idx[r] < 0 || bh_idx[r] >= BH || row_idx[r] < 0 || row_idx[r] >= Nq) return -1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if ((int64_t)nthreads > nrows) nthreads = nrows > 0 ? (int)nrows : 1;
    job_t jobs[256];
    pthread_t th[256];
    for (int t = 0; t < nthreads; ++t) {
        job_t jb = {q, k, v, Nq, N, d, causal, scale, block, bh_idx, row_idx, nrows, t, nthreads,
                    o_out, lse_out, 0};
        jobs[t] = jb;
    }
    int launched = 0;
    for (int t = 1; t < nthreads; ++t) {
        if (pthread_create(&th[t], NULL, run_rows, &jobs[t]) != 0) break;
        launched = t;
    }
    /* rows of threads that failed to start run on the calling thread */
    for (int t = launched + 1; t < nthreads; ++t) run_rows(&jobs[t]);
    run_rows(&jobs[0]);
    for (int t = 1; t <= launched; ++t) pthread_join(th[t], NULL);
    for (int t = 0; t < nthreads; ++t) if (jobs[t].status) return jobs[t].status;
    return 0;
}

/*
 * The oracle proper: standard three-step attention for the listed
 * (head, query-row) pairs.  q, k, v: [BH, N, d] fp64, contiguous.
 * Outputs: o_out [nrows, d], lse_out [nrows].  Returns 0, or -1 on bad
 * arguments, -2 when scratch memory cannot be had.
 */
int oracle_attention_rows(const double* q, const double* k, const double* v, int64_t BH,
                          int64_t N, int64_t d, int causal, double scale,
                          const int64_t* bh_idx, const int64_t* row_idx, int64_t nrows,
                          double* o_out, double* lse_out, int nthreads) {
    return run_parallel(q, k, v, BH, N, N, d, causal, scale, 0, bh_idx, row_idx, nrows,
                        o_out, lse_out, nthreads);
}

/*
 * Non-causal attention of Nq query rows against Nk key/value rows per head
 * (the decode case, Nq = 1: one new query attends to every cached key;
 * "GPU 学习日报 Day 21", section 9 and FAQ Q5).  q: [BH, Nq, d]; k, v: [BH, Nk, d].  The same
 * three-step definition per row.
 */
int oracle_attention_rows_qk(const double* q, const double* k, const double* v, int64_t BH,
                             int64_t Nq, int64_t Nk, int64_t d, double scale,
                             const int64_t* bh_idx, const int64_t* row_idx, int64_t nrows,
                             double* o_out, double* lse_out, int nthreads) {
    return run_parallel(q, k, v, BH, Nq, Nk, d, 0, scale, 0, bh_idx, row_idx, nrows,
                        o_out, lse_out, nthreads);
}

/* The one-pass online recurrence with key blocks of `block` keys (block >= 1). */
int oracle_attention_rows_online(const double* q, const double* k, const double* v,
                                 int64_t BH, int64_t N, int64_t d, int causal, double scale,
                                 int64_t block, const int64_t* bh_idx, const int64_t* row_idx,
                                 int64_t nrows, double* o_out, double* lse_out, int nthreads) {
    if (block < 1) return -1;
    return run_parallel(q, k, v, BH, N, N, d, causal, scale, block, bh_idx, row_idx, nrows,
                        o_out, lse_out, nthreads);
}

/* The probability row P_i of one query row (length N, zero for masked keys). */
int oracle_attention_prob_row(const double* q, const double* k, const double* v, int64_t BH,
                              int64_t N, int64_t d, int causal, double scale, int64_t bh,
                              int64_t i, double* p_out) {
    if (!q || !k || !v || !p_out || BH <= 0 || N <= 0 || d <= 0) return -1;
    if (bh < 0 || bh >= BH || i < 0 || i >= N) return -1;
    double* s = (double*)malloc(sizeof(double) * (size_t)N);
    double* o = (double*)malloc(sizeof(double) * (size_t)d);
    if (!s || !o) { free(s); free(o); return -2; }
    double lse;
    const int64_t head = N * d;
    attention_row_three_step(q + bh * head + i * d, k + bh * head, v + bh * head, N, d, i,
                             causal, scale, s, o, &lse, p_out);
    free(s);
    free(o);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Gradients of the definition (one head at a time, every matrix in full).  */
/* ------------------------------------------------------------------------ */
typedef struct {
    const double *q, *k, *v, *dout;
    double *P, *dS;
    int64_t N, d;
    int causal;
    double scale;
    int64_t first, stride;
    double *dq, *dk, *dv;
} bwd_job_t;

/* Rows: P_i (softmax of the masked, scaled score row), dP_i, dS_i, dQ_i. */
static void* bwd_rows(void* arg) {
    bwd_job_t* jb = (bwd_job_t*)arg;
    const int64_t N = jb->N, d = jb->d;
    double* dp = (double*)malloc(sizeof(double) * (size_t)N);
    if (!dp) return NULL;
    for (int64_t i = jb->first; i < N; i += jb->stride) {
        double* Pi = jb->P + i * N;
        double* dSi = jb->dS + i * N;
        const int64_t n = allowed_keys(i, N, jb->causal);
        double m = -INFINITY;
        for (int64_t j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int64_t c = 0; c < d; ++c) acc += jb->q[i * d + c] * jb->k[j * d + c];
            Pi[j] = jb->scale * acc;
            if (Pi[j] > m) m = Pi[j];
        }
        double l = 0.0;
        for (int64_t j = 0; j < n; ++j) { Pi[j] = exp(Pi[j] - m); l += Pi[j]; }
        for (int64_t j = 0; j < n; ++j) Pi[j] /= l;
        for (int64_t j = n; j < N; ++j) Pi[j] = 0.0;
        /* dP_ij = dO_i . v_j ;  dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik) */
        double row = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int64_t c = 0; c < d; ++c) acc += jb->dout[i * d + c] * jb->v[j * d + c];
            dp[j] = acc;
            row += Pi[j] * acc;
        }
        for (int64_t j = 0; j < n; ++j) dSi[j] = Pi[j] * (dp[j] - row);
        for (int64_t j = n; j < N; ++j) dSi[j] = 0.0;
        /* dQ_i = scale * sum_j dS_ij k_j */
        for (int64_t c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int64_t j = 0; j < n; ++j) acc += dSi[j] * jb->k[j * d + c];
            jb->dq[i * d + c] = jb->scale * acc;
        }
    }
    free(dp);
    return NULL;
}

/* Columns: dV_j = sum_i P_ij dO_i ;  dK_j = scale * sum_i dS_ij q_i. */
static void* bwd_cols(void* arg) {
    bwd_job_t* jb = (bwd_job_t*)arg;
    const int64_t N = jb->N, d = jb->d;
    for (int64_t j = jb->first; j < N; j += jb->stride) {
        for (int64_t c = 0; c < d; ++c) {
            double av = 0.0, ak = 0.0;
            for (int64_t i = 0; i < N; ++i) {
                av += jb->P[i * N + j] * jb->dout[i * d + c];
                ak += jb->dS[i * N + j] * jb->q[i * d + c];
            }
            jb->dv[j * d + c] = av;
            jb->dk[j * d + c] = jb->scale * ak;
        }
    }
    return NULL;
}

/*
 * Gradients of L = sum(dO * O) for one head: q, k, v, dout [N, d] fp64 in;
 * dq, dk, dv [N, d] fp64 out.  Returns 0, -1 on bad arguments, -2 when the
 * N x N scratch matrices cannot be allocated.
 */
int oracle_attention_backward(const double* q, const double* k, const double* v,
                              const double* dout, int64_t N, int64_t d, int causal, double scale,
                              double* dq, double* dk, double* dv, int nthreads) {
    if (!q || !k || !v || !dout || !dq || !dk || !dv || N <= 0 || d <= 0) return -1;
    double* P = (double*)malloc(sizeof(double) * (size_t)N * (size_t)N);
    double* dS = (double*)malloc(sizeof(double) * (size_t)N * (size_t)N);
    if (!P || !dS) { free(P); free(dS); return -2; }
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if ((int64_t)nthreads > N) nthreads = (int)N;
    bwd_job_t jobs[256];
    pthread_t th[256];
    for (int phase = 0; phase < 2; ++phase) {
        void* (*fn)(void*) = phase == 0 ? bwd_rows : bwd_cols;
        for (int t = 0; t < nthreads; ++t) {
            bwd_job_t jb = {q, k, v, dout, P, dS, N, d, causal, scale, t, nthreads, dq, dk, dv};
            jobs[t] = jb;
        }
        int launched = 0;
        for (int t = 1; t < nthreads; ++t) {
            if (pthread_create(&th[t], NULL, fn, &jobs[t]) != 0) break;
            launched = t;
        }
        for (int t = launched + 1; t < nthreads; ++t) fn(&jobs[t]);
        fn(&jobs[0]);
        for (int t = 1; t <= launched; ++t) pthread_join(th[t], NULL);
    }
    free(P);
    free(dS);
    return 0;
}
