/*
 * pi_oracle.c -- plain fp64 CPU oracle of the pi-attention forward operator.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the bench's CPU-baseline
 * leg may load this library.  The product path (the CUDA library) never calls, links or includes
 * anything from here, and nothing here comes from the CUDA path: the two share no code.
 *
 * What it computes, for every query row i of every (b, h), written out as the definition with no
 * blocking, fusion or reordering (sources: "pi-Attention: Periodic Sparse Transformers for
 * Efficient Long-Context Modeling", gist.science summary, section 2 "Methodology", Core
 * Components: Ring-Local Attention, pi-Skip Attention, Dynamic Adaptive Fusion):
 *
 *   window  L(i) = { j : max(0, i-k) <= j <= i }              the token and the k tokens before it
 *   skips   P(i) = { i - m*pi : 1 <= m <= S, m*pi > k, i - m*pi >= 0 }
 *           (a skip that lands inside the window is dropped; its key keeps the window's prior)
 *
 *   backward (the gradient of a scalar loss through out, given dO = dLoss/dout; not printed on the
 *   pages -- the chain rule through the forward above, for the training the pages report):
 *           dp_j = dO_i . v_j,  D_i = sum_j p_j dp_j,  ds_j = p_j (dp_j - D_i)
 *           dq_i = tau sum_j ds_j k_j + dz_i w_g[h],    dk_j += tau ds_j q_i,   dv_j += p_j dO_i
 *           dz_i = (1 - alpha) sum_{j in L} ds_j - alpha sum_{j in P} ds_j
 *                  (d log(alpha)/dz = 1 - alpha, d log(1 - alpha)/dz = -alpha)
 *           dw_g[h] += dz_i q_i,  db_g[h] += dz_i
 *
 *   bidirectional variant (same sections: the window reaches "both forward and backward", and "in
 *   bidirectional settings" the skips also reach i + pi), for a sequence of n tokens:
 *   window  L(i) = { j : max(0, i-k) <= j <= min(n-1, i+k) }
 *   skips   P(i) = { i - m*pi, i + m*pi : 1 <= m <= S, m*pi > k, 0 <= j < n }
 *   gate    z = q_i . w_g[h] + b_g[h],  alpha = sigmoid(z)        (on the unscaled query)
 *           lL = log(alpha),  lP = log(1 - alpha)                  (the log-priors)
 *   logits  s_j = tau * q_i . k_j + lL   for j in L(i)
 *           s_j = tau * q_i . k_j + lP   for j in P(i),    tau = 1/sqrt(d)
 *   one softmax over the union:  M = max_j s_j,  Z = sum_j exp(s_j - M),  p_j = exp(s_j - M) / Z
 *   out_i = sum_j p_j v_j,   lse_i = M + ln Z   (natural log)
 *
 * Inputs are read exactly as stored (fp32 as is, bf16 widened exactly) and all arithmetic is in
 * double.  Rows are independent; threads split the list of rows and never change the order of
 * any row's own sums.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_F32 = 0, OR_BF16 = 1 };

static double load_elem(const void* base, int64_t idx, int dtype) {
    if (dtype == OR_F32) return (double)((const float*)base)[idx];
    uint32_t u = (uint32_t)((const uint16_t*)base)[idx] << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* log(sigmoid(x)) without overflow: for x >= 0 it is -log(1 + e^-x); for x < 0 it is
 * x - log(1 + e^x).  Both are min(x, 0) - log1p(exp(-|x|)). */
static double log_sigmoid(double x) {
    return (x < 0 ? x : 0.0) - log1p(exp(-fabs(x)));
}

/* The index sets of query row i of a sequence of n tokens.  L ascending; P in order of
 * increasing m, and for each m the backward key before the forward one (bidir only). */
int64_t oracle_index_set_ex(int64_t i, int64_t n, int64_t kwin, int64_t pi, int64_t S, int bidir, int64_t* L,
                            int64_t* nL, int64_t* P, int64_t* nP) {
    int64_t a = i - kwin;
    if (a < 0) a = 0;
    int64_t b = i;  /* causal: the window ends at the token itself */
    if (bidir) {
        b = i + kwin;
        if (b > n - 1) b = n - 1;
    }
    int64_t c = 0;
    for (int64_t j = a; j <= b; ++j) {
        if (L) L[c] = j;
        ++c;
    }
    *nL = c;
    int64_t e = 0;
    for (int64_t m = 1; m <= S; ++m) {
        int64_t off = m * pi;
        if (off <= kwin) continue;  /* inside the window: already counted once, as a window key */
        int64_t j = i - off;
        if (j >= 0) {               /* before the sequence start: no such key */
            if (P) P[e] = j;
            ++e;
        }
        if (bidir && i + off <= n - 1) {  /* past the sequence end: no such key */
            if (P) P[e] = i + off;
            ++e;
        }
    }
    *nP = e;
    return c + e;
}

/* The causal index sets of query row i (the default operator): L ascending, P by increasing m. */
int64_t oracle_index_set(int64_t i, int64_t kwin, int64_t pi, int64_t S, int64_t* L, int64_t* nL,
                         int64_t* P, int64_t* nP) {
    return oracle_index_set_ex(i, i + 1, kwin, pi, S, 0, L, nL, P, nP);
}

/* Totals of |L(i)| and |P(i)| over i = 0..n-1, by enumeration. */
void oracle_counts_ex(int64_t n, int64_t kwin, int64_t pi, int64_t S, int bidir, int64_t* sumL, int64_t* sumP) {
    int64_t tl = 0, tp = 0;
    for (int64_t i = 0; i < n; ++i) {
        int64_t a, b;
        oracle_index_set_ex(i, n, kwin, pi, S, bidir, 0, &a, 0, &b);
        tl += a;
        tp += b;
    }
    *sumL = tl;
    *sumP = tp;
}

void oracle_counts(int64_t n, int64_t kwin, int64_t pi, int64_t S, int64_t* sumL, int64_t* sumP) {
    oracle_counts_ex(n, kwin, pi, S, 0, sumL, sumP);
}

/* Per-row index table: counts[i] = {|L(i)|, |P(i)|}; idx row i holds L(i) ascending, then P(i)
 * by increasing m, then -1 up to `width` entries. */
void oracle_index_table_ex(int64_t n, int64_t kwin, int64_t pi, int64_t S, int bidir, int64_t width,
                           int32_t* counts, int32_t* idx) {
    int64_t* L = (int64_t*)malloc(sizeof(int64_t) * (size_t)(2 * kwin + 1));
    int64_t* P = (int64_t*)malloc(sizeof(int64_t) * (size_t)(2 * S + 1));
    for (int64_t i = 0; i < n; ++i) {
        int64_t a, b;
        oracle_index_set_ex(i, n, kwin, pi, S, bidir, L, &a, P, &b);
        counts[2 * i] = (int32_t)a;
        counts[2 * i + 1] = (int32_t)b;
        int32_t* row = idx + i * width;
        int64_t w = 0;
        for (int64_t t = 0; t < a && w < width; ++t) row[w++] = (int32_t)L[t];
        for (int64_t t = 0; t < b && w < width; ++t) row[w++] = (int32_t)P[t];
        while (w < width) row[w++] = -1;
    }
    free(L);
    free(P);
}

void oracle_index_table(int64_t n, int64_t kwin, int64_t pi, int64_t S, int64_t width, int32_t* counts,
                        int32_t* idx) {
    oracle_index_table_ex(n, kwin, pi, S, 0, width, counts, idx);
}

/* One query row: q row at qbase (element offset qoff), keys/values of its (b, h) sequence at
 * kvoff (element offset of row 0), query position i.  Writes out[d], *lse, *rowsum. */
typedef struct {
    const void *q, *k, *v;
    int dtype;
    const float *w_g, *b_g;
    int64_t H, d, kwin, pi, S;
    int bidir;  /* 1: two-sided window and skips (prefill only) */
} problem_t;

static void attend_row(const problem_t* pr, int64_t h, int64_t qoff, int64_t kvoff, int64_t n, int64_t i,
                       double* out, double* lse, double* rowsum, int64_t* L, int64_t* P, double* s, double* qd) {
    const int64_t d = pr->d;
    for (int64_t c = 0; c < d; ++c) qd[c] = load_elem(pr->q, qoff + c, pr->dtype);

    /* gate on the unscaled query */
    double z = (double)pr->b_g[h];
    for (int64_t c = 0; c < d; ++c) z += qd[c] * (double)pr->w_g[h * d + c];
    const double lL = log_sigmoid(z);   /* log(alpha)     */
    const double lP = log_sigmoid(-z);  /* log(1 - alpha) */

    int64_t nL, nP;
    oracle_index_set_ex(i, n, pr->kwin, pr->pi, pr->S, pr->bidir, L, &nL, P, &nP);
    const double tau = 1.0 / sqrt((double)d);

    /* biased logits, window keys first, then skip keys */
    for (int64_t t = 0; t < nL + nP; ++t) {
        int64_t j = t < nL ? L[t] : P[t - nL];
        double dot = 0.0;
        for (int64_t c = 0; c < d; ++c) dot += qd[c] * load_elem(pr->k, kvoff + j * d + c, pr->dtype);
        s[t] = tau * dot + (t < nL ? lL : lP);
    }
    /* one softmax over the union */
    double M = -INFINITY;
    for (int64_t t = 0; t < nL + nP; ++t)
        if (s[t] > M) M = s[t];
    double Z = 0.0;
    for (int64_t t = 0; t < nL + nP; ++t) Z += exp(s[t] - M);
    for (int64_t c = 0; c < d; ++c) out[c] = 0.0;
    double ps = 0.0;
    for (int64_t t = 0; t < nL + nP; ++t) {
        int64_t j = t < nL ? L[t] : P[t - nL];
        double p = exp(s[t] - M) / Z;
        ps += p;
        for (int64_t c = 0; c < d; ++c) out[c] += p * load_elem(pr->v, kvoff + j * d + c, pr->dtype);
    }
    *lse = M + log(Z);
    *rowsum = ps;
}

typedef struct {
    const problem_t* pr;
    int64_t n;            /* rows per (b, h) sequence of k/v */
    int decode;           /* 1: q is [B, H, d]; row list holds (b*H + h); position from lengths */
    const int32_t* lengths;
    const int64_t* rows;  /* prefill: flat (b*H + h)*n + i; decode: b*H + h */
    int64_t begin, end;
    double *out, *lse, *rowsum;
} rjob_t;

static void* run_rows(void* arg) {
    rjob_t* jb = (rjob_t*)arg;
    const problem_t* pr = jb->pr;
    int64_t* L = (int64_t*)malloc(sizeof(int64_t) * (size_t)(2 * pr->kwin + 1));
    int64_t* P = (int64_t*)malloc(sizeof(int64_t) * (size_t)(2 * pr->S + 1));
    double* s = (double*)malloc(sizeof(double) * (size_t)(2 * pr->kwin + 2 * pr->S + 2));
    double* qd = (double*)malloc(sizeof(double) * (size_t)pr->d);
    for (int64_t t = jb->begin; t < jb->end; ++t) {
        int64_t r = jb->rows[t];
        int64_t bh, i, qoff;
        if (jb->decode) {
            bh = r;
            int64_t len = jb->lengths ? jb->lengths[bh / pr->H] : jb->n;
            i = len - 1;
            qoff = bh * pr->d;
        } else {
            bh = r / jb->n;
            i = r % jb->n;
            qoff = r * pr->d;
        }
        int64_t h = bh % pr->H;
        attend_row(pr, h, qoff, bh * jb->n * pr->d, jb->n, i, jb->out + t * pr->d, jb->lse + t, jb->rowsum + t, L, P,
                   s, qd);
    }
    free(L);
    free(P);
    free(s);
    free(qd);
    return 0;
}

#define MAX_THREADS 256

static void run_parallel(rjob_t* proto, int64_t total, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > MAX_THREADS) nthreads = MAX_THREADS;
    if (total < nthreads) nthreads = total > 0 ? (int)total : 1;
    pthread_t th[MAX_THREADS];
    int created[MAX_THREADS];
    rjob_t jobs[MAX_THREADS];
    int64_t chunk = (total + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = *proto;
        int64_t b = (int64_t)t * chunk, e = b + chunk;
        jobs[t].begin = b < total ? b : total;
        jobs[t].end = e < total ? e : total;
        created[t] = 0;
        if (t > 0 && jobs[t].begin < jobs[t].end) created[t] = pthread_create(&th[t], 0, run_rows, &jobs[t]) == 0;
    }
    run_rows(&jobs[0]);
    for (int t = 1; t < nthreads; ++t) {
        if (created[t]) pthread_join(th[t], 0);
        else if (jobs[t].begin < jobs[t].end) run_rows(&jobs[t]);
    }
}

/* Prefill.  q, k, v: [B, H, n, d] (dtype 0 = fp32, 1 = bf16 bit patterns); w_g [H, d], b_g [H] fp32.
 * rows: flat query rows (b*H + h)*n + i to evaluate (nrows of them).  Outputs, per listed row:
 * out [nrows, d], lse [nrows], rowsum [nrows] (sum of the probabilities, 1 up to rounding). */
void oracle_fwd_rows_ex(const void* q, const void* k, const void* v, int dtype, const float* w_g, const float* b_g,
                        int64_t B, int64_t H, int64_t n, int64_t d, int64_t kwin, int64_t pi, int64_t S, int bidir,
                        const int64_t* rows, int64_t nrows, double* out, double* lse, double* rowsum, int nthreads) {
    (void)B;
    problem_t pr = {q, k, v, dtype, w_g, b_g, H, d, kwin, pi, S, bidir};
    rjob_t jb;
    memset(&jb, 0, sizeof jb);
    jb.pr = &pr;
    jb.n = n;
    jb.rows = rows;
    jb.out = out;
    jb.lse = lse;
    jb.rowsum = rowsum;
    run_parallel(&jb, nrows, nthreads);
}

void oracle_fwd_rows(const void* q, const void* k, const void* v, int dtype, const float* w_g, const float* b_g,
                     int64_t B, int64_t H, int64_t n, int64_t d, int64_t kwin, int64_t pi, int64_t S,
                     const int64_t* rows, int64_t nrows, double* out, double* lse, double* rowsum, int nthreads) {
    oracle_fwd_rows_ex(q, k, v, dtype, w_g, b_g, B, H, n, d, kwin, pi, S, 0, rows, nrows, out, lse, rowsum, nthreads);
}

/* Decode.  q [B, H, d]; kc, vc [B, H, n_cache, d]; lengths: int32 [B] valid cache lengths (NULL
 * means every sequence holds n_cache tokens).  The query is the token at position length-1, and
 * it attends with the same rule as prefill.  bh: list of (b*H + h) to evaluate. */
void oracle_decode(const void* q, const void* kc, const void* vc, int dtype, const float* w_g, const float* b_g,
                   const int32_t* lengths, int64_t B, int64_t H, int64_t n_cache, int64_t d, int64_t kwin,
                   int64_t pi, int64_t S, const int64_t* bh, int64_t nbh, double* out, double* lse, double* rowsum,
                   int nthreads) {
    (void)B;
    /* q is read through qoff = bh*d, keys through kvoff = bh*n_cache*d */
    problem_t pr = {q, kc, vc, dtype, w_g, b_g, H, d, kwin, pi, S, 0};
    rjob_t jb;
    memset(&jb, 0, sizeof jb);
    jb.pr = &pr;
    jb.n = n_cache;
    jb.decode = 1;
    jb.lengths = lengths;
    jb.rows = bh;
    jb.out = out;
    jb.lse = lse;
    jb.rowsum = rowsum;
    run_parallel(&jb, nbh, nthreads);
}

/* Backward of one (b, h) sequence, every row, in double: accumulates dq [n, d], dk [n, d],
 * dv [n, d] (zeroed by the caller) and dw [d], db [1] of head h.  Rows in increasing order. */
static void backward_seq(const problem_t* pr, int64_t n, int64_t h, int64_t base, const double* dO, double* dq,
                         double* dk, double* dv, double* dw, double* db, double* terms) {
    const int64_t d = pr->d;
    const double tau = 1.0 / sqrt((double)d);
    int64_t* L = (int64_t*)malloc(sizeof(int64_t) * (size_t)(2 * pr->kwin + 1));
    int64_t* P = (int64_t*)malloc(sizeof(int64_t) * (size_t)(2 * pr->S + 1));
    const int64_t cap = 2 * pr->kwin + 2 * pr->S + 2;
    double* s = (double*)malloc(sizeof(double) * (size_t)cap);
    double* p = (double*)malloc(sizeof(double) * (size_t)cap);
    double* qd = (double*)malloc(sizeof(double) * (size_t)d);
    double* od = (double*)malloc(sizeof(double) * (size_t)d);
    for (int64_t i = 0; i < n; ++i) {
        const int64_t qoff = base + i * d;
        for (int64_t c = 0; c < d; ++c) qd[c] = load_elem(pr->q, qoff + c, pr->dtype);
        double z = (double)pr->b_g[h];
        for (int64_t c = 0; c < d; ++c) z += qd[c] * (double)pr->w_g[h * d + c];
        const double alpha = 1.0 / (1.0 + exp(-z));
        const double lL = log_sigmoid(z), lP = log_sigmoid(-z);
        int64_t nL, nP;
        oracle_index_set_ex(i, n, pr->kwin, pr->pi, pr->S, pr->bidir, L, &nL, P, &nP);
        const int64_t nU = nL + nP;
        /* forward of the row: logits, probabilities, output */
        for (int64_t t = 0; t < nU; ++t) {
            const int64_t j = t < nL ? L[t] : P[t - nL];
            double dot = 0.0;
            for (int64_t c = 0; c < d; ++c) dot += qd[c] * load_elem(pr->k, base + j * d + c, pr->dtype);
            s[t] = tau * dot + (t < nL ? lL : lP);
        }
        double M = -INFINITY;
        for (int64_t t = 0; t < nU; ++t)
            if (s[t] > M) M = s[t];
        double Z = 0.0;
        for (int64_t t = 0; t < nU; ++t) Z += exp(s[t] - M);
        for (int64_t c = 0; c < d; ++c) od[c] = 0.0;
        for (int64_t t = 0; t < nU; ++t) {
            const int64_t j = t < nL ? L[t] : P[t - nL];
            p[t] = exp(s[t] - M) / Z;
            for (int64_t c = 0; c < d; ++c) od[c] += p[t] * load_elem(pr->v, base + j * d + c, pr->dtype);
        }
        /* backward of the row */
        const double* g = dO + i * d;
        double Dsum = 0.0;
        for (int64_t c = 0; c < d; ++c) Dsum += g[c] * od[c];
        double dz = 0.0, sig2 = 0.0;
        for (int64_t t = 0; t < nU; ++t) {
            const int64_t j = t < nL ? L[t] : P[t - nL];
            double dpt = 0.0;
            for (int64_t c = 0; c < d; ++c) dpt += g[c] * load_elem(pr->v, base + j * d + c, pr->dtype);
            const double ds = p[t] * (dpt - Dsum);
            dz += t < nL ? (1.0 - alpha) * ds : -alpha * ds;
            sig2 += p[t] * p[t] * dpt * dpt;
            for (int64_t c = 0; c < d; ++c) {
                dq[i * d + c] += tau * ds * load_elem(pr->k, base + j * d + c, pr->dtype);
                dk[j * d + c] += tau * ds * qd[c];
                dv[j * d + c] += p[t] * g[c];
            }
        }
        for (int64_t c = 0; c < d; ++c) {
            dq[i * d + c] += dz * (double)pr->w_g[h * d + c];
            dw[c] += dz * qd[c];
        }
        *db += dz;
        if (terms) {
            terms[3 * i] = dz;
            terms[3 * i + 1] = Dsum;
            terms[3 * i + 2] = sig2;
        }
    }
    free(L);
    free(P);
    free(s);
    free(p);
    free(qd);
    free(od);
}

typedef struct {
    const problem_t* pr;
    int64_t n;
    const double* dO;
    double *dq, *dk, *dv, *dw_part, *db_part;  /* dw_part [B*H, d], db_part [B*H] */
    double* terms;                             /* [B*H, n, 3] or NULL */
    int64_t begin, end;                        /* (b, h) range */
} bjob_t;

static void* run_backward(void* arg) {
    bjob_t* jb = (bjob_t*)arg;
    const problem_t* pr = jb->pr;
    const int64_t n = jb->n, d = pr->d;
    for (int64_t bh = jb->begin; bh < jb->end; ++bh) {
        const int64_t off = bh * n * d;
        backward_seq(pr, n, bh % pr->H, off, jb->dO + off, jb->dq + off, jb->dk + off, jb->dv + off,
                     jb->dw_part + bh * d, jb->db_part + bh, jb->terms ? jb->terms + bh * n * 3 : 0);
    }
    return 0;
}

/* Backward.  q, k, v [B, H, n, d] as for oracle_fwd_rows_ex; dO [B, H, n, d] double.  Outputs, all
 * double and written whole: dq, dk, dv [B, H, n, d], dw_g [H, d], db_g [H] (sums over b and i,
 * added in increasing b); with terms non-NULL also, per row, [B, H, n, 3]: the row's dz_i (its
 * term in db_g), D_i = dO_i . out_i and sum_j p_j^2 (dO_i . v_j)^2 (the spread of the terms D_i is
 * summed from).  Threads split the (b, h) sequences. */
void oracle_bwd(const void* q, const void* k, const void* v, int dtype, const float* w_g, const float* b_g, int64_t B,
                int64_t H, int64_t n, int64_t d, int64_t kwin, int64_t pi, int64_t S, int bidir, const double* dO,
                double* dq, double* dk, double* dv, double* dw_g, double* db_g, double* terms, int nthreads) {
    problem_t pr = {q, k, v, dtype, w_g, b_g, H, d, kwin, pi, S, bidir};
    const int64_t BH = B * H;
    memset(dq, 0, sizeof(double) * (size_t)(BH * n * d));
    memset(dk, 0, sizeof(double) * (size_t)(BH * n * d));
    memset(dv, 0, sizeof(double) * (size_t)(BH * n * d));
    double* dw_part = (double*)calloc((size_t)(BH * d), sizeof(double));
    double* db_part = (double*)calloc((size_t)BH, sizeof(double));
    if (nthreads < 1) nthreads = 1;
    if (nthreads > MAX_THREADS) nthreads = MAX_THREADS;
    if (BH < nthreads) nthreads = (int)BH;
    pthread_t th[MAX_THREADS];
    int created[MAX_THREADS];
    bjob_t jobs[MAX_THREADS];
    const int64_t chunk = (BH + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; ++t) {
        bjob_t jb = {&pr, n, dO, dq, dk, dv, dw_part, db_part, terms, 0, 0};
        jb.begin = (int64_t)t * chunk < BH ? (int64_t)t * chunk : BH;
        jb.end = jb.begin + chunk < BH ? jb.begin + chunk : BH;
        jobs[t] = jb;
        created[t] = 0;
        if (t > 0 && jobs[t].begin < jobs[t].end) created[t] = pthread_create(&th[t], 0, run_backward, &jobs[t]) == 0;
    }
    run_backward(&jobs[0]);
    for (int t = 1; t < nthreads; ++t) {
        if (created[t]) pthread_join(th[t], 0);
        else if (jobs[t].begin < jobs[t].end) run_backward(&jobs[t]);
    }
    memset(dw_g, 0, sizeof(double) * (size_t)(H * d));
    memset(db_g, 0, sizeof(double) * (size_t)H);
    for (int64_t bh = 0; bh < BH; ++bh) {
        const int64_t h = bh % H;
        for (int64_t c = 0; c < d; ++c) dw_g[h * d + c] += dw_part[bh * d + c];
        db_g[h] += db_part[bh];
    }
    free(dw_part);
    free(db_part);
}
