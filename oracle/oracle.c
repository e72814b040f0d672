/*
 * oracle.c -- fp64 CPU oracle for causal / non-causal scaled-dot-product
 * attention and its gradients.  TEST INFRASTRUCTURE ONLY: nothing in the
 * product library (long_sequence_context_b200/) links, includes or calls this
 * file.  Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline /
 * reference arm load it.
 *
 * Source of the method: "Configuring RingAttention+FlashAttention for CP"
 * (devpress.csdn.net), section 1: every rank's Q takes turns against the K/V
 * blocks of all ranks and the results are combined, which must equal ordinary
 * attention over the whole sequence; section 3, note 2: the mask must be exact
 * so that no position sees a later one.  "Megatron-LM source analysis: Context
 * Parallel" (mieleap.com), section 3: causal attention with FlashAttention
 * semantics.  The pages never write the formulas down, so the functions below
 * are the plain textbook definitions:
 *
 *   allowed set   A_i = { j <= i } (causal)   or all j (non-causal)
 *   score         s_ij = scale * sum_d q_id k_jd
 *   log-sum-exp   LSE_i = log sum_{j in A_i} exp(s_ij)   (natural log)
 *   probability   P_ij = exp(s_ij - LSE_i)
 *   output        O_i  = sum_j P_ij v_j
 *
 * and the gradient of the scalar L = sum_i dO_i . O_i:
 *
 *   dV_j = sum_i P_ij dO_i            dP_ij = dO_i . v_j
 *   delta_i = sum_j P_ij dP_ij        dS_ij = P_ij (dP_ij - delta_i)
 *   dQ_i = scale sum_j dS_ij k_j      dK_j = scale sum_i dS_ij q_i
 *
 * The ring restatement (oracle_ring_fwd) follows the same pages' ring and
 * zigzag rules step by step: ranks own chunks {r, 2N-1-r} (section 5, item 1),
 * step t reads the K/V of rank (r - t) mod N (section 3 code), and blocks are
 * FULL / DIAG / SKIP by the exact causal mask (section 3, note 2).  Partials
 * are combined with the log-sum-exp merge, which the pages leave unwritten
 * (their listing simply adds outputs); the merge is the identity
 *   L = log(exp(La) + exp(Lb)),  O = exp(La - L) Oa + exp(Lb - L) Ob.
 *
 * Layout: one (batch, head) slice at a time, row-major [S][D] fp64.
 * No blocking, no reordering: loops in the order of the definitions above.
 * Parallelism: OpenMP over independent rows (or key columns).
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double dot(const double* a, const double* b, long D) {
    double acc = 0.0;
    for (long d = 0; d < D; ++d) acc += a[d] * b[d];
    return acc;
}

/* number of keys row i may see */
static long n_allowed(long i, long S, int causal) { return causal ? i + 1 : S; }

/* LSE_i and (optionally) O_i for one row; s is scratch of length S. */
static void row_forward(const double* q, const double* k, const double* v, long S, long D,
                        int causal, double scale, long i, double* s, double* o_row,
                        double* lse_out) {
    long n = n_allowed(i, S, causal);
    double m = -INFINITY;
    for (long j = 0; j < n; ++j) {
        s[j] = scale * dot(q + i * D, k + j * D, D);
        if (s[j] > m) m = s[j];
    }
    double sum = 0.0;
    for (long j = 0; j < n; ++j) sum += exp(s[j] - m);
    double lse = m + log(sum);
    if (lse_out) *lse_out = lse;
    if (o_row) {
        for (long d = 0; d < D; ++d) o_row[d] = 0.0;
        for (long j = 0; j < n; ++j) {
            double p = exp(s[j] - lse);
            for (long d = 0; d < D; ++d) o_row[d] += p * v[j * D + d];
        }
    }
}

int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Full forward: o [S][D], lse [S]. */
int oracle_attn_fwd(const double* q, const double* k, const double* v, long S, long D,
                    int causal, double scale, double* o, double* lse) {
    if (S < 0 || D <= 0) return 1;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (S > 0 ? S : 1));
#pragma omp for schedule(dynamic, 16)
        for (long i = 0; i < S; ++i) row_forward(q, k, v, S, D, causal, scale, i, s, o + i * D, lse + i);
        free(s);
    }
    return 0;
}

/* Forward for selected rows only: o_rows [n_rows][D], lse_rows [n_rows]. */
int oracle_attn_fwd_rows(const double* q, const double* k, const double* v, long S, long D,
                         int causal, double scale, const long* rows, long n_rows,
                         double* o_rows, double* lse_rows) {
    for (long r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= S) return 1;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (S > 0 ? S : 1));
#pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < n_rows; ++r)
            row_forward(q, k, v, S, D, causal, scale, rows[r], s, o_rows + r * D, lse_rows + r);
        free(s);
    }
    return 0;
}

/* Row pass of the backward for row i: LSE_i, delta_i and dQ_i.
 * delta_i is taken from the oracle's own P (sum_j P_ij dP_ij). */
static void row_backward(const double* q, const double* k, const double* v, const double* dout,
                         long S, long D, int causal, double scale, long i, double* s,
                         double* lse_out, double* delta_out, double* dq_row) {
    long n = n_allowed(i, S, causal);
    double lse;
    row_forward(q, k, v, S, D, causal, scale, i, s, NULL, &lse);
    /* s[j] now holds the scores of row i */
    double delta = 0.0;
    for (long j = 0; j < n; ++j) {
        double p = exp(s[j] - lse);
        double dp = dot(dout + i * D, v + j * D, D);
        delta += p * dp;
    }
    if (dq_row) {
        for (long d = 0; d < D; ++d) dq_row[d] = 0.0;
        for (long j = 0; j < n; ++j) {
            double p = exp(s[j] - lse);
            double dp = dot(dout + i * D, v + j * D, D);
            double ds = p * (dp - delta);
            for (long d = 0; d < D; ++d) dq_row[d] += scale * ds * k[j * D + d];
        }
    }
    if (lse_out) *lse_out = lse;
    if (delta_out) *delta_out = delta;
}

/* Column pass for key j given every row's LSE and delta. */
static void col_backward(const double* q, const double* k, const double* v, const double* dout,
                         long S, long D, int causal, double scale, long j, const double* lse,
                         const double* delta, double* dk_row, double* dv_row) {
    for (long d = 0; d < D; ++d) { dk_row[d] = 0.0; dv_row[d] = 0.0; }
    long i0 = causal ? j : 0;
    for (long i = i0; i < S; ++i) {
        double sij = scale * dot(q + i * D, k + j * D, D);
        double p = exp(sij - lse[i]);
        double dp = dot(dout + i * D, v + j * D, D);
        double ds = p * (dp - delta[i]);
        for (long d = 0; d < D; ++d) {
            dv_row[d] += p * dout[i * D + d];
            dk_row[d] += scale * ds * q[i * D + d];
        }
    }
}

/* Full backward: dq, dk, dv [S][D].  Two passes: rows (LSE, delta, dQ), then
 * key columns (dK, dV).  Each pass follows the definitions directly. */
int oracle_attn_bwd(const double* q, const double* k, const double* v, const double* dout,
                    long S, long D, int causal, double scale, double* dq, double* dk,
                    double* dv) {
    if (S < 0 || D <= 0) return 1;
    double* lse = (double*)malloc(sizeof(double) * (S > 0 ? S : 1));
    double* delta = (double*)malloc(sizeof(double) * (S > 0 ? S : 1));
    if (!lse || !delta) { free(lse); free(delta); return 2; }
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (S > 0 ? S : 1));
#pragma omp for schedule(dynamic, 16)
        for (long i = 0; i < S; ++i)
            row_backward(q, k, v, dout, S, D, causal, scale, i, s, lse + i, delta + i, dq + i * D);
        free(s);
    }
#pragma omp parallel for schedule(dynamic, 16)
    for (long j = 0; j < S; ++j)
        col_backward(q, k, v, dout, S, D, causal, scale, j, lse, delta, dk + j * D, dv + j * D);
    free(lse);
    free(delta);
    return 0;
}

/* dQ for selected rows only. */
int oracle_attn_bwd_dq_rows(const double* q, const double* k, const double* v,
                            const double* dout, long S, long D, int causal, double scale,
                            const long* rows, long n_rows, double* dq_rows) {
    for (long r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= S) return 1;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (S > 0 ? S : 1));
#pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < n_rows; ++r)
            row_backward(q, k, v, dout, S, D, causal, scale, rows[r], s, NULL, NULL,
                         dq_rows + r * D);
        free(s);
    }
    return 0;
}

/* dK and dV for selected key columns.  Only the rows that can see one of the
 * requested keys need their LSE and delta; for a causal mask those are the
 * rows at or after the smallest requested key. */
int oracle_attn_bwd_kv_cols(const double* q, const double* k, const double* v,
                            const double* dout, long S, long D, int causal, double scale,
                            const long* cols, long n_cols, double* dk_cols, double* dv_cols) {
    long jmin = S;
    for (long c = 0; c < n_cols; ++c) {
        if (cols[c] < 0 || cols[c] >= S) return 1;
        if (cols[c] < jmin) jmin = cols[c];
    }
    if (n_cols == 0) return 0;
    long i0 = causal ? jmin : 0;
    double* lse = (double*)malloc(sizeof(double) * S);
    double* delta = (double*)malloc(sizeof(double) * S);
    if (!lse || !delta) { free(lse); free(delta); return 2; }
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * S);
#pragma omp for schedule(dynamic, 4)
        for (long i = i0; i < S; ++i)
            row_backward(q, k, v, dout, S, D, causal, scale, i, s, lse + i, delta + i, NULL);
        free(s);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (long c = 0; c < n_cols; ++c)
        col_backward(q, k, v, dout, S, D, causal, scale, cols[c], lse, delta, dk_cols + c * D,
                     dv_cols + c * D);
    free(lse);
    free(delta);
    return 0;
}

/* ---------------------------------------------------------------------------
 * Ring restatement.  Virtual ranks r = 0..N-1.
 *   causal:     the sequence is cut into 2N chunks of length c = S / 2N and
 *               rank r owns chunks r and 2N-1-r (zigzag).
 *   non-causal: N contiguous chunks of length c = S / N, rank r owns chunk r.
 * At ring step t (t = 0..N-1) rank r holds the K/V of rank src = (r - t) mod N.
 * A (q chunk a, kv chunk b) block is SKIP when a < b (causal), DIAG when
 * a == b (mask j <= i inside it), FULL otherwise (and always FULL when
 * non-causal).  Each non-SKIP block yields a partial (O, LSE) for every row of
 * chunk a; partials are merged in ring order with the log-sum-exp rule.
 * ------------------------------------------------------------------------- */
static void merge_into(double* o_acc, double* lse_acc, const double* o_part, double lse_part,
                       long D) {
    if (lse_part == -INFINITY) return; /* empty partial: nothing to add */
    if (*lse_acc == -INFINITY) {       /* empty accumulator: take the partial */
        for (long d = 0; d < D; ++d) o_acc[d] = o_part[d];
        *lse_acc = lse_part;
        return;
    }
    double m = *lse_acc > lse_part ? *lse_acc : lse_part;
    double lse_new = m + log(exp(*lse_acc - m) + exp(lse_part - m));
    double wa = exp(*lse_acc - lse_new), wb = exp(lse_part - lse_new);
    for (long d = 0; d < D; ++d) o_acc[d] = wa * o_acc[d] + wb * o_part[d];
    *lse_acc = lse_new;
}

/* partial attention of global row i against keys [b0, b1) (restricted to
 * j <= i when diag): normalised O and its LSE; LSE = -inf when empty. */
static void block_partial(const double* q, const double* k, const double* v, long D,
                          double scale, long i, long b0, long b1, int diag, double* s,
                          double* o_part, double* lse_part) {
    long e = b1;
    if (diag && i + 1 < e) e = i + 1;
    for (long d = 0; d < D; ++d) o_part[d] = 0.0;
    if (e <= b0) { *lse_part = -INFINITY; return; }
    double m = -INFINITY;
    for (long j = b0; j < e; ++j) {
        s[j - b0] = scale * dot(q + i * D, k + j * D, D);
        if (s[j - b0] > m) m = s[j - b0];
    }
    double sum = 0.0;
    for (long j = b0; j < e; ++j) sum += exp(s[j - b0] - m);
    double lse = m + log(sum);
    for (long j = b0; j < e; ++j) {
        double p = exp(s[j - b0] - lse);
        for (long d = 0; d < D; ++d) o_part[d] += p * v[j * D + d];
    }
    *lse_part = lse;
}

int oracle_ring_fwd(const double* q, const double* k, const double* v, long S, long D,
                    int cp_size, int causal, double scale, double* o, double* lse) {
    long N = cp_size;
    if (N < 1) return 1;
    long n_chunks = causal ? 2 * N : N;
    if (S % n_chunks != 0) return 2;
    long c = S / n_chunks;
    for (long i = 0; i < S; ++i) {
        lse[i] = -INFINITY;
        for (long d = 0; d < D; ++d) o[i * D + d] = 0.0;
    }
    for (long r = 0; r < N; ++r) {
        long own[2];
        int n_own = 0;
        own[n_own++] = r;
        if (causal) own[n_own++] = 2 * N - 1 - r;
        for (int oa = 0; oa < n_own; ++oa) {
            long a = own[oa];
#pragma omp parallel
            {
                double* s = (double*)malloc(sizeof(double) * (c > 0 ? c : 1));
                double* o_part = (double*)malloc(sizeof(double) * D);
#pragma omp for schedule(static)
                for (long i = a * c; i < (a + 1) * c; ++i) {
                    for (long t = 0; t < N; ++t) {
                        long src = ((r - t) % N + N) % N;
                        long kv[2];
                        int n_kv = 0;
                        kv[n_kv++] = src;
                        if (causal) kv[n_kv++] = 2 * N - 1 - src;
                        for (int ob = 0; ob < n_kv; ++ob) {
                            long b = kv[ob];
                            if (causal && a < b) continue; /* SKIP */
                            int diag = causal && a == b;
                            double lp;
                            block_partial(q, k, v, D, scale, i, b * c, (b + 1) * c, diag, s,
                                          o_part, &lp);
                            merge_into(o + i * D, lse + i, o_part, lp, D);
                        }
                    }
                }
                free(s);
                free(o_part);
            }
        }
    }
    return 0;
}

/* The standalone merge rule on arrays: rows x D, in place on (o_acc, lse_acc). */
int oracle_merge(double* o_acc, double* lse_acc, const double* o_part, const double* lse_part,
                 long rows, long D) {
    for (long i = 0; i < rows; ++i) merge_into(o_acc + i * D, lse_acc + i, o_part + i * D, lse_part[i], D);
    return 0;
}

/* One ring step for every row: rank r(i) owning the chunk of row i reads the
 * K/V of rank src = (r - t) mod N; the partial of row i merges the (at most
 * two) non-SKIP blocks of that K/V.  Rows whose blocks are all SKIP get
 * O = 0 and LSE = -inf. */
int oracle_ring_step(const double* q, const double* k, const double* v, long S, long D,
                     int cp_size, int causal, double scale, int step, double* o_part,
                     double* lse_part) {
    long N = cp_size;
    if (N < 1 || step < 0 || step >= N) return 1;
    long n_chunks = causal ? 2 * N : N;
    if (S % n_chunks != 0) return 2;
    long c = S / n_chunks;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (c > 0 ? c : 1));
        double* tmp = (double*)malloc(sizeof(double) * D);
#pragma omp for schedule(static)
        for (long i = 0; i < S; ++i) {
            long a = i / c;
            long r = (causal && a >= N) ? 2 * N - 1 - a : a; /* owner of chunk a */
            long src = ((r - step) % N + N) % N;
            long kv[2];
            int n_kv = 0;
            kv[n_kv++] = src;
            if (causal) kv[n_kv++] = 2 * N - 1 - src;
            lse_part[i] = -INFINITY;
            for (long d = 0; d < D; ++d) o_part[i * D + d] = 0.0;
            for (int ob = 0; ob < n_kv; ++ob) {
                long b = kv[ob];
                if (causal && a < b) continue;
                int diag = causal && a == b;
                double lp;
                block_partial(q, k, v, D, scale, i, b * c, (b + 1) * c, diag, s, tmp, &lp);
                merge_into(o_part + i * D, lse_part + i, tmp, lp, D);
            }
        }
        free(s);
        free(tmp);
    }
    return 0;
}
