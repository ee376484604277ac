/*
 * kpa_oracle.c -- plain, slow float64 CPU oracle for factor-space
 * Kronecker Product Attention (KPA) and its degenerate split, Tensor Product
 * Attention (TPA).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or helper with the
 * CUDA library.
 *
 * What it computes is the plain definition of the method, written out with no
 * blocking, fusion or reordering:
 *   - the Kronecker product of Definition 2.1 and the normalised factor sums of
 *     eqs (2)-(4) ("Kronecker Product Attention", section 2.2);
 *   - Kronecker-Separable RoPE, I_{d1} (x) R_theta^(2)(t), Definition 2.3
 *     (same paper, section 2.4), applied to the RECONSTRUCTED query and key rows;
 *   - scaled dot-product softmax attention ("Tensor Product Attention Is All
 *     You Need", attention background section; the explainer's "Scaled
 *     Dot-Product Attention" component), scale 1/sqrt(d_h) by default
 *     (KPA paper, section 2.3, remark before Proposition 2.2);
 *   - the merged factor projection of eq (5) (KPA paper, section 2.2).
 *
 * Readings of points the pages leave open (each is listed in the design notes):
 *   - RoPE pairs are adjacent features (2m, 2m+1) inside each length-d2 chunk,
 *     theta_m = base^(-2m/d2) for m = 0 .. d2/2-1, and a pair (x0, x1) turns
 *     into (x0 cos phi - x1 sin phi, x0 sin phi + x1 cos phi), phi = pos*theta_m.
 *   - Head (i1, i2) is row i1*h2 + i2 of A (x) B and feature (j1, j2) is column
 *     j1*d2 + j2, the block order of Definition 2.1.
 *   - A token's factor record is [A_0 .. A_{R-1} | B_0 .. B_{R-1}], each A_r
 *     row-major h1 x d1 and each B_r row-major h2 x d2 (rank-major reshape of
 *     the merged projection, eq (5)).
 *   - The merged projection's output columns are ordered
 *     [A^Q | B^Q | A^K | B^K | A^V | B^V].  The pages fix no order: this one is a
 *     convention, and parity for it is unpinned beyond self-consistency.
 *   - Cache slot s holds the token at position s.  A query row sees the slots
 *     0 .. n_keys-1 that it is given (decode: the sequence length; causal
 *     prefill: start + t + 1).
 *   - A row with no visible slot attends to nothing and yields zeros.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_abi_version(void) { return 1; }

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
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

/* Definition 2.1: (A (x) B)[i1*m2 + i2][j1*n2 + j2] = A[i1][j1] * B[i2][j2],
 * A is m1 x n1 and B is m2 x n2, both row-major. */
void oracle_kron(int m1, int n1, const double *A, int m2, int n2, const double *B,
                 double *out)
{
    const int cols = n1 * n2;
    for (int i1 = 0; i1 < m1; ++i1)
        for (int i2 = 0; i2 < m2; ++i2)
            for (int j1 = 0; j1 < n1; ++j1)
                for (int j2 = 0; j2 < n2; ++j2)
                    out[(i1 * m2 + i2) * cols + j1 * n2 + j2] =
                        A[i1 * n1 + j1] * B[i2 * n2 + j2];
}

/* Row `row` (= i1*h2 + i2) of X = (1/R) sum_r A_r (x) B_r, eqs (3)-(4).
 * rec = [A_0 .. A_{R-1} | B_0 .. B_{R-1}]; out has d1*d2 entries. */
void oracle_kron_sum_row(int h1, int h2, int d1, int d2, int R, const double *rec,
                         int row, double *out)
{
    const int i1 = row / h2, i2 = row % h2;
    const double *A = rec;                  /* R blocks of h1*d1 */
    const double *B = rec + (size_t)R * h1 * d1; /* R blocks of h2*d2 */
    for (int j1 = 0; j1 < d1; ++j1)
        for (int j2 = 0; j2 < d2; ++j2) {
            double acc = 0.0;
            for (int r = 0; r < R; ++r)
                acc += A[(size_t)r * h1 * d1 + i1 * d1 + j1] *
                       B[(size_t)r * h2 * d2 + i2 * d2 + j2];
            out[j1 * d2 + j2] = acc / (double)R;
        }
}

/* The whole h x d_h matrix X = (1/R) sum_r A_r (x) B_r, eqs (2)-(4). */
void oracle_reconstruct(int h1, int h2, int d1, int d2, int R, const double *rec,
                        double *X)
{
    const int h = h1 * h2, dh = d1 * d2;
    for (int row = 0; row < h; ++row)
        oracle_kron_sum_row(h1, h2, d1, d2, R, rec, row, X + (size_t)row * dh);
}

/* R_theta^(2)(pos) acting on one length-d2 vector (Definition 2.3 with the
 * pairing and sign readings above). */
void oracle_rope_d2(int d2, double base, double pos, double *v)
{
    for (int m = 0; m < d2 / 2; ++m) {
        const double theta = pow(base, -2.0 * (double)m / (double)d2);
        const double phi = pos * theta;
        const double c = cos(phi), s = sin(phi);
        const double x0 = v[2 * m], x1 = v[2 * m + 1];
        v[2 * m] = x0 * c - x1 * s;
        v[2 * m + 1] = x0 * s + x1 * c;
    }
}

/* Definition 2.3: R_KPA(pos) = I_{d1} (x) R_theta^(2)(pos) on a d1*d2 vector,
 * i.e. the same d2-rotation applied to each of the d1 contiguous chunks. */
void oracle_rope_kpa(int d1, int d2, double base, double pos, double *v)
{
    for (int j1 = 0; j1 < d1; ++j1)
        oracle_rope_d2(d2, base, pos, v + (size_t)j1 * d2);
}

/* Theorem 2.4, right-hand side: rotate only the B factors of one token's
 * record (each of the R*h2 rows of length d2) by R_theta^(2)(pos). */
void oracle_rotate_record(int h1, int h2, int d1, int d2, int R, double base,
                          double pos, double *rec)
{
    double *B = rec + (size_t)R * h1 * d1;
    for (int r = 0; r < R; ++r)
        for (int i2 = 0; i2 < h2; ++i2)
            oracle_rope_d2(d2, base, pos, B + ((size_t)r * h2 + i2) * d2);
}

/* eq (5) with the ranks merged: factors[t][n] = sum_k W[n][k] * x[t][k]. */
void oracle_project(int n_tok, int d_model, int n_out, const double *x,
                    const double *W, double *factors)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < n_tok; ++t)
        for (int n = 0; n < n_out; ++n) {
            double acc = 0.0;
            for (int k = 0; k < d_model; ++k)
                acc += W[(size_t)n * d_model + k] * x[(size_t)t * d_model + k];
            factors[(size_t)t * n_out + n] = acc;
        }
}

/*
 * Softmax attention over factor-cache slots, the plain definition.
 *
 *  q        [batch][n_q][h][dh]  query rows (unrotated when q_pos != NULL)
 *  q_pos    [batch][n_q]         position of each query row, or NULL when the
 *                                rows are already rotated
 *  kf, vf   [batch][cap][E]      factor records, E = R*(h1*d1 + h2*d2); kf is
 *                                unrotated unless keys_rotated != 0
 *  n_keys   [batch][n_q]         query row (b, t) sees slots 0 .. n_keys-1
 *  out      [batch][n_q][h][dh]
 *  heads    optional list of n_heads flat (b*h + head) indices to compute;
 *           NULL computes all.  Rows of skipped heads are left untouched.
 *  lse      optional [batch][n_q][h]: the softmax normaliser of each row,
 *           ln sum_s exp(score_s) (-inf with no visible slot); NULL skips it.
 *
 * For each (b, head, t): k_s = row `head` of (1/R_K) sum_r A^K_r(s) (x) B^K_r(s)
 * rotated by R_KPA(s); q rotated by R_KPA(q_pos); score_s = sm_scale * q.k_s;
 * p = softmax(score) (max-subtracted); out = sum_s p_s v_s with v_s the same
 * row of (1/R_V) sum_r A^V_r(s) (x) B^V_r(s).  Returns 0, or -1 on a bad size
 * or an allocation failure.
 */
int oracle_attend(int h1, int h2, int d1, int d2, int r_k, int r_v, double rope_base,
                  int batch, int n_q, const double *q, const int64_t *q_pos,
                  const double *kf, const double *vf, int cap, const int32_t *n_keys,
                  int keys_rotated, double sm_scale, double *out,
                  int n_heads, const int32_t *heads, double *lse)
{
    const int h = h1 * h2, dh = d1 * d2;
    const int ek = r_k * (h1 * d1 + h2 * d2), ev = r_v * (h1 * d1 + h2 * d2);
    if (h <= 0 || dh <= 0 || r_k <= 0 || r_v <= 0 || batch < 0 || n_q < 0 || cap < 0)
        return -1;
    if (d2 % 2 != 0 && (q_pos || !keys_rotated)) return -1;   /* RoPE pairs, when it rotates */
    const int total = heads ? n_heads : batch * h;
    int failed = 0;

#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
    for (int task = 0; task < total; ++task) {
        const int flat = heads ? heads[task] : task;
        const int b = flat / h, head = flat % h;
        if (b < 0 || b >= batch) { failed |= 1; continue; }
        int max_keys = 0;
        for (int t = 0; t < n_q; ++t) {
            int nk = n_keys[(size_t)b * n_q + t];
            if (nk > cap) { failed |= 1; nk = cap; }
            if (nk > max_keys) max_keys = nk;
        }
        double *krow = (double *)malloc(sizeof(double) * (size_t)dh);
        double *qrot = (double *)malloc(sizeof(double) * ((size_t)n_q * dh + 1));
        double *scores = (double *)malloc(sizeof(double) * ((size_t)max_keys * n_q + 1));
        if (!krow || !qrot || !scores) {
            failed |= 1;
            free(krow); free(qrot); free(scores);
            continue;
        }
        /* the query rows of this head, rotated by R_KPA(q_pos) when asked */
        for (int t = 0; t < n_q; ++t) {
            double *qr = qrot + (size_t)t * dh;
            memcpy(qr, q + (((size_t)b * n_q + t) * h + head) * dh, sizeof(double) * (size_t)dh);
            if (q_pos) oracle_rope_kpa(d1, d2, rope_base, (double)q_pos[(size_t)b * n_q + t], qr);
        }
        /* pass 1: scores[t][s] for every visible slot */
        for (int s = 0; s < max_keys; ++s) {
            oracle_kron_sum_row(h1, h2, d1, d2, r_k, kf + ((size_t)b * cap + s) * ek,
                                head, krow);
            if (!keys_rotated) oracle_rope_kpa(d1, d2, rope_base, (double)s, krow);
            for (int t = 0; t < n_q; ++t) {
                if (s >= n_keys[(size_t)b * n_q + t]) continue;
                const double *qr = qrot + (size_t)t * dh;
                double dot = 0.0;
                for (int j = 0; j < dh; ++j) dot += qr[j] * krow[j];
                scores[(size_t)t * max_keys + s] = sm_scale * dot;
            }
        }
        /* softmax over each row's visible slots */
        for (int t = 0; t < n_q; ++t) {
            const int nk = n_keys[(size_t)b * n_q + t] < cap ? n_keys[(size_t)b * n_q + t] : cap;
            double *row = scores + (size_t)t * max_keys;
            double *lrow = lse ? lse + ((size_t)b * n_q + t) * h + head : NULL;
            if (nk <= 0) {
                if (lrow) *lrow = -INFINITY;
                continue;
            }
            double mx = row[0];
            for (int s = 1; s < nk; ++s) if (row[s] > mx) mx = row[s];
            double sum = 0.0;
            for (int s = 0; s < nk; ++s) { row[s] = exp(row[s] - mx); sum += row[s]; }
            for (int s = 0; s < nk; ++s) row[s] /= sum;
            if (lrow) *lrow = mx + log(sum);
        }
        /* pass 2: out[t] = sum_s p[t][s] v_s */
        for (int t = 0; t < n_q; ++t) {
            double *o = out + (((size_t)b * n_q + t) * h + head) * dh;
            for (int j = 0; j < dh; ++j) o[j] = 0.0;
        }
        for (int s = 0; s < max_keys; ++s) {
            oracle_kron_sum_row(h1, h2, d1, d2, r_v, vf + ((size_t)b * cap + s) * ev,
                                head, krow);
            for (int t = 0; t < n_q; ++t) {
                if (s >= n_keys[(size_t)b * n_q + t]) continue;
                const double p = scores[(size_t)t * max_keys + s];
                double *o = out + (((size_t)b * n_q + t) * h + head) * dh;
                for (int j = 0; j < dh; ++j) o[j] += p * krow[j];
            }
        }
        free(krow); free(qrot); free(scores);
    }
    return failed ? -1 : 0;
}

/* eq (10)/(11): cached numbers per token, (R_K + R_V)(h1 d1 + h2 d2), and the
 * MHA count 2 h1 h2 d1 d2 it is compared with. */
int64_t oracle_cache_numbers_per_token(int h1, int h2, int d1, int d2, int r_k, int r_v)
{
    return (int64_t)(r_k + r_v) * ((int64_t)h1 * d1 + (int64_t)h2 * d2);
}

int64_t oracle_mha_numbers_per_token(int h1, int h2, int d1, int d2)
{
    return (int64_t)2 * h1 * h2 * d1 * d2;
}

double oracle_compression(int h1, int h2, int d1, int d2, int r_k, int r_v)
{
    return (double)oracle_mha_numbers_per_token(h1, h2, d1, d2) /
           (double)oracle_cache_numbers_per_token(h1, h2, d1, d2, r_k, r_v);
}
