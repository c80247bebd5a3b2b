/*
 * Reference oracle for Looped Latent Attention decode and encode.
 *
 * TEST INFRASTRUCTURE. This file exists to check the CUDA library, never to
 * stand in for it. Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg may load it. It shares no code, header or table with the
 * CUDA path.
 *
 * Source: "Looped Latent Attention: Cross-Loop KV Compression for Looped
 * Transformers" (O'Neill & Reid, arXiv 2607.15456).
 *   - §3 "Teacher cache", Eq. 1: the per-loop vectors of one (token, layer,
 *     head, axis) are stacked loop-major, x = [x_1; ...; x_T].
 *   - §3 "Cross-loop codec", Eq. 2: latent c = (x - mu) W_down.
 *   - §3 Eq. 3: loop t is read back as xhat_t = c W_up,t^T + mu_t.
 *   - §3 "The LLA-2D variant": one latent per token and layer, decoded into
 *     every head.
 *   - §7 "Per-head LLA versus LLA-2D at inference": the bilinear identities
 *     q^T (W_up c) = (W_up^T q)^T c and sum_i a_i W_up^V c_i =
 *     W_up^V sum_i a_i c_i (the absorbed form).
 *
 * Everything is double precision. Matrices are row-major and dense. The
 * decode oracle is the plain definition: rebuild every cached K and V
 * vector explicitly (Eq. 3), then run textbook softmax attention over them.
 * The absorbed variant exists only so the tests can check the identity of
 * §7 against the explicit path by brute force.
 *
 * Softmax scale: the pages do not state it; the caller passes it (the usual
 * 1/sqrt(d_head)).
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Textbook scaled-dot-product attention of one query over N keys/values.
 * K is [N][d], V is [N][dv]. p_j = exp(s_j - max s) / sum_k exp(s_k - max s)
 * with s_j = scale * q . K_j; out = sum_j p_j V_j; lse = ln sum_j exp(s_j).
 * Returns 0, or -1 if N < 1 or memory runs out. */
int oracle_attend(int d, int dv, int N, const double *q, const double *K,
                  const double *V, double scale, double *out, double *lse)
{
    if (N < 1) return -1;
    double *s = (double *)malloc((size_t)N * sizeof(double));
    if (!s) return -1;
    double smax = -INFINITY;
    for (int j = 0; j < N; ++j) {
        double acc = 0.0;
        for (int i = 0; i < d; ++i) acc += q[i] * K[(size_t)j * d + i];
        s[j] = scale * acc;
        if (s[j] > smax) smax = s[j];
    }
    double denom = 0.0;
    for (int j = 0; j < N; ++j) denom += exp(s[j] - smax);
    for (int i = 0; i < dv; ++i) out[i] = 0.0;
    for (int j = 0; j < N; ++j) {
        double p = exp(s[j] - smax) / denom;
        for (int i = 0; i < dv; ++i) out[i] += p * V[(size_t)j * dv + i];
    }
    if (lse) *lse = smax + log(denom);
    free(s);
    return 0;
}

/* Eq. 3 for one latent: xhat[i] = sum_c W_up[i][c] * z[c] + mu[i].
 * W_up is [d][r]; mu may be NULL (taken as zero). */
void oracle_reconstruct(int d, int r, const double *w_up, const double *z,
                        const double *mu, double *xhat)
{
    for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int c = 0; c < r; ++c) acc += w_up[(size_t)i * r + c] * z[c];
        xhat[i] = acc + (mu ? mu[i] : 0.0);
    }
}

/* One decode unit (one batch row, one head, one layer, one loop t), explicit
 * form. zk is [N][r_k], zv is [N][r_v]; dk = W^K_up,t is [d][r_k], dv =
 * W^V_up,t is [d][r_v]; mu_k, mu_v are this loop's slices mu_t (nullable).
 * Rebuilds khat_j and vhat_j for every cached token, then attends. */
int oracle_decode_unit(int d, int N, int r_k, int r_v, const double *q,
                       const double *zk, const double *zv, const double *dk,
                       const double *dv, const double *mu_k,
                       const double *mu_v, double scale, double *out,
                       double *lse)
{
    if (N < 1) return -1;
    double *K = (double *)malloc((size_t)N * d * sizeof(double));
    double *V = (double *)malloc((size_t)N * d * sizeof(double));
    if (!K || !V) { free(K); free(V); return -1; }
    for (int j = 0; j < N; ++j) {
        oracle_reconstruct(d, r_k, dk, zk + (size_t)j * r_k, mu_k, K + (size_t)j * d);
        oracle_reconstruct(d, r_v, dv, zv + (size_t)j * r_v, mu_v, V + (size_t)j * d);
    }
    int rc = oracle_attend(d, d, N, q, K, V, scale, out, lse);
    free(K);
    free(V);
    return rc;
}

/* The same unit through the §7 absorbed identities, kept apart from the
 * explicit form so the two can be compared:
 *   q' = W^K_up,t^T q            (scores read latents directly)
 *   s_j = scale * (q' . zk_j + q . mu_k)
 *   ubar = sum_j p_j zv_j        (value sum taken in latent space)
 *   out = W^V_up,t ubar + mu_v   (sum_j p_j = 1 carries mu_v through) */
int oracle_decode_unit_absorbed(int d, int N, int r_k, int r_v,
                                const double *q, const double *zk,
                                const double *zv, const double *dk,
                                const double *dv, const double *mu_k,
                                const double *mu_v, double scale,
                                double *out, double *lse)
{
    if (N < 1) return -1;
    double *qp = (double *)malloc((size_t)r_k * sizeof(double));
    double *s = (double *)malloc((size_t)N * sizeof(double));
    double *ub = (double *)malloc((size_t)r_v * sizeof(double));
    if (!qp || !s || !ub) { free(qp); free(s); free(ub); return -1; }
    for (int c = 0; c < r_k; ++c) {
        double acc = 0.0;
        for (int i = 0; i < d; ++i) acc += dk[(size_t)i * r_k + c] * q[i];
        qp[c] = acc;
    }
    double c0 = 0.0;
    if (mu_k) for (int i = 0; i < d; ++i) c0 += q[i] * mu_k[i];
    double smax = -INFINITY;
    for (int j = 0; j < N; ++j) {
        double acc = 0.0;
        for (int c = 0; c < r_k; ++c) acc += qp[c] * zk[(size_t)j * r_k + c];
        s[j] = scale * (acc + c0);
        if (s[j] > smax) smax = s[j];
    }
    double denom = 0.0;
    for (int j = 0; j < N; ++j) denom += exp(s[j] - smax);
    for (int c = 0; c < r_v; ++c) ub[c] = 0.0;
    for (int j = 0; j < N; ++j) {
        double p = exp(s[j] - smax) / denom;
        for (int c = 0; c < r_v; ++c) ub[c] += p * zv[(size_t)j * r_v + c];
    }
    oracle_reconstruct(d, r_v, dv, ub, mu_v, out);
    if (lse) *lse = smax + log(denom);
    free(qp);
    free(s);
    free(ub);
    return 0;
}

/* Per-head decode over a list of units, each with its own pointers gathered
 * by the caller into flat arrays:
 *   q      [U][d]
 *   zk     [U][N][r_k],  zv [U][N][r_v]
 *   dk     [U][d][r_k],  dv [U][d][r_v]
 *   mu_k, mu_v [U][d] or NULL
 *   out    [U][d],  lse [U] (nullable)
 * Units run in parallel when OpenMP is on; nthreads <= 0 keeps the
 * runtime default. Returns 0, or the number of units that failed. */
int oracle_decode_units(int U, int d, int N, int r_k, int r_v,
                        const double *q, const double *zk, const double *zv,
                        const double *dk, const double *dv,
                        const double *mu_k, const double *mu_v, double scale,
                        double *out, double *lse, int nthreads)
{
    int bad = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : bad)
#endif
    for (int u = 0; u < U; ++u) {
        int rc = oracle_decode_unit(
            d, N, r_k, r_v, q + (size_t)u * d, zk + (size_t)u * N * r_k,
            zv + (size_t)u * N * r_v, dk + (size_t)u * d * r_k,
            dv + (size_t)u * d * r_v, mu_k ? mu_k + (size_t)u * d : NULL,
            mu_v ? mu_v + (size_t)u * d : NULL, scale, out + (size_t)u * d,
            lse ? lse + u : NULL);
        if (rc) bad += 1;
    }
    return bad;
}

/* Number of threads an OpenMP region would use (1 without OpenMP). */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Eq. 2, the latent write, for every token of every group:
 *   x    [T][N][G][d_loop]   loop-major, as each loop emits its K (or V)
 *   w    [G][T*d_loop][r]    W_down per group; stacked index k = t*d_loop + i
 *   mu   [G][T*d_loop] or NULL
 *   z    [G][N][r]
 * z[g][n][c] = sum_k (x_stack[k] - mu[g][k]) * w[g][k][c], where
 * x_stack[t*d_loop + i] = x[t][n][g][i] (Eq. 1). nthreads > 0 sets the
 * OpenMP thread count; otherwise the runtime default is kept. */
void oracle_encode(int T, int N, int G, int d_loop, int r, const double *x,
                   const double *w, const double *mu, double *z, int nthreads)
{
    const size_t K = (size_t)T * d_loop;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for collapse(2) schedule(static)
#endif
    for (int g = 0; g < G; ++g) {
        for (int n = 0; n < N; ++n) {
            double *zo = z + ((size_t)g * N + n) * r;
            for (int c = 0; c < r; ++c) zo[c] = 0.0;
            for (int t = 0; t < T; ++t) {
                const double *xt = x + (((size_t)t * N + n) * G + g) * d_loop;
                for (int i = 0; i < d_loop; ++i) {
                    size_t k = (size_t)t * d_loop + i;
                    double xc = xt[i] - (mu ? mu[(size_t)g * K + k] : 0.0);
                    const double *wr = w + ((size_t)g * K + k) * r;
                    for (int c = 0; c < r; ++c) zo[c] += xc * wr[c];
                }
            }
        }
    }
}
