/*
 * Gated KalmaNet (GKA) layer: plain float64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the package smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library; the two are independent restatements of the same method.
 *
 * Source: "Gated KalmaNet: A Fading Memory Layer Through Test-Time Ridge
 * Regression" (arXiv 2511.21016), as summarised on the ai.info page
 * (Key Contributions 2-3, Main Findings, Methodology in Plain English) and
 * the appendix fragments on the pith.science page (Lemma 3 / Lemma 4 on the
 * Chebyshev weight schedule, and the rate table for kappa = 51).
 *
 * What it computes, per (batch, head), token by token (no chunking, no
 * blocking, no fusion):
 *   H_t = beta_t H_{t-1} + k_t k_t^T          (gated fading Gram state)
 *   M_t = beta_t M_{t-1} + v_t k_t^T          (value state; the pages' U_t)
 *   n_t = ||H_t||_F,  lambda_t = a n_t        (adaptive ridge)
 *   x_t = r-step Chebyshev iterate for (H_t + lambda_t I) x = q_t on the
 *         spectral interval [a n_t, (1+a) n_t], started at x = 0
 *   o_t = M_t x_t
 * The decay beta_t multiplies the old state (the pages' gate gamma_t of the
 * weighted ridge objective, Eq. 3, with eta_{t,i} = prod_{j=i+1..t} gamma_j).
 *
 * Write-gated variant (ai.info page, Main Findings, "The beta_t-augmented
 * variant", and Future Directions): a per-token input-selectivity gate in
 * [0, 1] scales the token's write into both states.  Named g_t here, since
 * beta_t already names the decay:
 *   H_t = beta_t H_{t-1} + g_t k_t k_t^T,   M_t = beta_t M_{t-1} + g_t v_t k_t^T
 * Every entry point below takes the gate as a nullable array; NULL means
 * g_t = 1 for every token (the layer of the paper's experiments).
 *
 * All arithmetic is float64.  Matrices are dense row-major.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/*
 * Chebyshev weight schedule (pith.science appendix, Lemma 3 "weight
 * schedule"): omega_0 = 2 and omega_i = 1 / (1 - rho^2 omega_{i-1} / 4),
 * where rho = (L - mu) / (L + mu).  omega_i is used by the i-th update that
 * follows the first step x_1 = q / d.  Fills omega[0..n-1].
 */
void gka_oracle_omegas(double rho, int n, double *omega)
{
    if (n <= 0) return;
    omega[0] = 2.0;
    for (int i = 1; i < n; ++i)
        omega[i] = 1.0 / (1.0 - rho * rho * omega[i - 1] / 4.0);
}

/*
 * r-step Chebyshev iteration for A x = q, where A (D x D, symmetric) has its
 * spectrum in [mu, L] (ai.info, Key Contributions 2 and Methodology: the
 * iteration needs only matrix-vector products).  Three-term form with
 * d = (L + mu)/2:
 *   x_0 = 0,  x_1 = q / d,
 *   x_{i+1} = x_{i-1} + omega_i * ( (q - A x_i) / d + x_i - x_{i-1} ),
 *   i = 1 .. r-1,  result x_r  (r - 1 matrix-vector products).
 * r must be >= 1.  work must hold 3*D doubles.
 */
void gka_oracle_cheb_solve(const double *A, const double *q, int D,
                           double mu, double L, int r, double *x, double *work)
{
    double d = 0.5 * (L + mu);
    double rho = (L - mu) / (L + mu);
    double *xprev = work, *xnew = work + D, *y = work + 2 * D;
    double *omega = (double *)malloc(sizeof(double) * (size_t)(r > 1 ? r : 1));
    gka_oracle_omegas(rho, r, omega);

    for (int i = 0; i < D; ++i) {
        xprev[i] = 0.0;
        x[i] = q[i] / d;
    }
    for (int it = 1; it < r; ++it) {
        for (int i = 0; i < D; ++i) {
            double s = 0.0;
            for (int j = 0; j < D; ++j) s += A[(size_t)i * D + j] * x[j];
            y[i] = s;
        }
        double w = omega[it];
        for (int i = 0; i < D; ++i)
            xnew[i] = xprev[i] + w * ((q[i] - y[i]) / d + x[i] - xprev[i]);
        for (int i = 0; i < D; ++i) {
            xprev[i] = x[i];
            x[i] = xnew[i];
        }
    }
    free(omega);
}

/*
 * One token of the recurrence on one head, in place on (H, M), with decay
 * beta and write gate g.
 * Writes the token's output o (D) and returns n_t = ||H_t||_F.
 * If solve == 0 only the state update and the norm are done.
 * work: D*D + 4*D doubles.
 */
static double gka_token(double *H, double *M, const double *q, const double *k,
                        const double *v, double beta, double g, int D, double a, int r,
                        int solve, double *o, double *work)
{
    /* state update (ai.info, Methodology: running weighted covariances
     * with a decay factor; Main Findings: the write gate g scales the
     * token's own term) */
    for (int i = 0; i < D; ++i)
        for (int j = 0; j < D; ++j) {
            H[(size_t)i * D + j] = beta * H[(size_t)i * D + j] + g * k[i] * k[j];
            M[(size_t)i * D + j] = beta * M[(size_t)i * D + j] + g * v[i] * k[j];
        }
    /* Frobenius norm and adaptive ridge (ai.info, Key Contributions 2) */
    double n2 = 0.0;
    for (size_t e = 0; e < (size_t)D * D; ++e) n2 += H[e] * H[e];
    double n = sqrt(n2);
    if (!solve) return n;

    double *A = work, *x = work + (size_t)D * D, *cw = x + D;
    if (n == 0.0) {
        /* zero state: the regularised system degenerates; the output is 0 */
        for (int i = 0; i < D; ++i) o[i] = 0.0;
        return n;
    }
    double lam = a * n;
    memcpy(A, H, sizeof(double) * (size_t)D * D);
    for (int i = 0; i < D; ++i) A[(size_t)i * D + i] += lam;
    gka_oracle_cheb_solve(A, q, D, lam, (1.0 + a) * n, r, x, cw);
    /* readout o_t = M_t x_t (ai.info, Methodology: "then multiplying by U_t") */
    for (int i = 0; i < D; ++i) {
        double s = 0.0;
        for (int j = 0; j < D; ++j) s += M[(size_t)i * D + j] * x[j];
        o[i] = s;
    }
    return n;
}

/*
 * Token-by-token forward over [B, Hh, T, D] inputs (row-major, D fastest).
 *   gate        nullable, [B, Hh, T]: write gate g_t (NULL: 1 everywhere)
 *   init_state  nullable, [B, Hh, 2, D, D]: H then M at t = -1 (zero if NULL)
 *   solve_from  tokens t < solve_from only advance the state (o not written)
 *   o           [B, Hh, T, D]
 *   norms       nullable, [B, Hh, T]: ||H_t||_F
 *   final_state nullable, [B, Hh, 2, D, D]
 *   chunk, chunk_states  nullable pair: when chunk > 0 and chunk_states is
 *               given, the state in force before token n*chunk is stored at
 *               chunk_states[B, Hh, T/chunk, 2, D, D]
 *   nthreads    OpenMP threads over (b, h); <= 0 means the runtime default
 * Returns 0, or -1 on bad arguments.
 */
int gka_oracle_forward(const double *q, const double *k, const double *v,
                       const double *beta, const double *gate, int B, int Hh, int T, int D,
                       double a, int r, const double *init_state,
                       int solve_from, double *o, double *norms,
                       double *final_state, int chunk, double *chunk_states,
                       int nthreads)
{
    if (B < 0 || Hh < 0 || T < 0 || D <= 0 || r < 1 || !(a > 0.0)) return -1;
    long nh = (long)B * Hh;
    size_t DD = (size_t)D * D;
    int nchunks = (chunk > 0) ? T / chunk : 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (long h = 0; h < nh; ++h) {
        double *H = (double *)calloc(2 * DD, sizeof(double));
        double *M = H + DD;
        double *work = (double *)malloc(sizeof(double) * (DD + 4 * (size_t)D));
        if (init_state) memcpy(H, init_state + (size_t)h * 2 * DD, sizeof(double) * 2 * DD);
        for (int t = 0; t < T; ++t) {
            if (chunk_states && chunk > 0 && t % chunk == 0 && t / chunk < nchunks)
                memcpy(chunk_states + ((size_t)h * nchunks + t / chunk) * 2 * DD, H,
                       sizeof(double) * 2 * DD);
            size_t row = ((size_t)h * T + t) * D;
            double g = gate ? gate[(size_t)h * T + t] : 1.0;
            double n = gka_token(H, M, q + row, k + row, v + row, beta[(size_t)h * T + t],
                                 g, D, a, r, t >= solve_from, o + row, work);
            if (norms) norms[(size_t)h * T + t] = n;
        }
        if (final_state) memcpy(final_state + (size_t)h * 2 * DD, H, sizeof(double) * 2 * DD);
        free(work);
        free(H);
    }
    return 0;
}

/*
 * One recurrent decode step for [B, Hh] heads: the same token update as the
 * forward, applied in place to state [B, Hh, 2, D, D] (H then M).
 * q, k, v, o: [B, Hh, D];  beta: [B, Hh];  gate: nullable [B, Hh].
 */
int gka_oracle_decode_step(double *state, const double *q, const double *k,
                           const double *v, const double *beta, const double *gate,
                           int B, int Hh,
                           int D, double a, int r, double *o, int nthreads)
{
    if (B < 0 || Hh < 0 || D <= 0 || r < 1 || !(a > 0.0)) return -1;
    long nh = (long)B * Hh;
    size_t DD = (size_t)D * D;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (long h = 0; h < nh; ++h) {
        double *work = (double *)malloc(sizeof(double) * (DD + 4 * (size_t)D));
        double *H = state + (size_t)h * 2 * DD;
        gka_token(H, H + DD, q + (size_t)h * D, k + (size_t)h * D, v + (size_t)h * D,
                  beta[h], gate ? gate[h] : 1.0, D, a, r, 1, o + (size_t)h * D, work);
        free(work);
    }
    return 0;
}

/*
 * Chunk-wise ||H_t||_F (ai.info, Key Contributions 3 and Methodology: a
 * closed-form chunk-wise expression through the Gram matrix of the keys;
 * only the chunk-start state is carried from chunk to chunk).
 * Within a chunk with start state H_s and positions j = 0..C-1:
 *   b_j    = prod_{m <= j} beta_m               (decay of H_s to token j)
 *   w_{ji} = prod_{i < m <= j} beta_m, i <= j   (decay of token i to token j)
 *   H_j    = b_j H_s + sum_{i<=j} w_{ji} g_i k_i k_i^T
 *   ||H_j||_F^2 = b_j^2 ||H_s||_F^2 + 2 b_j sum_{i<=j} w_{ji} g_i k_i^T H_s k_i
 *               + sum_{i,l<=j} w_{ji} g_i w_{jl} g_l (k_i^T k_l)^2
 * and the next chunk starts from
 *   H_s' = b_{C-1} H_s + sum_i w_{C-1,i} g_i k_i k_i^T.
 * g is the write gate (nullable, [B, Hh, T]; NULL: 1).  The products are
 * formed directly (no logarithms).  T must be a multiple of C.
 * norms: [B, Hh, T].
 */
int gka_oracle_chunked_norms(const double *k, const double *beta, const double *gate,
                             int B, int Hh, int T, int D, int C, double *norms,
                             int nthreads)
{
    if (B < 0 || Hh < 0 || T < 0 || D <= 0 || C <= 0 || T % C != 0) return -1;
    long nh = (long)B * Hh;
    size_t DD = (size_t)D * D;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (long h = 0; h < nh; ++h) {
        double *Hs = (double *)calloc(DD, sizeof(double));
        double *Hn = (double *)malloc(sizeof(double) * DD);
        double *u = (double *)malloc(sizeof(double) * C);
        double *G = (double *)malloc(sizeof(double) * (size_t)C * C);
        double *w = (double *)malloc(sizeof(double) * (size_t)C * C);
        double *b = (double *)malloc(sizeof(double) * C);
        for (int c0 = 0; c0 < T; c0 += C) {
            const double *K = k + ((size_t)h * T + c0) * D;
            const double *bt = beta + (size_t)h * T + c0;
            const double *gt = gate ? gate + (size_t)h * T + c0 : NULL;
            /* decays, each column i times the write gate of token i */
            for (int j = 0; j < C; ++j) {
                double p = 1.0;
                for (int m = 0; m <= j; ++m) p *= bt[m];
                b[j] = p;
                for (int i = 0; i < C; ++i) {
                    double wji = 0.0;
                    if (i <= j) {
                        wji = 1.0;
                        for (int m = i + 1; m <= j; ++m) wji *= bt[m];
                        if (gt) wji *= gt[i];
                    }
                    w[(size_t)j * C + i] = wji;
                }
            }
            /* ||H_s||^2, u_i = k_i^T H_s k_i, G = K K^T */
            double hs2 = 0.0;
            for (size_t e = 0; e < DD; ++e) hs2 += Hs[e] * Hs[e];
            for (int i = 0; i < C; ++i) {
                double s = 0.0;
                for (int p = 0; p < D; ++p)
                    for (int qd = 0; qd < D; ++qd)
                        s += K[(size_t)i * D + p] * Hs[(size_t)p * D + qd] * K[(size_t)i * D + qd];
                u[i] = s;
                for (int l = 0; l < C; ++l) {
                    double g = 0.0;
                    for (int p = 0; p < D; ++p) g += K[(size_t)i * D + p] * K[(size_t)l * D + p];
                    G[(size_t)i * C + l] = g;
                }
            }
            for (int j = 0; j < C; ++j) {
                double cross = 0.0, intra = 0.0;
                for (int i = 0; i <= j; ++i) cross += w[(size_t)j * C + i] * u[i];
                for (int i = 0; i <= j; ++i)
                    for (int l = 0; l <= j; ++l) {
                        double g = G[(size_t)i * C + l];
                        intra += w[(size_t)j * C + i] * w[(size_t)j * C + l] * g * g;
                    }
                double n2 = b[j] * b[j] * hs2 + 2.0 * b[j] * cross + intra;
                norms[(size_t)h * T + c0 + j] = sqrt(n2 > 0.0 ? n2 : 0.0);
            }
            /* chunk-start state for the next chunk */
            for (int p = 0; p < D; ++p)
                for (int qd = 0; qd < D; ++qd) {
                    double s = b[C - 1] * Hs[(size_t)p * D + qd];
                    for (int i = 0; i < C; ++i)
                        s += w[(size_t)(C - 1) * C + i] * K[(size_t)i * D + p] * K[(size_t)i * D + qd];
                    Hn[(size_t)p * D + qd] = s;
                }
            memcpy(Hs, Hn, sizeof(double) * DD);
        }
        free(Hs); free(Hn); free(u); free(G); free(w); free(b);
    }
    return 0;
}

/* Threads OpenMP would use for the calls above (1 without OpenMP). */
int gka_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Backward pass by implicit differentiation (ai.info page, Key Contributions
 * 3 and Methodology: the backward treats x_t as the solution of the linear
 * system that the Chebyshev iteration approximately solves and reuses the
 * iteration on the upstream gradient; Main Findings: Lemma 2, dq_t = dq^_t;
 * pith.science appendix, Eq. 50, the key gradient with its ||H_t||_F term).
 *
 * With g_o = dL/do_t (the upstream gradient), x_t the forward iterate and
 * A_t = H_t + a ||H_t||_F I:
 *   u_t = M_t^T g_o                 (dL/dx_t)
 *   y_t = r-step Chebyshev for A_t y = u_t   (the same iteration as the forward)
 *   dq_t = y_t
 *   dL/dH_t = -y_t x_t^T - c_t H_t,  c_t = a (y_t . x_t) / ||H_t||_F
 *     (from dx = -A^-1 dA x and d||H||_F = <H, dH> / ||H||_F)
 *   dL/dM_t = g_o x_t^T
 * then back through H_t = beta_t H_{t-1} + g_t k_t k_t^T (and M) with the
 * adjoint states  Hb_t = dL/dH_t + beta_{t+1} Hb_{t+1},  Mb_t likewise:
 *   dk_t = g_t ((Hb_t + Hb_t^T) k_t + Mb_t^T v_t),   dv_t = g_t Mb_t k_t,
 *   dbeta_t = <Hb_t, H_{t-1}> + <Mb_t, M_{t-1}>,
 *   dg_t = k_t^T Hb_t k_t + v_t^T Mb_t k_t       (the write gate g, if any).
 * A token with ||H_t||_F = 0 has x_t = 0 and contributes nothing.
 *
 * Inputs as for gka_oracle_forward plus dout [B, Hh, T, D]; outputs dq, dk,
 * dv [B, Hh, T, D], dbeta [B, Hh, T] and, when gate is given, dgate
 * [B, Hh, T] (nullable).  Keeps every H_t and M_t of a head in memory
 * (T * 2 * D * D doubles per thread): meant for test sizes.
 * Returns 0, -1 on bad arguments, -2 if memory runs out.
 */
int gka_oracle_backward(const double *q, const double *k, const double *v,
                        const double *beta, const double *gate, const double *dout,
                        int B, int Hh, int T, int D, double a, int r,
                        double *dq, double *dk, double *dv, double *dbeta,
                        double *dgate, int nthreads)
{
    if (B < 0 || Hh < 0 || T < 0 || D <= 0 || r < 1 || !(a > 0.0)) return -1;
    long nh = (long)B * Hh;
    size_t DD = (size_t)D * D;
    int fail = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (long h = 0; h < nh; ++h) {
        /* S[t] = (H_t, M_t) for t = 0..T-1, plus the zero state at index -1 */
        double *S = (double *)calloc((size_t)(T + 1) * 2 * DD, sizeof(double));
        double *X = (double *)malloc(sizeof(double) * ((size_t)T * D + 1));
        double *Y = (double *)malloc(sizeof(double) * ((size_t)T * D + 1));
        double *cn = (double *)malloc(sizeof(double) * ((size_t)T + 1));
        double *work = (double *)malloc(sizeof(double) * (DD + 4 * (size_t)D));
        double *A = (double *)malloc(sizeof(double) * DD);
        double *u = (double *)malloc(sizeof(double) * D);
        double *o = (double *)malloc(sizeof(double) * D);
        double *Hb = (double *)calloc(2 * DD, sizeof(double));
        if (!S || !X || !Y || !cn || !work || !A || !u || !o || !Hb) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            fail = 1;
            free(S); free(X); free(Y); free(cn); free(work); free(A); free(u); free(o); free(Hb);
            continue;
        }
        double *Mb = Hb + DD;
        const double *bt = beta + (size_t)h * T;
        const double *gt = gate ? gate + (size_t)h * T : NULL;
        /* forward sweep: states, iterates x_t, adjoint solves y_t */
        for (int t = 0; t < T; ++t) {
            double *Ht = S + (size_t)(t + 1) * 2 * DD, *Mt = Ht + DD;
            memcpy(Ht, S + (size_t)t * 2 * DD, sizeof(double) * 2 * DD);
            size_t row = ((size_t)h * T + t) * D;
            double n = gka_token(Ht, Mt, q + row, k + row, v + row, bt[t], gt ? gt[t] : 1.0,
                                 D, a, r, 1, o, work);
            double *xt = X + (size_t)t * D, *yt = Y + (size_t)t * D;
            if (n == 0.0) {
                for (int i = 0; i < D; ++i) xt[i] = yt[i] = 0.0;
                cn[t] = 0.0;
                continue;
            }
            /* gka_token left the forward iterate at work + D*D */
            memcpy(xt, work + DD, sizeof(double) * D);
            const double *g = dout + row;
            for (int j = 0; j < D; ++j) {
                double s = 0.0;
                for (int i = 0; i < D; ++i) s += Mt[(size_t)i * D + j] * g[i];
                u[j] = s;
            }
            memcpy(A, Ht, sizeof(double) * DD);
            for (int i = 0; i < D; ++i) A[(size_t)i * D + i] += a * n;
            gka_oracle_cheb_solve(A, u, D, a * n, (1.0 + a) * n, r, yt, work);
            double yx = 0.0;
            for (int i = 0; i < D; ++i) yx += yt[i] * xt[i];
            cn[t] = a * yx / n;
        }
        /* reverse sweep over the adjoint states */
        for (int t = T - 1; t >= 0; --t) {
            const double *Ht = S + (size_t)(t + 1) * 2 * DD;
            const double *Hp = S + (size_t)t * 2 * DD, *Mp = Hp + DD;
            const double bnext = (t + 1 < T) ? bt[t + 1] : 0.0;
            const double *xt = X + (size_t)t * D, *yt = Y + (size_t)t * D;
            size_t row = ((size_t)h * T + t) * D;
            const double *g = dout + row;
            for (int i = 0; i < D; ++i)
                for (int j = 0; j < D; ++j) {
                    size_t e = (size_t)i * D + j;
                    Hb[e] = bnext * Hb[e] - yt[i] * xt[j] - cn[t] * Ht[e];
                    Mb[e] = bnext * Mb[e] + g[i] * xt[j];
                }
            const double *kt = k + row, *vt = v + row;
            const double gw = gt ? gt[t] : 1.0;
            double db = 0.0, dg = 0.0;
            for (size_t e = 0; e < DD; ++e) db += Hb[e] * Hp[e] + Mb[e] * Mp[e];
            for (int i = 0; i < D; ++i) {
                double sk = 0.0, sv = 0.0;
                for (int j = 0; j < D; ++j) {
                    sk += (Hb[(size_t)i * D + j] + Hb[(size_t)j * D + i]) * kt[j]
                          + Mb[(size_t)j * D + i] * vt[j];
                    sv += Mb[(size_t)i * D + j] * kt[j];
                }
                dk[row + i] = gw * sk;
                dv[row + i] = gw * sv;
                double hk = 0.0, mk = 0.0;
                for (int j = 0; j < D; ++j) {
                    hk += Hb[(size_t)i * D + j] * kt[j];
                    mk += Mb[(size_t)i * D + j] * kt[j];
                }
                dg += kt[i] * hk + vt[i] * mk;
                dq[row + i] = yt[i];
            }
            dbeta[(size_t)h * T + t] = db;
            if (dgate) dgate[(size_t)h * T + t] = dg;
        }
        free(S); free(X); free(Y); free(cn); free(work); free(A); free(u); free(o); free(Hb);
    }
    return fail ? -2 : 0;
}

/*
 * Solver study (ai.info page, Key Contributions 2 and Main Findings: CH is
 * compared with gradient descent, accelerated gradient descent and conjugate
 * gradient on the layer's systems; pith.science page, Fig. 1a and Fig. 8:
 * residual norms per iteration in a random-regression setup, and for several
 * regularisation strengths).
 *
 * For every token t the system A_t x = q_t of the layer (A_t = H_t + a n_t I,
 * spectrum in [mu, L] = [a n_t, (1+a) n_t]) is solved from x_0 = 0 by
 *   solver 0  Chebyshev (the layer's iteration)
 *   solver 1  gradient descent with the fixed step 2/(L + mu)
 *   solver 2  Nesterov's accelerated gradient descent for strongly convex
 *             quadratics: y = x_i + m (x_i - x_{i-1}), x_{i+1} = y + (q - A y)/L,
 *             m = (sqrt(kappa) - 1)/(sqrt(kappa) + 1), kappa = L / mu
 *   solver 3  conjugate gradient (Hestenes-Stiefel)
 * and resid[t][i] = ||q_t - A_t x_i|| / ||q_t|| for i = 0..r (the true residual,
 * formed from x_i; resid[t][0] = 1).  A token with n_t = 0 or q_t = 0 gets zeros.
 * Inputs as gka_oracle_forward (gate nullable); resid: [B, Hh, T, r + 1].
 */
static void solver_residuals(const double *A, const double *q, int D, double mu, double L,
                             int r, int solver, double *res, double *work)
{
    double *x = work, *xp = work + D, *y = work + 2 * D, *Ay = work + 3 * D;
    double *rr = work + 4 * D, *p = work + 5 * D, *Ap = work + 6 * D;
    double qn = 0.0;
    for (int i = 0; i < D; ++i) qn += q[i] * q[i];
    qn = sqrt(qn);
    if (qn == 0.0) {
        for (int i = 0; i <= r; ++i) res[i] = 0.0;
        return;
    }
    for (int i = 0; i < D; ++i) x[i] = xp[i] = 0.0;
    res[0] = 1.0;
    const double d = 0.5 * (L + mu), rho = (L - mu) / (L + mu);
    const double kap = L / mu, m = (sqrt(kap) - 1.0) / (sqrt(kap) + 1.0);
    double *omega = (double *)malloc(sizeof(double) * (size_t)(r > 1 ? r : 1));
    gka_oracle_omegas(rho, r, omega);
    double rs = 0.0;
    if (solver == 3) {
        for (int i = 0; i < D; ++i) rr[i] = p[i] = q[i];
        for (int i = 0; i < D; ++i) rs += rr[i] * rr[i];
    }
    for (int it = 0; it < r; ++it) {
        if (solver == 0) {
            if (it == 0) {
                for (int i = 0; i < D; ++i) x[i] = q[i] / d;
            } else {
                /* x_{it+1} = x_{it-1} + omega_it ((q - A x_it)/d + x_it - x_{it-1}) */
                for (int i = 0; i < D; ++i) {
                    double s = 0.0;
                    for (int j = 0; j < D; ++j) s += A[(size_t)i * D + j] * x[j];
                    Ay[i] = s;
                }
                for (int i = 0; i < D; ++i) {
                    double xn = xp[i] + omega[it] * ((q[i] - Ay[i]) / d + x[i] - xp[i]);
                    xp[i] = x[i];
                    x[i] = xn;
                }
            }
        } else if (solver == 1 || solver == 2) {
            for (int i = 0; i < D; ++i) y[i] = solver == 2 ? x[i] + m * (x[i] - xp[i]) : x[i];
            for (int i = 0; i < D; ++i) {
                double s = 0.0;
                for (int j = 0; j < D; ++j) s += A[(size_t)i * D + j] * y[j];
                Ay[i] = s;
            }
            const double step = solver == 2 ? 1.0 / L : 1.0 / d;
            for (int i = 0; i < D; ++i) {
                xp[i] = x[i];
                x[i] = y[i] + step * (q[i] - Ay[i]);
            }
        } else {
            for (int i = 0; i < D; ++i) {
                double s = 0.0;
                for (int j = 0; j < D; ++j) s += A[(size_t)i * D + j] * p[j];
                Ap[i] = s;
            }
            double pAp = 0.0;
            for (int i = 0; i < D; ++i) pAp += p[i] * Ap[i];
            const double alpha = pAp > 0.0 ? rs / pAp : 0.0;
            double rs1 = 0.0;
            for (int i = 0; i < D; ++i) {
                x[i] += alpha * p[i];
                rr[i] -= alpha * Ap[i];
                rs1 += rr[i] * rr[i];
            }
            const double beta = rs > 0.0 ? rs1 / rs : 0.0;
            for (int i = 0; i < D; ++i) p[i] = rr[i] + beta * p[i];
            rs = rs1;
        }
        /* true residual of the new iterate */
        double e2 = 0.0;
        for (int i = 0; i < D; ++i) {
            double s = 0.0;
            for (int j = 0; j < D; ++j) s += A[(size_t)i * D + j] * x[j];
            e2 += (q[i] - s) * (q[i] - s);
        }
        res[it + 1] = sqrt(e2) / qn;
    }
    free(omega);
}

int gka_oracle_solver_study(const double *q, const double *k, const double *beta,
                            const double *gate, int B, int Hh, int T, int D, double a,
                            int r, int solver, double *resid, int nthreads)
{
    if (B < 0 || Hh < 0 || T < 0 || D <= 0 || r < 1 || !(a > 0.0) || solver < 0 || solver > 3)
        return -1;
    long nh = (long)B * Hh;
    size_t DD = (size_t)D * D;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (long h = 0; h < nh; ++h) {
        double *H = (double *)calloc(DD, sizeof(double));
        double *A = (double *)malloc(sizeof(double) * DD);
        double *work = (double *)malloc(sizeof(double) * 8 * (size_t)D);
        for (int t = 0; t < T; ++t) {
            size_t row = ((size_t)h * T + t) * D;
            const double g = gate ? gate[(size_t)h * T + t] : 1.0;
            const double b = beta[(size_t)h * T + t];
            const double *kt = k + row;
            double n2 = 0.0;
            for (int i = 0; i < D; ++i)
                for (int j = 0; j < D; ++j) {
                    double v = b * H[(size_t)i * D + j] + g * kt[i] * kt[j];
                    H[(size_t)i * D + j] = v;
                    n2 += v * v;
                }
            double *res = resid + ((size_t)h * T + t) * (size_t)(r + 1);
            const double n = sqrt(n2);
            if (n == 0.0) {
                for (int i = 0; i <= r; ++i) res[i] = 0.0;
                continue;
            }
            memcpy(A, H, sizeof(double) * DD);
            for (int i = 0; i < D; ++i) A[(size_t)i * D + i] += a * n;
            solver_residuals(A, q + row, D, a * n, (1.0 + a) * n, r, solver, res, work);
        }
        free(H); free(A); free(work);
    }
    return 0;
}

/*
 * The residual history of one solver on one system A x = q (A: D x D symmetric
 * with its spectrum in [mu, L]); res: r + 1 values (see gka_oracle_solver_study).
 */
void gka_oracle_solver_residuals(const double *A, const double *q, int D, double mu, double L,
                                 int r, int solver, double *res)
{
    double *work = (double *)malloc(sizeof(double) * 8 * (size_t)D);
    solver_residuals(A, q, D, mu, L, r, solver, res, work);
    free(work);
}
