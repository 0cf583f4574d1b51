// Solver study on CUDA cores (fp32): the residual history of one of four
// iterative solvers on every token's system A_t x = q_t of the layer.
//
// Method: "Gated KalmaNet" (arXiv 2511.21016), ai.info page, Key Contributions
// 2 and Main Findings (Chebyshev is compared with gradient descent,
// accelerated gradient descent and conjugate gradient); pith.science page,
// Fig. 1a and Fig. 8 (residual norms per iteration, for several
// regularisation strengths).
//
// A_t = H_t + a n_t I with n_t = ||H_t||_F, spectrum in [mu, L] = [a n_t, (1+a) n_t],
// d = (L + mu) / 2.  From x_0 = 0:
//   0 Chebyshev          the layer's three-term iteration
//   1 gradient descent   x_{i+1} = x_i + (q - A x_i) / d
//   2 Nesterov           y = x_i + m (x_i - x_{i-1}), x_{i+1} = y + (q - A y) / L,
//                        m = (sqrt(kappa) - 1) / (sqrt(kappa) + 1), kappa = (1+a)/a
//   3 conjugate gradient Hestenes-Stiefel
// resid[t][i] = ||q_t - A_t x_i|| / ||q_t||, i = 0..r, the true residual of each
// iterate (one extra product per step for conjugate gradient); zero for a token
// with n_t = 0 or q_t = 0.  A x is formed in chunk form as in the solve:
// b_j H_s x + sum_{i<=j} w_ji k~_i (k~_i . x) + lambda x.
#pragma once

#include "chunk_simt.cuh"
#include "common.cuh"

namespace gka {

template <typename Tin, int D, int SOLVER>
__global__ void __launch_bounds__(kSimtThreads)
k_solver_study(const Tin *__restrict__ q, const Tin *__restrict__ k, const float *__restrict__ beta,
               const float *__restrict__ gate, const float *__restrict__ states,
               const float *__restrict__ norms, float *__restrict__ resid, int T, int N, int C,
               const ChebParams P) {
    constexpr int TG = kSolveTG;
    constexpr int KP = SolveSmem<D>::KP;
    constexpr int NJ = TG * D / kSimtThreads;   // tokens per thread in the D-parallel phase
    constexpr int NW = D / 32;                  // warps sharing a token group
    extern __shared__ __align__(16) float sm[];
    float *Ms = sm;                    // [D][KP] H_s
    float *Ks = Ms + D * KP;           // [C][KP] written keys
    float *Xc = Ks + C * KP;           // [TG][D] the vector being multiplied by A
    float *Ps = Xc + TG * D;           // [TG][C]
    float *Ws = Ps + TG * C;           // [TG][C] w_ji, 0 for i > j
    __shared__ double ell[256], wtot[kSimtThreads / 32];
    __shared__ float s_b[TG], s_lam[TG], s_d[TG], s_L[TG], s_qn[TG];
    __shared__ float red[TG][NW];

    const int tid = threadIdx.x, lane = tid & 31;
    const int j0 = blockIdx.x * TG, n = blockIdx.y, bh = blockIdx.z;
    const int jend = j0 + TG;
    const size_t tok0 = (size_t)bh * T + (size_t)n * C;
    chunk_log_prefix(beta + tok0, C, ell, wtot);
    const float *Hg = states + ((size_t)bh * (N + 1) + n) * 2 * D * D;
    for (int e = tid; e < D * D; e += kSimtThreads) Ms[(e / D) * KP + e % D] = Hg[e];
    for (int e = tid; e < jend * D; e += kSimtThreads) {
        float x = load_f(k + tok0 * D + e);
        if (gate) x *= sqrtf(gate[tok0 + e / D]);
        Ks[(e / D) * KP + e % D] = x;
    }
    if (tid < TG) {
        const float nj = norms[tok0 + j0 + tid];
        s_b[tid] = decay_exp(ell[j0 + tid]);
        s_lam[tid] = P.a * nj;
        s_d[tid] = P.half_1p2a * nj;
        s_L[tid] = (1.f + P.a) * nj;
    }
    for (int e = tid; e < TG * C; e += kSimtThreads) {
        const int jj = e / C, i = e % C;
        Ws[e] = (i <= j0 + jj) ? decay_exp(ell[j0 + jj] - ell[i]) : 0.f;
    }

    const int c = tid % D, jg = tid / D, w_in = (tid % D) >> 5;
    // per-token sums over the D columns of the thread's tokens (all threads call it)
    auto token_sums = [&](float (&v)[NJ]) {
#pragma unroll
        for (int u = 0; u < NJ; ++u) {
            const float s = warp_sum(v[u]);
            if (lane == 0) red[jg * NJ + u][w_in] = s;
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < NJ; ++u) {
            float s = 0.f;
#pragma unroll
            for (int w = 0; w < NW; ++w) s += red[jg * NJ + u][w];
            v[u] = s;
        }
        __syncthreads();
    };
    // out[u] = (A v)[c] of token jg*NJ + u for the vector v (this thread's elements
    // vin[u]; the whole vectors go through Xc)
    auto apply_A = [&](const float (&vin)[NJ], float (&out)[NJ]) {
#pragma unroll
        for (int u = 0; u < NJ; ++u) Xc[(jg * NJ + u) * D + c] = vin[u];
        __syncthreads();
        for (int p = tid; p < TG * jend; p += kSimtThreads) {
            const int jj = p / jend, i = p % jend;
            Ps[jj * C + i] = Ws[jj * C + i] * dot4<D>(Ks + i * KP, Xc + jj * D);
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < NJ; ++u) out[u] = 0.f;
        for (int d = 0; d < D; d += 4) {
            float h[4];
#pragma unroll
            for (int s = 0; s < 4; ++s) h[s] = Ms[(d + s) * KP + c];
#pragma unroll
            for (int u = 0; u < NJ; ++u) {
                const float4 x4 = *reinterpret_cast<const float4 *>(Xc + (jg * NJ + u) * D + d);
                out[u] = fmaf(h[0], x4.x, fmaf(h[1], x4.y, fmaf(h[2], x4.z, fmaf(h[3], x4.w, out[u]))));
            }
        }
#pragma unroll
        for (int u = 0; u < NJ; ++u) out[u] *= s_b[jg * NJ + u];
        for (int i = 0; i < jend; i += 4) {
            float kv[4];
#pragma unroll
            for (int s = 0; s < 4; ++s) kv[s] = Ks[(i + s) * KP + c];
#pragma unroll
            for (int u = 0; u < NJ; ++u) {
                const float4 p4 = *reinterpret_cast<const float4 *>(Ps + (jg * NJ + u) * C + i);
                out[u] = fmaf(kv[0], p4.x, fmaf(kv[1], p4.y, fmaf(kv[2], p4.z, fmaf(kv[3], p4.w, out[u]))));
            }
        }
#pragma unroll
        for (int u = 0; u < NJ; ++u) out[u] = fmaf(s_lam[jg * NJ + u], vin[u], out[u]);
        __syncthreads();   // Xc and Ps free again
    };
    // record ||q - A x|| / ||q|| for step i
    auto record = [&](const float (&qv)[NJ], const float (&ax)[NJ], int i) {
        float e2[NJ];
#pragma unroll
        for (int u = 0; u < NJ; ++u) {
            const float rr = qv[u] - ax[u];
            e2[u] = rr * rr;
        }
        token_sums(e2);
        if (c == 0) {
#pragma unroll
            for (int u = 0; u < NJ; ++u) {
                const int jj = jg * NJ + u;
                const bool live = s_qn[jj] > 0.f && s_lam[jj] > 0.f;
                resid[(tok0 + j0 + jj) * (size_t)(P.r + 1) + i] = live ? sqrtf(e2[u]) / s_qn[jj] : 0.f;
            }
        }
    };

    float qv[NJ], x[NJ], xp[NJ], ax[NJ], axp[NJ];
#pragma unroll
    for (int u = 0; u < NJ; ++u) {
        qv[u] = load_f(q + (tok0 + j0 + jg * NJ + u) * D + c);
        x[u] = xp[u] = ax[u] = axp[u] = 0.f;
    }
    {
        float q2[NJ];
#pragma unroll
        for (int u = 0; u < NJ; ++u) q2[u] = qv[u] * qv[u];
        __syncthreads();   // s_* complete before token_sums' barriers
        token_sums(q2);
        if (c == 0)
#pragma unroll
            for (int u = 0; u < NJ; ++u) s_qn[jg * NJ + u] = sqrtf(q2[u]);
        __syncthreads();
    }
    record(qv, ax, 0);
    const float kap = (1.f + P.a) / P.a;
    const float mom = (sqrtf(kap) - 1.f) / (sqrtf(kap) + 1.f);
    float rv[NJ], pv[NJ], rs[NJ];
    if (SOLVER == 3) {
#pragma unroll
        for (int u = 0; u < NJ; ++u) rv[u] = pv[u] = rs[u] = qv[u] * qv[u];
        token_sums(rs);
#pragma unroll
        for (int u = 0; u < NJ; ++u) rv[u] = pv[u] = qv[u];
    }
#pragma unroll 1
    for (int it = 0; it < P.r; ++it) {
        if (SOLVER == 0) {
            // Chebyshev: x_1 = q / d, then the three-term update from A x_it
#pragma unroll
            for (int u = 0; u < NJ; ++u) {
                const int jj = jg * NJ + u;
                const float invd = s_d[jj] > 0.f ? 1.f / s_d[jj] : 0.f;
                const float xn = it == 0 ? qv[u] * invd
                                         : fmaf(P.omega[it], fmaf(qv[u] - ax[u], invd, x[u] - xp[u]), xp[u]);
                xp[u] = x[u];
                x[u] = xn;
            }
        } else if (SOLVER == 1) {
#pragma unroll
            for (int u = 0; u < NJ; ++u) {
                const int jj = jg * NJ + u;
                const float invd = s_d[jj] > 0.f ? 1.f / s_d[jj] : 0.f;
                x[u] = fmaf(qv[u] - ax[u], invd, x[u]);
            }
        } else if (SOLVER == 2) {
            // y = x + m (x - x_prev); A y by linearity from the stored products
#pragma unroll
            for (int u = 0; u < NJ; ++u) {
                const int jj = jg * NJ + u;
                const float invL = s_L[jj] > 0.f ? 1.f / s_L[jj] : 0.f;
                const float y = fmaf(mom, x[u] - xp[u], x[u]);
                const float ay = fmaf(mom, ax[u] - axp[u], ax[u]);
                xp[u] = x[u];
                x[u] = fmaf(qv[u] - ay, invL, y);
            }
        } else {
            // conjugate gradient: alpha = r.r / p.Ap, beta = r'.r' / r.r
            float ap[NJ], pap[NJ];
            apply_A(pv, ap);
#pragma unroll
            for (int u = 0; u < NJ; ++u) pap[u] = pv[u] * ap[u];
            token_sums(pap);
            float rs1[NJ];
#pragma unroll
            for (int u = 0; u < NJ; ++u) {
                const float alpha = pap[u] > 0.f ? rs[u] / pap[u] : 0.f;
                x[u] = fmaf(alpha, pv[u], x[u]);
                rv[u] = fmaf(-alpha, ap[u], rv[u]);
                rs1[u] = rv[u] * rv[u];
            }
            token_sums(rs1);
#pragma unroll
            for (int u = 0; u < NJ; ++u) {
                const float bt = rs[u] > 0.f ? rs1[u] / rs[u] : 0.f;
                pv[u] = fmaf(bt, pv[u], rv[u]);
                rs[u] = rs1[u];
            }
        }
        // the new iterate's product and true residual
#pragma unroll
        for (int u = 0; u < NJ; ++u) axp[u] = ax[u];
        apply_A(x, ax);
        record(qv, ax, it + 1);
    }
}

}  // namespace gka
