// Chunk-wise backward pass of the GKA layer on CUDA cores (fp32 arithmetic).
//
// Method: "Gated KalmaNet" (arXiv 2511.21016).  ai.info page, Key
// Contributions 3 and Methodology: the backward uses implicit differentiation
// through the linear system the Chebyshev iteration approximately solves, and
// reuses the iteration on the upstream gradient; Main Findings: Lemma 2
// (dq_t = dq^_t) and the full intra-chunk interaction of the backward;
// pith.science appendix, Eq. 50 (the key gradient with its ||H_t||_F term).
//
// Per token t, with x_t the forward iterate, g_t = dL/do_t and
// A_t = H_t + a ||H_t||_F I:
//   y_t = Chebyshev(A_t, M_t^T g_t),  dq_t = y_t,  c_t = a (y_t . x_t) / ||H_t||_F,
//   G^H_t = dL/dH_t = -y_t x_t^T - c_t H_t,   G^M_t = dL/dM_t = g_t x_t^T,
// and the adjoint states Hb_t = G^H_t + beta_{t+1} Hb_{t+1} (Mb likewise) give
//   dk_t = w_t ((Hb_t + Hb_t^T) k_t + Mb_t^T v_t),  dv_t = w_t Mb_t k_t,
//   dbeta_t = <Hb_t, H_{t-1}> + <Mb_t, M_{t-1}>,  dw_t = k_t^T Hb_t k_t + v_t^T Mb_t k_t
// (w_t the write gate; 1 without one).  Chunk form, positions j = 0..C-1 of a
// chunk with start state (H_s, M_s), chunk-relative decays b_j = exp(l_j) and
// w_{sj} = exp(l_s - l_j) (s >= j), written keys and values k~_i = sqrt(w_i) k_i,
// v~_i = sqrt(w_i) v_i:
//   - the adjoint arriving at the chunk's last token from later chunks, E_n, obeys
//     E_{n-1} = b_{C-1} E_n + dE_n with dE_n = sum_s b_s G_s, where
//     sum_s b_s c_s H_s = (sum_s b_s^2 c_s) H_s + sum_i e_i k~_i k~_i^T,
//     e_i = sum_{s>=i} b_s c_s w_si;
//   - within the chunk Hb_j = sum_{s>=j} w_sj G_s + w_{C-1,j} E_n.  The H_s-term
//     of G expands through H_s = b_s H_start + sum_{i<=s} w_si k~_i k~_i^T into
//     products with the C x C interaction matrix
//     Mw[l][i] = sum_{s>=max(i,l)} c_s w_sl w_si = R_m w_ml w_mi (m = max(i,l),
//     R_m = sum_{s>=m} c_s w_sm^2), which is full rather than triangular;
//   - dbeta_j = <Hb_j, H_{j-1}> + <Mb_j, M_{j-1}> is evaluated directly (no
//     division by beta, so resets are exact) through prefix recurrences over
//     the C x C dot-product matrices.
// Kernels (grid over chunks and heads; chunk C = 16 or 32):
//   k_bwd_solve    u = M^T g and the Chebyshev solve for y; dq, c
//   k_bwd_delta    dE_n per chunk
//   k_adjoint_scan E_n from the dE_n, last chunk first
//   k_bwd_rows     the products of the chunk's rows with H_s, M_s, E^H, E^M
//   k_bwd_grads    dk, dv, dbeta, dw of the chunk's tokens
#pragma once

#include "chunk_simt.cuh"
#include "common.cuh"
#include "ptx.cuh"

namespace gka {

// ---------------------------------------------------------------------------
// k_bwd_solve: for TG tokens of a chunk, u_j = M_j^T g_j = b_j M_s^T g_j +
// sum_{i<=j} w_ji k~_i (v~_i . g_j), then y_j = r-step Chebyshev for
// A_j y = u_j (the forward's iteration with q replaced by u).  Writes dq = y
// (input dtype), y (fp32, for the next kernels) and c_j = a (y_j . x_j) / n_j.
// grid (C/TG, N, B*H), block 256, shared memory SolveSmem<D>::bytes(C).
// ---------------------------------------------------------------------------
template <typename Tin, int D>
__global__ void __launch_bounds__(kSimtThreads)
k_bwd_solve(const Tin *__restrict__ k, const Tin *__restrict__ v, const float *__restrict__ beta,
            const float *__restrict__ gate, const Tin *__restrict__ dout,
            const float *__restrict__ states, const float *__restrict__ norms,
            const float *__restrict__ xs, Tin *__restrict__ dq, float *__restrict__ ys,
            float *__restrict__ cvec, Tin *__restrict__ u_out, int T, int N, int C,
            const ChebParams P) {
    constexpr int TG = kSolveTG;
    constexpr int KP = SolveSmem<D>::KP;
    constexpr int NJ = TG * D / kSimtThreads;
    extern __shared__ __align__(16) float sm[];
    float *Ms = sm;                    // [D][KP]: M_s, then H_s
    float *Ks = Ms + D * KP;           // [C][KP]: written values, then written keys
    float *Xc = Ks + C * KP;           // [TG][D] g, then the current iterate
    float *Xp = Xc + TG * D;           // [TG][D] previous iterate
    float *Qs = Xp + TG * D;           // [TG][D] u
    float *Ps = Qs + TG * D;           // [TG][C]
    float *Ws = Ps + TG * C;           // [TG][C] w_ji, 0 for i > j
    __shared__ double ell[256], wtot[kSimtThreads / 32];
    __shared__ float s_b[TG], s_lam[TG], s_invd[TG];

    const int tid = threadIdx.x;
    const int j0 = blockIdx.x * TG, n = blockIdx.y, bh = blockIdx.z;
    const int jend = j0 + TG;
    const size_t tok0 = (size_t)bh * T + (size_t)n * C;
    chunk_log_prefix(beta + tok0, C, ell, wtot);

    const float *Sg = states + ((size_t)bh * (N + 1) + n) * 2 * D * D;   // H_s, then M_s
    auto load_rows = [&](const Tin *src) {
        for (int e = tid; e < jend * D; e += kSimtThreads) {
            float x = load_f(src + tok0 * D + e);
            if (gate) x *= sqrtf(gate[tok0 + e / D]);
            Ks[(e / D) * KP + e % D] = x;
        }
    };
    for (int e = tid; e < D * D; e += kSimtThreads) Ms[(e / D) * KP + e % D] = Sg[D * D + e];
    load_rows(v);
    for (int e = tid; e < TG * D; e += kSimtThreads) Xc[e] = load_f(dout + (tok0 + j0) * D + e);
    if (tid < TG) {
        const float nj = norms[tok0 + j0 + tid];
        s_b[tid] = decay_exp(ell[j0 + tid]);
        s_lam[tid] = P.a * nj;
        s_invd[tid] = nj > 0.f ? 1.f / (P.half_1p2a * nj) : 0.f;
    }
    __syncthreads();
    for (int e = tid; e < TG * C; e += kSimtThreads) {
        const int jj = e / C, i = e % C;
        Ws[e] = (i <= j0 + jj) ? decay_exp(ell[j0 + jj] - ell[i]) : 0.f;
    }
    __syncthreads();

    const int c = tid % D, jg = tid / D;
    auto form_p = [&]() {
        for (int p = tid; p < TG * jend; p += kSimtThreads) {
            const int jj = p / jend, i = p % jend;
            Ps[jj * C + i] = Ws[jj * C + i] * dot4<D>(Ks + i * KP, Xc + jj * D);
        }
    };
    // acc[u] = b_j sum_d Ms[d][c] x_j[d] + sum_i P[j][i] Ks[i][c]
    auto apply = [&](float (&acc)[NJ]) {
#pragma unroll
        for (int u = 0; u < NJ; ++u) acc[u] = 0.f;
        for (int d = 0; d < D; d += 4) {
            float h[4];
#pragma unroll
            for (int s = 0; s < 4; ++s) h[s] = Ms[(d + s) * KP + c];
#pragma unroll
            for (int u = 0; u < NJ; ++u) {
                const float4 x4 = *reinterpret_cast<const float4 *>(Xc + (jg * NJ + u) * D + d);
                acc[u] = fmaf(h[0], x4.x, fmaf(h[1], x4.y, fmaf(h[2], x4.z, fmaf(h[3], x4.w, acc[u]))));
            }
        }
#pragma unroll
        for (int u = 0; u < NJ; ++u) acc[u] *= s_b[jg * NJ + u];
        for (int i = 0; i < jend; i += 4) {
            float kv[4];
#pragma unroll
            for (int s = 0; s < 4; ++s) kv[s] = Ks[(i + s) * KP + c];
#pragma unroll
            for (int u = 0; u < NJ; ++u) {
                const float4 p4 = *reinterpret_cast<const float4 *>(Ps + (jg * NJ + u) * C + i);
                acc[u] = fmaf(kv[0], p4.x, fmaf(kv[1], p4.y, fmaf(kv[2], p4.z, fmaf(kv[3], p4.w, acc[u]))));
            }
        }
    };

    // u_j = M_j^T g_j: P = W o (V~ G^T) with the values, then M_s^T g and the keys
    form_p();
    __syncthreads();
    load_rows(k);
    __syncthreads();
    {
        float acc[NJ];
        apply(acc);
#pragma unroll
        for (int u = 0; u < NJ; ++u) Qs[(jg * NJ + u) * D + c] = acc[u];
    }
    __syncthreads();
    if (u_out) {
        // u only (the solve runs elsewhere)
        for (int e = tid; e < TG * D; e += kSimtThreads) store_f(u_out + (tok0 + j0) * D + e, Qs[e]);
        return;
    }
    for (int e = tid; e < D * D; e += kSimtThreads) Ms[(e / D) * KP + e % D] = Sg[e];
    for (int e = tid; e < TG * D; e += kSimtThreads) {
        Xc[e] = Qs[e] * s_invd[e / D];
        Xp[e] = 0.f;
    }
    __syncthreads();

#pragma unroll 1
    for (int it = 1; it < P.r; ++it) {
        form_p();
        __syncthreads();
        float acc[NJ];
        apply(acc);
        const float w = P.omega[it];
        float xn[NJ];
#pragma unroll
        for (int u = 0; u < NJ; ++u) {
            const int jj = jg * NJ + u;
            const float xc = Xc[jj * D + c], xp = Xp[jj * D + c];
            const float yv = fmaf(s_lam[jj], xc, acc[u]);
            xn[u] = fmaf(w, fmaf(Qs[jj * D + c] - yv, s_invd[jj], xc - xp), xp);
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < NJ; ++u) {
            const int jj = jg * NJ + u;
            Xp[jj * D + c] = Xc[jj * D + c];
            Xc[jj * D + c] = xn[u];
        }
        __syncthreads();
    }
    for (int e = tid; e < TG * D; e += kSimtThreads) {
        const size_t g = (tok0 + j0) * D + e;
        ys[g] = Xc[e];
        store_f(dq + g, Xc[e]);
    }
    // c_j = a (y_j . x_j) / n_j, one warp per token
    const int lane = tid & 31, warp = tid >> 5;
    for (int jj = warp; jj < TG; jj += kSimtThreads / 32) {
        float s = 0.f;
        for (int d = lane; d < D; d += 32) s = fmaf(Xc[jj * D + d], xs[(tok0 + j0 + jj) * D + d], s);
        s = warp_sum(s);
        if (lane == 0) {
            const float nj = norms[tok0 + j0 + jj];
            cvec[tok0 + j0 + jj] = nj > 0.f ? P.a * s / nj : 0.f;
        }
    }
}

// ---------------------------------------------------------------------------
// k_bwd_yfinish: after an adjoint solve done elsewhere (y in ys), dq = y and
// c_t = a (y_t . x_t) / n_t.  One warp per token; grid ceil(tokens / 8), block 256.
// ---------------------------------------------------------------------------
template <typename Tin, int D>
__global__ void __launch_bounds__(kSimtThreads)
k_bwd_yfinish(const float *__restrict__ ys, const float *__restrict__ xs,
              const float *__restrict__ norms, Tin *__restrict__ dq, float *__restrict__ cvec,
              size_t tokens, float a) {
    const int lane = threadIdx.x & 31;
    const size_t t = (size_t)blockIdx.x * (kSimtThreads / 32) + (threadIdx.x >> 5);
    if (t >= tokens) return;
    float s = 0.f;
    for (int d = lane; d < D; d += 32) {
        const float y = ys[t * D + d];
        s = fmaf(y, xs[t * D + d], s);
        store_f(dq + t * D + d, y);
    }
    s = warp_sum(s);
    if (lane == 0) {
        const float n = norms[t];
        cvec[t] = n > 0.f ? a * s / n : 0.f;
    }
}

// Decays of one chunk from its cumulative logs: b_j, the one-step factor beta_j
// and w_{C-1,j} (thread j < C).
struct ChunkDecays {
    float b, step, wend;
};
__device__ __forceinline__ ChunkDecays chunk_decays(const double *ell, int C, int j) {
    ChunkDecays r;
    r.b = decay_exp(ell[j]);
    r.step = decay_exp(j == 0 ? ell[0] : ell[j] - ell[j - 1]);
    r.wend = decay_exp(ell[C - 1] - ell[j]);
    return r;
}

// ---------------------------------------------------------------------------
// k_bwd_delta: dE_n = sum_s b_s G_s of one chunk, into adjoint slot n:
//   dE^H = -(b o Y)^T X - (sum_s b_s^2 c_s) H_start - (e o K~)^T K~,
//   dE^M = (b o G)^T X,   e_i = sum_{s>=i} b_s c_s w_si.
// grid (N, B*H), block 256, shared memory 5 * C * D floats.
// ---------------------------------------------------------------------------
template <typename Tin, int D>
__global__ void __launch_bounds__(kSimtThreads)
k_bwd_delta(const Tin *__restrict__ k, const float *__restrict__ beta,
            const float *__restrict__ gate, const Tin *__restrict__ dout,
            const float *__restrict__ states, const float *__restrict__ xs,
            const float *__restrict__ ys, const float *__restrict__ cvec,
            float *__restrict__ adj, int T, int N, int C) {
    extern __shared__ __align__(16) float sm[];
    float *Ya = sm;              // [C][D] -b_s y_s
    float *Xs = Ya + C * D;      // [C][D] x_s
    float *Ka = Xs + C * D;      // [C][D] -e_i k~_i
    float *Kw = Ka + C * D;      // [C][D] k~_i
    float *Ga = Kw + C * D;      // [C][D] b_s g_s
    __shared__ double ell[256], wtot[kSimtThreads / 32];
    __shared__ float s_b[64], s_e[64], s_c1;

    const int n = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const size_t tok0 = (size_t)bh * T + (size_t)n * C;
    chunk_log_prefix(beta + tok0, C, ell, wtot);
    if (tid == 0) {
        // e_i by the suffix recurrence e_i = b_i c_i + beta_{i+1} e_{i+1}
        float e = 0.f, c1 = 0.f;
        for (int i = C - 1; i >= 0; --i) {
            const ChunkDecays dc = chunk_decays(ell, C, i);
            const float bc = dc.b * cvec[tok0 + i];
            const float nxt = i + 1 < C ? decay_exp(ell[i + 1] - ell[i]) : 0.f;
            e = fmaf(nxt, e, bc);
            s_e[i] = e;
            s_b[i] = dc.b;
            c1 = fmaf(dc.b, bc, c1);
        }
        s_c1 = c1;
    }
    __syncthreads();
    for (int e = tid; e < C * D; e += kSimtThreads) {
        const int i = e / D;
        const size_t g = tok0 * D + e;
        float kv = load_f(k + g);
        if (gate) kv *= sqrtf(gate[tok0 + i]);
        Ya[e] = -s_b[i] * ys[g];
        Xs[e] = xs[g];
        Ka[e] = -s_e[i] * kv;
        Kw[e] = kv;
        Ga[e] = s_b[i] * load_f(dout + g);
    }
    __syncthreads();

    constexpr int TS = D / 16;
    const int tx = tid & 15, ty = tid >> 4;
    const float *Hst = states + ((size_t)bh * (N + 1) + n) * 2 * D * D;
    float *out = adj + ((size_t)bh * (N + 1) + n) * 2 * D * D;
#pragma unroll 1
    for (int mat = 0; mat < 2; ++mat) {
        float acc[TS][TS];
#pragma unroll
        for (int u = 0; u < TS; ++u)
#pragma unroll
            for (int w = 0; w < TS; ++w) acc[u][w] = 0.f;
        const float *R1 = mat == 0 ? Ya : Ga;
        for (int i = 0; i < C; ++i) {
            float ra[TS], cb[TS];
#pragma unroll
            for (int u = 0; u < TS; ++u) {
                ra[u] = R1[i * D + ty * TS + u];
                cb[u] = Xs[i * D + tx * TS + u];
            }
#pragma unroll
            for (int u = 0; u < TS; ++u)
#pragma unroll
                for (int w = 0; w < TS; ++w) acc[u][w] = fmaf(ra[u], cb[w], acc[u][w]);
        }
        if (mat == 0) {
            for (int i = 0; i < C; ++i) {
                float ra[TS], cb[TS];
#pragma unroll
                for (int u = 0; u < TS; ++u) {
                    ra[u] = Ka[i * D + ty * TS + u];
                    cb[u] = Kw[i * D + tx * TS + u];
                }
#pragma unroll
                for (int u = 0; u < TS; ++u)
#pragma unroll
                    for (int w = 0; w < TS; ++w) acc[u][w] = fmaf(ra[u], cb[w], acc[u][w]);
            }
        }
        float *o = out + (size_t)mat * D * D;
#pragma unroll
        for (int u = 0; u < TS; ++u)
#pragma unroll
            for (int w = 0; w < TS; ++w) {
                const size_t e = (size_t)(ty * TS + u) * D + tx * TS + w;
                o[e] = mat == 0 ? fmaf(-s_c1, Hst[e], acc[u][w]) : acc[u][w];
            }
    }
}

// ---------------------------------------------------------------------------
// k_adjoint_scan: in place over the adjoint slots of a head, last chunk first:
//   E_{N-1} = 0,  E_{n-1} = b_n E_n + dE_n   (slot n: dE_n in, E_n out).
// grid (ceil(2*D*D / 1024), B*H), block 256, 4 elements per thread.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
k_adjoint_scan(float *__restrict__ adj, const float *__restrict__ decay, int N, int DD2) {
    const int bh = blockIdx.y;
    const int e = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (e >= DD2) return;
    float *base = adj + (size_t)bh * (N + 1) * DD2 + e;
    const float *dec = decay + (size_t)bh * N;
    float4 carry = make_float4(0.f, 0.f, 0.f, 0.f);
    // the loads of a batch of 8 slots are issued before the dependent stores
    for (int n1 = N - 1; n1 >= 0; n1 -= 8) {
        const int nb = n1 >= 7 ? 8 : n1 + 1;
        float4 d[8];
        float b[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (u < nb) {
                d[u] = __ldcs(reinterpret_cast<const float4 *>(base + (size_t)(n1 - u) * DD2));
                b[u] = dec[n1 - u];
            }
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (u < nb) {
                *reinterpret_cast<float4 *>(base + (size_t)(n1 - u) * DD2) = carry;
                carry.x = fmaf(b[u], carry.x, d[u].x);
                carry.y = fmaf(b[u], carry.y, d[u].y);
                carry.z = fmaf(b[u], carry.z, d[u].z);
                carry.w = fmaf(b[u], carry.w, d[u].w);
            }
    }
}

// ---------------------------------------------------------------------------
// k_bwd_rows: products of a chunk's rows (its own, unwritten keys and values,
// iterates and gradients) with the chunk's D x D matrices:
//   R1_t = H_s k_t,  R2_t = (E^H + E^H^T) k_t,  R3_t = E^M^T v_t,  R4_t = E^M k_t
//   (rows of [B*H*T, D] each), and per token uk_t = k_t^T H_s k_t,
//   yhx_t = y_t^T H_s x_t, gmx_t = g_t^T M_s x_t, qe_t = k_t^T E^H k_t + v_t^T E^M k_t;
//   per chunk hs2 = ||H_s||_F^2 and eh = <E^H, H_s> + <E^M, M_s>.
// Every product is out[t][c] = sum_d row_t[d] Mt[d][c], the matrix staged in
// shared memory half a column range at a time in the orientation the product
// needs (E^M transposed for R4, E^H symmetrised for R2).  Warp w computes tokens
// w*C/8.., lane l the columns l and l + 32 of the half, in registers; the
// per-token dots are reduced from the registers.  k, v and g rows are kept as
// their bf16 values when the inputs are bf16 (exact).
// grid (N, B*H), block 256, shared memory BwdRowsSmem<Tin, D, C>::bytes (two CTAs
// per SM at D = 128, C = 32).
// ---------------------------------------------------------------------------
template <typename Tin, int D, int C>
struct BwdRowsSmem {
    static constexpr int NH = D >= 64 ? 2 : 1;   // column ranges staged one after another
    static constexpr int HC = D / NH;            // columns per staged range
    static constexpr int DP = HC + 4;         // 16-byte aligned rows
    static constexpr size_t mat = sizeof(float) * (size_t)D * DP;
    static constexpr size_t in_rows = sizeof(Tin) * (size_t)C * D;     // k, v, g
    static constexpr size_t f_rows = sizeof(float) * (size_t)C * D;    // x, y
    static constexpr size_t bytes = mat + 3 * in_rows + 2 * f_rows;
};

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

// Mt[d][c'] = A'[d][h*HC + c'] for the column range h, A' = A (mode 0), A^T (1),
// A + A^T (2); global reads are coalesced in every mode.  All threads call it.
template <int D, int HC, int DP>
__device__ __forceinline__ void bwd_stage(float *Mt, const float *__restrict__ A, int mode, int h) {
    const int tid = threadIdx.x;
    __syncthreads();
    if (mode != 1) {
        for (int e = tid; e < D * HC; e += kSimtThreads) {
            const int d = e / HC, c = e % HC;
            Mt[d * DP + c] = A[d * D + h * HC + c];
        }
    }
    if (mode == 2) __syncthreads();
    if (mode != 0) {
        for (int e = tid; e < HC * D; e += kSimtThreads) {
            const int c = e / D, d = e % D;
            const float x = A[(h * HC + c) * D + d];
            Mt[d * DP + c] = mode == 2 ? Mt[d * DP + c] + x : x;
        }
    }
    __syncthreads();
}

// For the column range h staged in Mt: out[t][h*HC + c] = sum_d rows[t][d] Mt[d][c]
// over this warp's TT tokens and this lane's CC columns; written to R + gout (if
// gout != -1) and its dot with dotB[t][.] added to dacc.
template <int D, int HC, int DP, int TT, typename RowT, typename DotT>
__device__ __forceinline__ void bwd_half_product(const float *Mt, const RowT *rows,
                                                 const DotT *dotB, int h, float *__restrict__ R,
                                                 size_t gout, size_t tok0, float (&dacc)[TT]) {
    constexpr int CC = HC / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float acc[TT][CC];
#pragma unroll
    for (int a = 0; a < TT; ++a)
#pragma unroll
        for (int b = 0; b < CC; ++b) acc[a][b] = 0.f;
    const int t0 = warp * TT;
#pragma unroll 2
    for (int d = 0; d < D; d += 4) {
        float m[4][CC];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int b = 0; b < CC; ++b) m[u][b] = Mt[(d + u) * DP + lane + 32 * b];
#pragma unroll
        for (int a = 0; a < TT; ++a) {
            float r[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) r[u] = to_f(rows[(t0 + a) * D + d + u]);
#pragma unroll
            for (int b = 0; b < CC; ++b)
                acc[a][b] = fmaf(r[0], m[0][b], fmaf(r[1], m[1][b],
                            fmaf(r[2], m[2][b], fmaf(r[3], m[3][b], acc[a][b]))));
        }
    }
#pragma unroll
    for (int a = 0; a < TT; ++a)
#pragma unroll
        for (int b = 0; b < CC; ++b) {
            const int p = (t0 + a) * D + h * HC + lane + 32 * b;
            if (gout != (size_t)-1) R[gout + tok0 * D + p] = acc[a][b];
            dacc[a] = fmaf(acc[a][b], to_f(dotB[p]), dacc[a]);
        }
}

// One product over all column ranges; the per-token dot (times scale) written to
// dst[tok0 + t] (or added), unless dst is null.
template <int D, int HC, int DP, int NH, int TT, typename RowT, typename DotT>
__device__ __forceinline__ void bwd_product(float *Mt, const float *__restrict__ A, int mode,
                                            const RowT *rows, size_t gout, const DotT *dotB,
                                            float *dst, float scale, bool add,
                                            float *__restrict__ R, size_t tok0) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float dacc[TT];
#pragma unroll
    for (int a = 0; a < TT; ++a) dacc[a] = 0.f;
    for (int h = 0; h < NH; ++h) {
        bwd_stage<D, HC, DP>(Mt, A, mode, h);
        bwd_half_product<D, HC, DP, TT>(Mt, rows, dotB, h, R, gout, tok0, dacc);
    }
#pragma unroll
    for (int a = 0; a < TT; ++a) {
        const float s = warp_sum(dacc[a]) * scale;
        if (dst && lane == 0) {
            const size_t t = tok0 + warp * TT + a;
            dst[t] = add ? dst[t] + s : s;
        }
    }
}

template <typename Tin, int D, int C>
__global__ void __launch_bounds__(kSimtThreads, 2)
k_bwd_rows(const Tin *__restrict__ k, const Tin *__restrict__ v, const Tin *__restrict__ dout,
           const float *__restrict__ states, const float *__restrict__ adj,
           const float *__restrict__ xs, const float *__restrict__ ys, float *__restrict__ R,
           float *__restrict__ tokq, float *__restrict__ chq, int T, int N) {
    using L = BwdRowsSmem<Tin, D, C>;
    constexpr int HC = L::HC, DP = L::DP, NH = L::NH;
    constexpr int TT = C / 8;          // tokens per warp
    static_assert(kSimtThreads == 256 && C % 8 == 0 && HC % 32 == 0, "tiling");
    extern __shared__ __align__(16) uint8_t smb[];
    float *Mt = reinterpret_cast<float *>(smb);                       // [D][DP] staged columns
    Tin *Kr = reinterpret_cast<Tin *>(smb + L::mat);                  // [C][D] k_t
    Tin *Vr = Kr + C * D;                                             // [C][D] v_t
    Tin *Gr = Vr + C * D;                                             // [C][D] g_t
    float *Xr = reinterpret_cast<float *>(smb + L::mat + 3 * L::in_rows);   // [C][D] x_t
    float *Yr = Xr + C * D;                                                 // [C][D] y_t
    __shared__ float red[2][kSimtThreads / 32];

    const int n = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const size_t tok0 = (size_t)bh * T + (size_t)n * C;
    const size_t plane = (size_t)gridDim.y * T;   // B*H*T
    const size_t RD = plane * D;                  // one [B*H*T, D] array
    const float *Hs = states + ((size_t)bh * (N + 1) + n) * 2 * D * D, *Mst = Hs + D * D;
    const float *EH = adj + ((size_t)bh * (N + 1) + n) * 2 * D * D, *EM = EH + D * D;
    for (int e = tid; e < C * D; e += kSimtThreads) {
        const size_t g = tok0 * D + e;
        Kr[e] = k[g];
        Vr[e] = v[g];
        Gr[e] = dout[g];
        Xr[e] = xs[g];
        Yr[e] = ys[g];
    }
    {
        float h2 = 0.f, eh = 0.f;
        for (int e = tid; e < D * D; e += kSimtThreads) {
            const float h = Hs[e];
            h2 = fmaf(h, h, h2);
            eh = fmaf(EH[e], h, fmaf(EM[e], Mst[e], eh));
        }
        h2 = warp_sum(h2);
        eh = warp_sum(eh);
        if (lane == 0) {
            red[0][warp] = h2;
            red[1][warp] = eh;
        }
    }
    __syncthreads();
    if (tid < 2) {
        float s = 0.f;
        for (int w = 0; w < kSimtThreads / 32; ++w) s += red[tid][w];
        chq[((size_t)bh * N + n) * 2 + tid] = s;
    }
    constexpr size_t none = (size_t)-1;
    // H_s (symmetric): R1 = K H_s with uk = k . R1; x^T H_s with yhx = (x^T H_s) . y
    bwd_product<D, HC, DP, NH, TT>(Mt, Hs, 0, Kr, 0, Kr, tokq, 1.f, false, R, tok0);
    bwd_product<D, HC, DP, NH, TT>(Mt, Hs, 0, Xr, none, Yr, tokq + plane, 1.f, false, R, tok0);
    // M_s: g^T M_s x = (g^T M_s) . x
    bwd_product<D, HC, DP, NH, TT>(Mt, Mst, 0, Gr, none, Xr, tokq + 2 * plane, 1.f, false, R,
                                   tok0);
    // E^H + E^H^T: R2, qe = k^T E^H k = (k . R2) / 2
    bwd_product<D, HC, DP, NH, TT>(Mt, EH, 2, Kr, RD, Kr, tokq + 3 * plane, 0.5f, false, R, tok0);
    // E^M: R3 = rows v^T E^M (its dot is not needed)
    bwd_product<D, HC, DP, NH, TT>(Mt, EM, 0, Vr, 2 * RD, Vr, (float *)nullptr, 0.f, false, R,
                                   tok0);
    // E^M^T: R4 = rows k^T E^M^T = (E^M k)^T; qe += v . R4
    bwd_product<D, HC, DP, NH, TT>(Mt, EM, 1, Kr, 3 * RD, Vr, tokq + 3 * plane, 1.f, true, R,
                                   tok0);
}

// ---------------------------------------------------------------------------
// k_bwd_grads: dk, dv, dbeta and the write-gate gradient of one chunk.
// Shared memory: the chunk's k, x, y, g rows (fp32, rows padded to 16 bytes),
// the C x C matrices, and one region that holds the v rows until their dot
// products are formed and the four coefficient matrices after.  Products run
// in register tiles: the dot-product matrices in TI x TI tiles over rows
// (l0 + 8i, s0 + 8j) (conflict-free 16-byte loads), the row outputs with a warp
// per group of tokens and a lane per group of columns.
// grid (N, B*H), block 256, shared memory BwdGradSmem<D, C>::bytes (2 CTAs per SM
// at D = 128, C = 32).
// ---------------------------------------------------------------------------
template <int D, int C>
struct BwdGradSmem {
    static constexpr int KP = D + 4;
    static constexpr int CP = C + 1;
    static constexpr size_t rows = (size_t)C * KP;
    static constexpr size_t mats = (size_t)C * CP;
    // k, x, y, g rows; v rows / Py Px Pk Pg; KX KY VG GK Wt Q
    static constexpr size_t union_floats = rows > 4 * mats ? rows : 4 * mats;
    static constexpr size_t bytes = sizeof(float) * (4 * rows + union_floats + 6 * mats);
};

template <typename Tin, int D, int C>
__global__ void __launch_bounds__(kSimtThreads, 2)
k_bwd_grads(const Tin *__restrict__ k, const Tin *__restrict__ v, const float *__restrict__ beta,
            const float *__restrict__ gate, const Tin *__restrict__ dout,
            const float *__restrict__ xs, const float *__restrict__ ys,
            const float *__restrict__ cvec, const float *__restrict__ R,
            const float *__restrict__ tokq, const float *__restrict__ chq, Tin *__restrict__ dk,
            Tin *__restrict__ dv, float *__restrict__ dbeta, float *__restrict__ dgate, int T,
            int N) {
    using L = BwdGradSmem<D, C>;
    constexpr int KP = L::KP, CP = L::CP;
    constexpr int TI = C / 8;          // dot tile edge; tokens per warp in the row outputs
    constexpr int CC = D / 32;         // columns per lane in the row outputs
    static_assert(kSimtThreads == 256 && (C == 16 || C == 32) && D % 32 == 0, "tiling");
    extern __shared__ __align__(16) float sm[];
    float *Kr = sm;                          // [C][KP] k_t (as given)
    float *Xr = Kr + L::rows;                // [C][KP] x_t
    float *Yr = Xr + L::rows;                // [C][KP] y_t
    float *Gr = Yr + L::rows;                // [C][KP] g_t = dL/do_t
    float *Un = Gr + L::rows;                // v rows, then Py Px Pk Pg
    float *Vr = Un;
    float *Py = Un, *Px = Py + L::mats, *Pk = Px + L::mats, *Pg = Pk + L::mats;
    float *KX = Un + L::union_floats;        // [C][CP] k_l . x_s
    float *KY = KX + L::mats;                // [C][CP] k_l . y_s
    float *VG = KY + L::mats;                // [C][CP] v_l . g_s
    float *GK = VG + L::mats;                // [C][CP] k_l . k_i
    float *Wt = GK + L::mats;                // [C][CP] w_sl at [l][s], 0 for s < l
    float *Qm = Wt + L::mats;                // [C][CP] Q[i][s]
    __shared__ double ell[C], wtot[kSimtThreads / 32];
    __shared__ float s_b[C], s_step[C], s_wend[C], s_w[C], s_c[C], s_f[C], s_R[C];
    __shared__ float s_uk[C], s_yhx[C], s_gmx[C], s_qe[C], s_X1[C], s_bm1[C];

    const int n = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const size_t tok0 = (size_t)bh * T + (size_t)n * C;
    const size_t plane = (size_t)gridDim.y * T;
    const size_t RD = plane * D;
    chunk_log_prefix(beta + tok0, C, ell, wtot);
    const float hs2 = chq[((size_t)bh * N + n) * 2], eh = chq[((size_t)bh * N + n) * 2 + 1];
    if (tid < C) {
        const ChunkDecays dc = chunk_decays(ell, C, tid);
        s_b[tid] = dc.b;
        s_step[tid] = dc.step;
        s_wend[tid] = dc.wend;
        s_w[tid] = gate ? gate[tok0 + tid] : 1.f;
        s_c[tid] = cvec[tok0 + tid];
        s_uk[tid] = tokq[tok0 + tid];
        s_yhx[tid] = tokq[plane + tok0 + tid];
        s_gmx[tid] = tokq[2 * plane + tok0 + tid];
        s_qe[tid] = tokq[3 * plane + tok0 + tid];
        s_bm1[tid] = tid == 0 ? 1.f : decay_exp(ell[tid - 1]);
    }
    for (int e = tid; e < C * D; e += kSimtThreads) {
        const size_t g = tok0 * D + e;
        const int t = e / D, d = e % D;
        Kr[t * KP + d] = load_f(k + g);
        Vr[t * KP + d] = load_f(v + g);
        Xr[t * KP + d] = xs[g];
        Yr[t * KP + d] = ys[g];
        Gr[t * KP + d] = load_f(dout + g);
    }
    for (int e = tid; e < C * C; e += kSimtThreads) {
        const int l = e / C, s2 = e % C;
        Wt[l * CP + s2] = s2 >= l ? decay_exp(ell[s2] - ell[l]) : 0.f;
    }
    __syncthreads();
    // dot-product matrices: 64 threads per matrix, a TI x TI tile each
    {
        const int m = tid >> 6, q = tid & 63, lt = q >> 3, st = q & 7;
        const float *A = m == 2 ? Vr : Kr;
        const float *B = m == 0 ? Xr : (m == 1 ? Yr : (m == 2 ? Gr : Kr));
        float acc[TI][TI];
#pragma unroll
        for (int i = 0; i < TI; ++i)
#pragma unroll
            for (int j = 0; j < TI; ++j) acc[i][j] = 0.f;
#pragma unroll 2
        for (int d = 0; d < D; d += 4) {
            float4 a4[TI], b4[TI];
#pragma unroll
            for (int i = 0; i < TI; ++i) {
                a4[i] = *reinterpret_cast<const float4 *>(A + (lt + 8 * i) * KP + d);
                b4[i] = *reinterpret_cast<const float4 *>(B + (st + 8 * i) * KP + d);
            }
#pragma unroll
            for (int i = 0; i < TI; ++i)
#pragma unroll
                for (int j = 0; j < TI; ++j)
                    acc[i][j] = fmaf(a4[i].x, b4[j].x, fmaf(a4[i].y, b4[j].y,
                                fmaf(a4[i].z, b4[j].z, fmaf(a4[i].w, b4[j].w, acc[i][j]))));
        }
        float *dst = m == 0 ? KX : (m == 1 ? KY : (m == 2 ? VG : GK));
#pragma unroll
        for (int i = 0; i < TI; ++i)
#pragma unroll
            for (int j = 0; j < TI; ++j) dst[(lt + 8 * i) * CP + st + 8 * j] = acc[i][j];
    }
    if (tid == 0) {
        // f_l = sum_{s>=l} w_sl c_s b_s and R_m = sum_{s>=m} c_s w_sm^2 (suffix recurrences)
        float f = 0.f, Rm = 0.f;
        for (int l = C - 1; l >= 0; --l) {
            const float nxt = l + 1 < C ? s_step[l + 1] : 0.f;
            f = fmaf(nxt, f, s_c[l] * s_b[l]);
            Rm = fmaf(nxt * nxt, Rm, s_c[l]);
            s_f[l] = f;
            s_R[l] = Rm;
        }
        // X1_s = sum_{l<=s} w_sl w_l uk_l (the written keys' H_s quadratic forms)
        float x1 = 0.f;
        for (int s2 = 0; s2 < C; ++s2) {
            x1 = fmaf(s2 == 0 ? 0.f : s_step[s2], x1, s_w[s2] * s_uk[s2]);
            s_X1[s2] = x1;
        }
    }
    __syncthreads();   // dot matrices complete; the v rows are dead from here on
    // coefficient matrices of the row outputs (over the v rows)
    for (int e = tid; e < C * C; e += kSimtThreads) {
        const int l = e / C, s2 = e % C;
        const float w = Wt[l * CP + s2];
        Py[l * CP + s2] = -w * KX[l * CP + s2];
        Px[l * CP + s2] = w * (VG[l * CP + s2] - KY[l * CP + s2]);
        Pg[l * CP + s2] = w * KX[l * CP + s2];
        // Mw[l][i] = R_m w_ml w_mi, m = max(l, i); here i = s2
        const int m = l > s2 ? l : s2;
        Pk[l * CP + s2] = -2.f * s_R[m] * Wt[l * CP + m] * Wt[s2 * CP + m] * s_w[s2] * GK[l * CP + s2];
    }
    // Q[i][s] = sum_{l<=s} w_sl w_l w_i (k_l . k_i)^2, thread i over s
    if (tid < C) {
        const int i = tid;
        float qv = 0.f;
        for (int s2 = 0; s2 < C; ++s2) {
            const float g2 = GK[s2 * CP + i];
            qv = fmaf(s2 == 0 ? 0.f : s_step[s2], qv, s_w[s2] * s_w[i] * g2 * g2);
            Qm[i * CP + s2] = qv;
        }
    }
    __syncthreads();
    // row outputs: warp w takes tokens w + 8i, lane the columns lane + 32b
    {
        float a0[TI][CC], b0[TI][CC];
#pragma unroll
        for (int i = 0; i < TI; ++i)
#pragma unroll
            for (int b = 0; b < CC; ++b) a0[i][b] = b0[i][b] = 0.f;
#pragma unroll 4
        for (int s2 = 0; s2 < C; ++s2) {
            float yv[CC], xv[CC], kv[CC], gv[CC];
#pragma unroll
            for (int b = 0; b < CC; ++b) {
                const int c = lane + 32 * b;
                yv[b] = Yr[s2 * KP + c];
                xv[b] = Xr[s2 * KP + c];
                kv[b] = Kr[s2 * KP + c];
                gv[b] = Gr[s2 * KP + c];
            }
#pragma unroll
            for (int i = 0; i < TI; ++i) {
                const int l = warp + 8 * i;
                const float py = Py[l * CP + s2], px = Px[l * CP + s2], pk = Pk[l * CP + s2],
                            pg = Pg[l * CP + s2];
#pragma unroll
                for (int b = 0; b < CC; ++b) {
                    a0[i][b] = fmaf(py, yv[b], fmaf(px, xv[b], fmaf(pk, kv[b], a0[i][b])));
                    b0[i][b] = fmaf(pg, gv[b], b0[i][b]);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < TI; ++i) {
            const int l = warp + 8 * i;
            const size_t row = (tok0 + l) * D;
            float dgp = 0.f;
#pragma unroll
            for (int b = 0; b < CC; ++b) {
                const int c = lane + 32 * b;
                const size_t g = row + c;
                float a = fmaf(-2.f * s_f[l], R[g], a0[i][b]);
                a = fmaf(s_wend[l], R[RD + g] + R[2 * RD + g], a);
                const float bb = fmaf(s_wend[l], R[3 * RD + g], b0[i][b]);
                store_f(dk + g, s_w[l] * a);
                store_f(dv + g, s_w[l] * bb);
                dgp = fmaf(Kr[l * KP + c], a, fmaf(load_f(v + g), bb, dgp));
            }
            // write-gate gradient: (k . A0 + v . B0) / 2 over the row
            dgp = warp_sum(dgp);
            if (dgate && lane == 0) dgate[tok0 + l] = 0.5f * dgp;
        }
    }
    // dbeta_j = sum_{s>=j} w_sj Phi[j][s] + (adjoint from later chunks), with
    //   Phi[j][s] = -y_s^T H_{j-1} x_s - c_s <H_s, H_{j-1}> + g_s^T M_{j-1} x_s
    // (H_s here the state at token s, H_{j-1} the one before token j, H_{-1} = H_start).
    // Thread s runs the prefix recurrences over j <= s (reading column s of the dot
    // matrices and of Q) and stores w_sj Phi[j][s] into Py[j][s] (free by now).
    __syncthreads();
    if (tid < C) {
        const int s2 = tid;
        float t1 = 0.f, t2 = 0.f, t3 = 0.f, u1 = 0.f;
        for (int j = 0; j <= s2; ++j) {
            if (j > 0) {
                const int i = j - 1;
                const float st = s_step[i];
                t1 = fmaf(st, t1, s_w[i] * KY[i * CP + s2] * KX[i * CP + s2]);
                t3 = fmaf(st, t3, s_w[i] * VG[i * CP + s2] * KX[i * CP + s2]);
                t2 = fmaf(st, t2, Qm[i * CP + s2]);
                u1 = fmaf(st, u1, s_w[i] * s_uk[i]);
            }
            const float bm = s_bm1[j];
            const float phi = -(bm * s_yhx[s2] + t1)
                              - s_c[s2] * (s_b[s2] * bm * hs2 + s_b[s2] * u1 + bm * s_X1[s2] + t2)
                              + (bm * s_gmx[s2] + t3);
            Py[j * CP + s2] = Wt[j * CP + s2] * phi;   // w_sj Phi[j][s]
        }
    }
    __syncthreads();
    if (tid < C) {
        const int j = tid;
        float acc = 0.f;
        for (int s2 = j; s2 < C; ++s2) acc += Py[j * CP + s2];
        // the adjoint from later chunks: w_{C-1,j} (b_{j-1} eh + sum_{i<j} w_{j-1,i} w_i qe_i)
        float qe = 0.f;
        for (int i = 0; i < j; ++i) qe = fmaf(s_step[i], qe, s_w[i] * s_qe[i]);
        acc = fmaf(s_wend[j], fmaf(s_bm1[j], eh, qe), acc);
        dbeta[tok0 + j] = acc;
    }
}

}  // namespace gka
