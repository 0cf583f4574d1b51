// Chunk-wise GKA forward on CUDA cores: state scan, per-token norm, and the
// Chebyshev solve with readout.
//
// Method: "Gated KalmaNet" (arXiv 2511.21016), ai.info page, Key
// Contributions 3 and Methodology in Plain English: the sequence is cut into
// chunks of C tokens; only each chunk's start state (H_s, M_s) is carried
// across chunks, every token inside a chunk is handled in parallel from it.
// Within a chunk, with l_j = sum_{m<=j} log beta_m (positions 0..C-1):
//   b_j    = exp(l_j)             decay of the chunk-start state to token j
//   w_{ji} = exp(l_j - l_i)       decay of token i's write to token j (i <= j)
//   H_j    = b_j H_s + sum_{i<=j} w_{ji} k_i k_i^T
//   M_j    = b_j M_s + sum_{i<=j} w_{ji} v_i k_i^T
// so H_j x = b_j H_s x + sum_{i<=j} w_{ji} (k_i . x) k_i never needs H_j.
// With the write gate g_i (the paper's beta_t-augmented variant, ai.info page,
// Main Findings; `gate` nullable, NULL = 1) every w_{ji} above becomes
// w_{ji} g_i: the increments take g_i into the weight, the norm and the solve
// read sqrt(g_i) k_i and sqrt(g_i) v_i (the same products in exact arithmetic).
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace gka {

constexpr int kSimtThreads = 256;

// ---------------------------------------------------------------------------
// Step 1a: per-chunk increments dH_n = sum_i w_{C-1,i} k_i k_i^T,
// dM_n = sum_i w_{C-1,i} v_i k_i^T and the chunk decay b_{C-1}, written into
// state slot n+1 (the scan of step 1b turns them into chunk-start states).
// grid (N, B*H), block 256, dynamic smem 3*C*D floats.
// ---------------------------------------------------------------------------
template <typename Tin, int D>
__global__ void __launch_bounds__(kSimtThreads)
k_chunk_delta(const Tin *__restrict__ k, const Tin *__restrict__ v,
              const float *__restrict__ beta, const float *__restrict__ gate,
              float *__restrict__ states,
              float *__restrict__ decay, float *__restrict__ bound_inc, int T, int N, int C) {
    extern __shared__ __align__(16) float sm[];
    float *Ks = sm;            // [C][D] keys
    float *Kw = Ks + C * D;    // [C][D] w_i k_i
    float *Vw = Kw + C * D;    // [C][D] w_i v_i
    __shared__ double ell[256];
    __shared__ double wtot[kSimtThreads / 32];

    const int n = blockIdx.x, bh = blockIdx.y;
    const size_t tok0 = (size_t)bh * T + (size_t)n * C;
    chunk_log_prefix(beta + tok0, C, ell, wtot);
    const double lend = ell[C - 1];
    for (int e = threadIdx.x; e < C * D; e += kSimtThreads) {
        const int i = e / D;
        float w = decay_exp(lend - ell[i]);
        if (gate) w *= gate[tok0 + i];
        const float kv = load_f(k + tok0 * D + e);
        Ks[e] = kv;
        Kw[e] = w * kv;
        Vw[e] = w * load_f(v + tok0 * D + e);
    }
    if (threadIdx.x == 0) decay[(size_t)bh * N + n] = decay_exp(lend);
    __syncthreads();
    if (bound_inc) {
        // sum_i w_i ||k_i k_i^T||_F and sum_i w_i ||v_i k_i^T||_F: the increments of a
        // bound on ||H_s||_F and ||M_s||_F (triangle inequality) used to scale the
        // low-precision copies of the states
        __shared__ float bpart[2][kSimtThreads / 32];
        float bh2 = 0.f, bm2 = 0.f;
        const int t = threadIdx.x;
        if (t < C) {
            float kw = 0.f, kk = 0.f, vv = 0.f;
            for (int d0 = 0; d0 < D; ++d0) {
                const int d = (d0 + t) % D;
                kw = fmaf(Kw[t * D + d], Ks[t * D + d], kw);
                kk = fmaf(Ks[t * D + d], Ks[t * D + d], kk);
                vv = fmaf(Vw[t * D + d], Vw[t * D + d], vv);
            }
            bh2 = kw;
            bm2 = sqrtf(vv) * sqrtf(kk);
        }
        bh2 = warp_sum(bh2);
        bm2 = warp_sum(bm2);
        if ((t & 31) == 0) {
            bpart[0][t >> 5] = bh2;
            bpart[1][t >> 5] = bm2;
        }
        __syncthreads();
        if (t < 2) {
            float sum = 0.f;
            for (int w = 0; w < kSimtThreads / 32; ++w) sum += bpart[t][w];
            bound_inc[((size_t)bh * N + n) * 2 + t] = sum;
        }
    }

    constexpr int TS = D / 16;  // TS x TS outputs per thread, 16 x 16 threads
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float *out = states + ((size_t)bh * (N + 1) + n + 1) * 2 * D * D;
#pragma unroll 1
    for (int mat = 0; mat < 2; ++mat) {
        const float *Rw = mat == 0 ? Kw : Vw;
        float acc[TS][TS];
#pragma unroll
        for (int u = 0; u < TS; ++u)
#pragma unroll
            for (int w = 0; w < TS; ++w) acc[u][w] = 0.f;
        for (int i = 0; i < C; ++i) {
            float ra[TS], cb[TS];
#pragma unroll
            for (int u = 0; u < TS; ++u) {
                ra[u] = Rw[i * D + ty * TS + u];
                cb[u] = Ks[i * D + tx * TS + u];
            }
#pragma unroll
            for (int u = 0; u < TS; ++u)
#pragma unroll
                for (int w = 0; w < TS; ++w) acc[u][w] = fmaf(ra[u], cb[w], acc[u][w]);
        }
        float *o = out + (size_t)mat * D * D;
#pragma unroll
        for (int u = 0; u < TS; ++u)
#pragma unroll
            for (int w = 0; w < TS; ++w) o[(size_t)(ty * TS + u) * D + tx * TS + w] = acc[u][w];
    }
}

// ---------------------------------------------------------------------------
// Step 1b: the sequential part.  Per state element e (of [2, D, D]):
//   S_0 = 0,  S_{n+1} = b^{(n)} S_n + dS_n   (in place over slots 1..N)
// grid (ceil(2*D*D/1024), B*H), block 256, 4 elements per thread.  Optionally copies S_N out and
// writes an fp16 copy of every chunk-start state S_n, n < N, scaled by a power
// of two 2^e_n chosen from the running bound ||S_n||_F <= bound_n (the
// tensor-core operands; e_n goes to state_exp[bh][n][H or M]).  Without
// write_fp32 the fp32 slots keep the increments and only S_N is written out.
// ---------------------------------------------------------------------------
// Exponent e such that |value| <= bound implies |value * 2^e| <= 2^14.
__device__ __forceinline__ int lp_exponent(float bound) {
    if (!(bound > 0.f)) return 0;
    const int e = 14 - (ilogbf(bound) + 1);
    return e < -120 ? -120 : (e > 120 ? 120 : e);
}

constexpr int kScanTile = 256;   // chunks whose scales are prepared per pass
constexpr int kScanVec = 4;      // state elements per thread (one 16-byte load)

__global__ void __launch_bounds__(256)
k_state_scan(float *__restrict__ states, const float *__restrict__ decay,
             float *__restrict__ final_state, __half *__restrict__ states_lp,
             const float *__restrict__ bound_inc, int *__restrict__ state_exp, int N, int DD2,
             bool write_fp32) {
    __shared__ float s_dec[kScanTile], s_scale[2][kScanTile], s_binc[2][kScanTile];
    __shared__ float s_bound[2];
    const int bh = blockIdx.y;
    const int e = (blockIdx.x * blockDim.x + threadIdx.x) * kScanVec;   // first of 4 elements
    const bool active = e < DD2;
    float *base = states + (size_t)bh * (N + 1) * DD2 + e;
    __half *lbase = states_lp ? states_lp + (size_t)bh * N * DD2 + e : nullptr;
    const int mat = e < DD2 / 2 ? 0 : 1;          // H or M elements (DD2/2 is a multiple of 4)
    const float *dec = decay + (size_t)bh * N;
    if (threadIdx.x < 2) s_bound[threadIdx.x] = 0.f;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    if (active) *reinterpret_cast<float4 *>(base) = s;
    for (int n0 = 0; n0 < N; n0 += kScanTile) {
        const int nt = min(kScanTile, N - n0);
        __syncthreads();
        for (int i = threadIdx.x; i < nt; i += blockDim.x) s_dec[i] = dec[n0 + i];
        if (lbase)
            for (int i = threadIdx.x; i < 2 * nt; i += blockDim.x)
                s_binc[i & 1][i >> 1] = bound_inc[((size_t)bh * N + n0) * 2 + i];
        __syncthreads();
        if (lbase && threadIdx.x < 2) {
            // power-of-two scales of the chunk-start states from the running bound
            // ||S_n||_F <= bound_n (one thread per matrix; same for every block of bh)
            const int m = threadIdx.x;
            float bound = s_bound[m];
            for (int i = 0; i < nt; ++i) {
                const int ex = lp_exponent(bound);
                s_scale[m][i] = ldexpf(1.f, ex);
                if (blockIdx.x == 0) state_exp[((size_t)bh * N + n0 + i) * 2 + m] = ex;
                bound = fmaf(s_dec[i], bound, s_binc[m][i]);
            }
            s_bound[m] = bound;
        }
        __syncthreads();
        if (!active) continue;
        auto step = [&](int i, float4 dl) {
            const int n = n0 + i;
            if (lbase) {
                const float sc = s_scale[mat][i];
                const __half2 h01 = __floats2half2_rn(s.x * sc, s.y * sc);
                const __half2 h23 = __floats2half2_rn(s.z * sc, s.w * sc);
                uint2 pk;
                pk.x = *reinterpret_cast<const uint32_t *>(&h01);
                pk.y = *reinterpret_cast<const uint32_t *>(&h23);
                *reinterpret_cast<uint2 *>(lbase + (size_t)n * DD2) = pk;
            }
            const float b = s_dec[i];
            s.x = fmaf(b, s.x, dl.x);
            s.y = fmaf(b, s.y, dl.y);
            s.z = fmaf(b, s.z, dl.z);
            s.w = fmaf(b, s.w, dl.w);
            if (write_fp32) *reinterpret_cast<float4 *>(base + (size_t)(n + 1) * DD2) = s;
        };
        int i = 0;
        for (; i + 8 <= nt; i += 8) {   // loads of a batch issued before its dependent stores
            float4 dl[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                dl[u] = __ldcs(reinterpret_cast<const float4 *>(base + (size_t)(n0 + i + u + 1) * DD2));
#pragma unroll
            for (int u = 0; u < 8; ++u) step(i + u, dl[u]);
        }
        for (; i < nt; ++i)
            step(i, __ldcs(reinterpret_cast<const float4 *>(base + (size_t)(n0 + i + 1) * DD2)));
    }
    if (active && final_state) *reinterpret_cast<float4 *>(final_state + (size_t)bh * DD2 + e) = s;
}

// ---------------------------------------------------------------------------
// Step 2: per-token ||H_j||_F from the chunk-start state and the key Gram
// matrix (ai.info page, Methodology: closed-form chunk-wise expression):
//   ||H_j||^2 = b_j^2 ||H_s||^2 + 2 b_j X_j + R_j,
//   X_j = sum_{i<=j} w_{ji} k_i^T H_s k_i,
//   R_j = sum_{i,l<=j} w_{ji} w_{jl} (k_i.k_l)^2, evaluated with the exact
//         identity R_j = beta_j^2 R_{j-1} + 2 sum_{i<j} w_{ji} (k_i.k_j)^2 + |k_j|^4
//         (the first sum splits off the terms with i = j or l = j).
// grid (N, B*H), block 256, dynamic smem (D*D + C*(D+1)) floats.
// ---------------------------------------------------------------------------
template <typename Tin, int D>
__global__ void __launch_bounds__(kSimtThreads)
k_chunk_norm(const Tin *__restrict__ k, const float *__restrict__ beta,
             const float *__restrict__ gate, const float *__restrict__ states, float *__restrict__ norms, int T, int N,
             int C) {
    extern __shared__ __align__(16) float sm[];
    float *Hs = sm;                 // [D][D]
    float *Ks = Hs + D * D;         // [C][D+1]
    constexpr int KP = D + 1;
    __shared__ double ell[256];
    __shared__ float bj[256], betaj[256], ui[256], Xj[256], Ej[256], Gjj[256];
    __shared__ double wtot[kSimtThreads / 32];
    __shared__ float upart[256][D / 32 > 0 ? D / 32 : 1];
    __shared__ float hs2_part[kSimtThreads / 32];

    const int n = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const size_t tok0 = (size_t)bh * T + (size_t)n * C;
    chunk_log_prefix(beta + tok0, C, ell, wtot);
    const float *Hg = states + ((size_t)bh * (N + 1) + n) * 2 * D * D;
    float ss = 0.f;
    for (int e = tid; e < D * D; e += kSimtThreads) {
        const float h = Hg[e];
        Hs[e] = h;
        ss = fmaf(h, h, ss);
    }
    for (int e = tid; e < C * D; e += kSimtThreads) {
        float kv = load_f(k + tok0 * D + e);
        if (gate) kv *= sqrtf(gate[tok0 + e / D]);
        Ks[(e / D) * KP + e % D] = kv;
    }
    for (int j = tid; j < C; j += kSimtThreads) {
        bj[j] = decay_exp(ell[j]);
        betaj[j] = decay_exp(j == 0 ? ell[0] : ell[j] - ell[j - 1]);
    }
    ss = warp_sum(ss);
    if (lane == 0) hs2_part[warp] = ss;
    __syncthreads();
    float hs2 = 0.f;
    for (int w = 0; w < kSimtThreads / 32; ++w) hs2 += hs2_part[w];

    // u_i = k_i^T H_s k_i: thread (column b, group g) forms y_ib = sum_a k_ia H_ab
    constexpr int NG = kSimtThreads / D;
    const int b = tid % D, g = tid / D;
    for (int i0 = g * 4; i0 < C; i0 += NG * 4) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        const int ni = min(4, C - i0);
        for (int a = 0; a < D; ++a) {
            const float h = Hs[a * D + b];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (u < ni) acc[u] = fmaf(Ks[(i0 + u) * KP + a], h, acc[u]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            float p = (u < ni) ? acc[u] * Ks[(i0 + u) * KP + b] : 0.f;
            p = warp_sum(p);
            if (lane == 0 && u < ni) upart[i0 + u][b / 32] = p;
        }
    }
    __syncthreads();
    for (int i = tid; i < C; i += kSimtThreads) {
        float s = 0.f;
        for (int w = 0; w < D / 32; ++w) s += upart[i][w];
        ui[i] = s;
    }
    __syncthreads();

    // per token j (one warp each): X_j, E_j = sum_{i<j} w_{ji} G_ij^2, G_jj
    for (int j = warp; j < C; j += kSimtThreads / 32) {
        float xs = 0.f, es = 0.f;
        for (int i = lane; i <= j; i += 32) {
            float dot = 0.f;
            for (int d = 0; d < D; ++d) dot = fmaf(Ks[i * KP + d], Ks[j * KP + d], dot);
            const float w = decay_exp(ell[j] - ell[i]);
            xs = fmaf(w, ui[i], xs);
            if (i < j) es = fmaf(w * dot, dot, es);
        }
        float gjj = 0.f;
        for (int d = lane; d < D; d += 32) gjj = fmaf(Ks[j * KP + d], Ks[j * KP + d], gjj);
        xs = warp_sum(xs);
        es = warp_sum(es);
        gjj = warp_sum(gjj);
        if (lane == 0) {
            Xj[j] = xs;
            Ej[j] = es;
            Gjj[j] = gjj;
        }
    }
    __syncthreads();
    if (tid == 0) {
        float R = 0.f;
        for (int j = 0; j < C; ++j) {
            R = betaj[j] * betaj[j] * R + 2.f * Ej[j] + Gjj[j] * Gjj[j];
            const float n2 = bj[j] * bj[j] * hs2 + 2.f * bj[j] * Xj[j] + R;
            norms[tok0 + j] = sqrtf(fmaxf(n2, 0.f));
        }
    }
}

// ---------------------------------------------------------------------------
// Steps 3 + 4: r-step Chebyshev solve of (H_j + lambda_j I) x = q_j for TG
// tokens of one chunk, then o_j = b_j M_s x_j + sum_{i<=j} w_{ji} (k_i.x_j) v_i.
// With x_out (nullable, fp32 [B*H*T, D]) the kernel writes the iterates x_j there
// instead and skips the readout (the backward pass recomputes them this way).
// Chebyshev (ai.info, Key Contributions 2; pith.science appendix, Lemma 3):
//   x_1 = q/d,  x_{i+1} = x_{i-1} + omega_i ((q - A x_i)/d + x_i - x_{i-1}),
//   A = H_j + lambda_j I,  d = (1+2a) n_j / 2,  lambda_j = a n_j.
// grid (C/TG, N, B*H), block 256.
// ---------------------------------------------------------------------------
constexpr int kSolveTG = 16;

// Dot product of two 16-byte aligned rows of D floats in shared memory, 4 at a time.
template <int D>
__device__ __forceinline__ float dot4(const float *a, const float *b) {
    float s0 = 0.f, s1 = 0.f;
#pragma unroll 8
    for (int d = 0; d < D; d += 8) {
        const float4 a0 = *reinterpret_cast<const float4 *>(a + d);
        const float4 b0 = *reinterpret_cast<const float4 *>(b + d);
        const float4 a1 = *reinterpret_cast<const float4 *>(a + d + 4);
        const float4 b1 = *reinterpret_cast<const float4 *>(b + d + 4);
        s0 = fmaf(a0.x, b0.x, fmaf(a0.y, b0.y, fmaf(a0.z, b0.z, fmaf(a0.w, b0.w, s0))));
        s1 = fmaf(a1.x, b1.x, fmaf(a1.y, b1.y, fmaf(a1.z, b1.z, fmaf(a1.w, b1.w, s1))));
    }
    return s0 + s1;
}

template <int D>
struct SolveSmem {
    static constexpr int KP = D + 4;   // 16-byte aligned rows (float4 dots, conflict-free)
    static size_t bytes(int C) {
        return sizeof(float) * ((size_t)D * KP + (size_t)C * KP + 3 * kSolveTG * D +
                                2 * kSolveTG * C);
    }
};

template <typename Tin, int D>
__global__ void __launch_bounds__(kSimtThreads)
k_chunk_solve(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
              const float *__restrict__ beta, const float *__restrict__ gate,
              const float *__restrict__ states,
              const float *__restrict__ norms, Tin *__restrict__ o, float *__restrict__ x_out,
              int T, int N, int C, const ChebParams P) {
    constexpr int TG = kSolveTG;
    constexpr int KP = SolveSmem<D>::KP;
    constexpr int NJ = TG * D / kSimtThreads;   // tokens per thread in the D-parallel phase
    extern __shared__ __align__(16) float sm[];
    float *Ms = sm;                    // [D][KP]: H_s (symmetric), later M_s^T
    float *Ks = Ms + D * KP;           // [C][KP]: keys, later values
    float *Xc = Ks + C * KP;           // [TG][D] current iterate
    float *Xp = Xc + TG * D;           // [TG][D] previous iterate
    float *Qs = Xp + TG * D;           // [TG][D] q
    float *Ps = Qs + TG * D;           // [TG][C] w_{ji} (k_i . x_j)
    float *Ws = Ps + TG * C;           // [TG][C] w_{ji}, 0 for i > j
    __shared__ double ell[256], wtot[kSimtThreads / 32];
    __shared__ float s_b[TG], s_lam[TG], s_invd[TG];

    const int tid = threadIdx.x;
    const int j0 = blockIdx.x * TG, n = blockIdx.y, bh = blockIdx.z;
    const int jend = j0 + TG;          // keys 0..jend-1 are needed
    const size_t tok0 = (size_t)bh * T + (size_t)n * C;
    chunk_log_prefix(beta + tok0, C, ell, wtot);

    const float *Hg = states + ((size_t)bh * (N + 1) + n) * 2 * D * D;
    for (int e = tid; e < D * D; e += kSimtThreads) Ms[(e / D) * KP + e % D] = Hg[e];
    // keys (and at the readout values) of token i scaled by sqrt(g_i)
    auto load_rows = [&](const Tin *src) {
        for (int e = tid; e < jend * D; e += kSimtThreads) {
            float x = load_f(src + tok0 * D + e);
            if (gate) x *= sqrtf(gate[tok0 + e / D]);
            Ks[(e / D) * KP + e % D] = x;
        }
    };
    load_rows(k);
    for (int e = tid; e < TG * D; e += kSimtThreads) Qs[e] = load_f(q + (tok0 + j0) * D + e);
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
    for (int e = tid; e < TG * D; e += kSimtThreads) {
        Xc[e] = Qs[e] * s_invd[e / D];
        Xp[e] = 0.f;
    }
    __syncthreads();

    const int c = tid % D, jg = tid / D;   // column and token group of the D-parallel phase

    // P[jj][i] = w_{ji} (k_i . x_j), i < jend
    auto form_p = [&]() {
        for (int p = tid; p < TG * jend; p += kSimtThreads) {
            const int jj = p / jend, i = p % jend;
            Ps[jj * C + i] = Ws[jj * C + i] * dot4<D>(Ks + i * KP, Xc + jj * D);
        }
    };
    // acc[u] = b_j sum_d S[d][c] x_j[d] + sum_i P[j][i] R[i][c] for the thread's tokens
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
            const float y = fmaf(s_lam[jj], xc, acc[u]);
            xn[u] = fmaf(w, fmaf(Qs[jj * D + c] - y, s_invd[jj], xc - xp), xp);
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

    if (x_out) {
        for (int e = tid; e < TG * D; e += kSimtThreads) x_out[(tok0 + j0) * D + e] = Xc[e];
        return;
    }
    // readout: P with the keys, then swap in M_s^T and the values
    form_p();
    __syncthreads();
    const float *Mg = Hg + D * D;
    for (int e = tid; e < D * D; e += kSimtThreads) {
        const int row = e / D, col = e % D;   // M[row][col]; stored as Ms[col][row]
        Ms[col * KP + row] = Mg[e];
    }
    load_rows(v);
    __syncthreads();
    float acc[NJ];
    apply(acc);
#pragma unroll
    for (int u = 0; u < NJ; ++u) {
        const int jj = jg * NJ + u;
        store_f(o + (tok0 + j0 + jj) * D + c, s_invd[jj] > 0.f ? acc[u] : 0.f);
    }
}

}  // namespace gka
