// Tensor-core gradients of the backward pass (bf16 inputs, D = 128, chunks of 32
// tokens): the work of k_bwd_grads (backward_simt.cuh) with its two dense parts on
// tcgen05.
//
// Method: "Gated KalmaNet" (arXiv 2511.21016), ai.info page, Key Contributions 3 and
// Main Findings (the full intra-chunk interaction of the backward); pith.science
// appendix, Eq. 50 (the key gradient with its ||H_t||_F term).  Per chunk, with the
// row products R1..R4 and the per-token and per-chunk scalars of k_bwd_rows_tc:
//   dot matrices   KX[l][s] = k_l . x_s,  KY = k_l . y_s,  GK = k_l . k_s,  VG = v_l . g_s;
//   coefficients   Py = -W o KX,  Px = W o (VG - KY),  Pg = W o KX,
//                  Pk[l][s] = -2 R_m W[l][m] W[s][m] w_s GK[l][s]  (m = max(l, s)),
//                  W[l][s] = w_sl for s >= l (0 otherwise);
//   row outputs    A0[l] = sum_s Py[l][s] y_s + Px[l][s] x_s + Pk[l][s] k_s,
//                  B0[l] = sum_s Pg[l][s] g_s;
//   gradients      dk_l = w_l (A0 - 2 f_l R1 + wend_l (R2 + R3)),  dv_l = w_l (B0 + wend_l R4),
//                  dw_l = (k_l . A + v_l . B) / 2,  and dbeta by the prefix recurrences of
//                  k_bwd_grads over the dot matrices.
// The five row tiles (x, y, k, g, v) are fp16 with one power-of-two scale per row (its
// largest entry in [1/2, 1)), in one 160-row region [X; Y; K; G; V] (two 64-column halves):
//   - the dot matrices are one 128 x 128 x 128 MMA, A = rows [K; G; V; -] (K-major),
//     B = rows [X; Y; K; G]; the lanes of K and V hold the four matrices;
//   - the row outputs are M = 128 (column c), N = 32 (token l), K = 32 (token s) MMAs
//     with the same row tiles read MN-major and the coefficient tiles (fp16, K-major,
//     the row scales folded in) as B; A0's three products share one power-of-two scale.
// Warps 1 and 3 form dbeta (its prefix sums over the chunk as 32 x 32 matrix products)
// while the other warps form the coefficient tiles; thread 0 issues every MMA.
// grid (N, B*H), block 256.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "backward_simt.cuh"
#include "common.cuh"
#include "ptx.cuh"
#include "solve_tc.cuh"
#include "state_tc.cuh"
#include "tcgen05.cuh"

namespace gka {

struct BwdGradTcSmem {
    static constexpr uint32_t HALF = 20480;                 // one 64-column half: 160 rows
    static constexpr uint32_t RGN = 0;                      // [2][160][64] fp16 rows X Y K G V
    static constexpr uint32_t PT = RGN + 2 * HALF;          // 4 x [32][64] fp16: Py Px Pk Pg
    static constexpr uint32_t MAT = PT + 4 * 4096;          // 6 x float[32][33]: KX KY VG GK Q W
    static constexpr uint32_t SIG = MAT + 6 * 32 * 33 * 4;  // float[5][32] inverse row scales x y k g v
    static constexpr uint32_t SCAL = SIG + 5 * 128;         // float[13][32] per-token scalars
    static constexpr uint32_t RED = SCAL + 13 * 128;        // float[32][4] token sums
    static constexpr uint32_t MRED = RED + 512;             // float[8][2] maxima, 2 scales
    static constexpr uint32_t BARS = MRED + 80;             // 3 mbarriers: dots, rows, drain
    static constexpr uint32_t TBASE = BARS + 24;
    static constexpr uint32_t END = TBASE + 16;
    static constexpr size_t bytes = END + 1024;             // + alignment slack
};

__global__ void __launch_bounds__(kSimtThreads, 2)
k_bwd_grads_tc(const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v,
               const float *__restrict__ beta, const float *__restrict__ gate,
               const __nv_bfloat16 *__restrict__ dout, const float *__restrict__ xs,
               const float *__restrict__ ys, const float *__restrict__ cvec,
               const float *__restrict__ R, const float *__restrict__ tokq,
               const float *__restrict__ chq, __nv_bfloat16 *__restrict__ dk,
               __nv_bfloat16 *__restrict__ dv, float *__restrict__ dbeta,
               float *__restrict__ dgate, int T, int N, int *__restrict__ timeout_flag) {
    using L = BwdGradTcSmem;
    constexpr int D = 128, C = kBrC, CP = C + 1;
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = smem_align1024(smraw);
    const uint32_t sb = smem_u32(sm);
    float *KX = reinterpret_cast<float *>(sm + L::MAT), *KY = KX + C * CP, *VG = KY + C * CP,
          *GK = VG + C * CP, *Qm = GK + C * CP, *Wt = Qm + C * CP;
    float *isig = reinterpret_cast<float *>(sm + L::SIG);   // 1 / row scale: x y k g v
    float *sc = reinterpret_cast<float *>(sm + L::SCAL);
    float *s_b = sc, *s_step = sc + 32, *s_wend = sc + 64, *s_w = sc + 96, *s_c = sc + 128,
          *s_uk = sc + 160, *s_yhx = sc + 192, *s_gmx = sc + 224, *s_qe = sc + 256,
          *s_bm1 = sc + 288, *s_f = sc + 320, *s_R = sc + 352, *s_X1 = sc + 384;
    float *red = reinterpret_cast<float *>(sm + L::RED);
    float *mred = reinterpret_cast<float *>(sm + L::MRED);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BARS);
    uint32_t *tbase = reinterpret_cast<uint32_t *>(sm + L::TBASE);
    __shared__ double ell[C], wtot[kSimtThreads / 32];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = blockIdx.x, bh = blockIdx.y;
    const size_t tok0 = (size_t)bh * T + (size_t)n * C;
    const size_t plane = (size_t)gridDim.y * T, RD = plane * D;

    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    if (tid == 32) {
        // the row products, read in the epilogue
        for (int p = 0; p < 4; ++p) bulk_prefetch_l2(R + p * RD + tok0 * D, C * D * 4);
    }
    if (warp == 0) {
        tc::tmem_alloc(tbase, 256);
        tc::tmem_relinquish();
    }
    // per-token scalars (threads tid < 32) and the chunk's two scalars, loaded first so that
    // their latency runs under the row loads and the log prefix
    float p_beta = 1.f, p_w = 1.f, p_c = 0.f, p_tq[4] = {0.f, 0.f, 0.f, 0.f};
    if (tid < C) {
        const size_t tt = tok0 + tid;
        p_beta = beta[tt];
        p_w = gate ? gate[tt] : 1.f;
        p_c = cvec[tt];
        p_tq[0] = tokq[tt];
        p_tq[1] = tokq[plane + tt];
        p_tq[2] = tokq[2 * plane + tt];
        p_tq[3] = tokq[3 * plane + tt] + tokq[4 * plane + tt];   // qe: the H and M parts
    }
    const float hs2 = chq[((size_t)bh * N + n) * 2], eh = chq[((size_t)bh * N + n) * 2 + 1];
    // this thread's items: token t = tid / 16 + 16 r, columns 8j .. 8j + 7
    const int j = tid & 15;
    uint4 ku[2], vu[2], gu[2];
    float4 xa[2], xb[2], ya[2], yb[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const size_t g = (tok0 + (tid >> 4) + 16 * r) * D + 8 * j;
        ku[r] = *reinterpret_cast<const uint4 *>(k + g);
        vu[r] = *reinterpret_cast<const uint4 *>(v + g);
        gu[r] = *reinterpret_cast<const uint4 *>(dout + g);
        xa[r] = *reinterpret_cast<const float4 *>(xs + g);
        xb[r] = *reinterpret_cast<const float4 *>(xs + g + 4);
        ya[r] = *reinterpret_cast<const float4 *>(ys + g);
        yb[r] = *reinterpret_cast<const float4 *>(ys + g + 4);
    }
    // the log prefix reads beta from shared memory (thread t wrote entry t itself)
    if (tid < C) s_b[tid] = p_beta;
    chunk_log_prefix_f32log(s_b, C, ell, wtot);
    if (tid < C) {
        const ChunkDecays dc = chunk_decays(ell, C, tid);
        s_b[tid] = dc.b;
        s_step[tid] = dc.step;
        s_wend[tid] = dc.wend;
        s_w[tid] = p_w;
        s_c[tid] = p_c;
        s_uk[tid] = p_tq[0];
        s_yhx[tid] = p_tq[1];
        s_gmx[tid] = p_tq[2];
        s_qe[tid] = p_tq[3];
        s_bm1[tid] = tid == 0 ? 1.f : decay_exp(ell[tid - 1]);
    }
    // W[l][s] = w_sl for s >= l, else 0
    for (int e = tid; e < C * C; e += kSimtThreads) {
        const int l = e >> 5, s2 = e & 31;
        Wt[l * CP + s2] = s2 >= l ? decay_exp(ell[s2] - ell[l]) : 0.f;
    }
    // the row tiles, one power-of-two scale per row (16 threads share a row)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int t = (tid >> 4) + 16 * r;
        auto put = [&](int tensor, const float *x8) {
            float mx = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(x8[e]));
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float s = inv_pow2_above(mx);
            if (j == 0) isig[tensor * 32 + t] = 1.f / s;   // a power of two: exact
            const uint32_t row = (uint32_t)(tensor * 32 + t);
            st_shared_v4(sb + L::RGN + (uint32_t)(j >> 3) * L::HALF + row * 128u +
                             (((uint32_t)j ^ row) & 7u) * 16u,
                         pack_f16(x8[0] * s, x8[1] * s), pack_f16(x8[2] * s, x8[3] * s),
                         pack_f16(x8[4] * s, x8[5] * s), pack_f16(x8[6] * s, x8[7] * s));
        };
        float x8[8];
        auto from_bf16 = [&](const uint4 &u) {
            const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                x8[2 * q] = bf16_lo(w4[q]);
                x8[2 * q + 1] = bf16_hi(w4[q]);
            }
        };
        x8[0] = xa[r].x; x8[1] = xa[r].y; x8[2] = xa[r].z; x8[3] = xa[r].w;
        x8[4] = xb[r].x; x8[5] = xb[r].y; x8[6] = xb[r].z; x8[7] = xb[r].w;
        put(0, x8);
        x8[0] = ya[r].x; x8[1] = ya[r].y; x8[2] = ya[r].z; x8[3] = ya[r].w;
        x8[4] = yb[r].x; x8[5] = yb[r].y; x8[6] = yb[r].z; x8[7] = yb[r].w;
        put(1, x8);
        from_bf16(ku[r]);
        put(2, x8);
        from_bf16(gu[r]);
        put(3, x8);
        from_bf16(vu[r]);
        put(4, x8);
    }
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tbase;
    // K-major rows from `row0` of the region (K = d in the two halves)
    auto kdesc = [&](int row0, int kk) {
        return tc::sdesc(sb + L::RGN + (uint32_t)row0 * 128u + (kk >> 2) * L::HALF + (kk & 3) * 32,
                         16, 1024);
    };
    if (tid == 0) {
        // dots: A = rows 64..191 (K, G, V; rows past V only reach lanes 96..127, unused),
        // B = rows 0..127 (X, Y, K, G)
        constexpr uint32_t ID = tc::idesc_f16(128, 128, false, false);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) tc::mma_f16(tmem, kdesc(64, kk), kdesc(0, kk), ID, kk > 0);
        tc::commit(&bars[0]);
    }
    if (tid == 32) {
        // f_l = sum_{s>=l} w_sl c_s b_s, R_m = sum_{s>=m} c_s w_sm^2 (suffix recurrences),
        // X1_s = sum_{l<=s} w_sl w_l uk_l
        float f = 0.f, Rm = 0.f;
        for (int l = C - 1; l >= 0; --l) {
            const float nxt = l + 1 < C ? s_step[l + 1] : 0.f;
            f = fmaf(nxt, f, s_c[l] * s_b[l]);
            Rm = fmaf(nxt * nxt, Rm, s_c[l]);
            s_f[l] = f;
            s_R[l] = Rm;
        }
        float x1 = 0.f;
        for (int s2 = 0; s2 < C; ++s2) {
            x1 = fmaf(s2 == 0 ? 0.f : s_step[s2], x1, s_w[s2] * s_uk[s2]);
            s_X1[s2] = x1;
        }
    }
    bool ok = mbar_wait_bounded(&bars[0], 0, kTcWaitProbes);
    tc::fence_after_sync();
    if (warp == 0 || warp == 4 || warp == 2) {
        // lane l of K (lanes 0..31) or V (lanes 64..95): its row of the dot matrices
        const int l = lane;
        const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        float d32[32];
        auto row = [&](int col0, float *dst, const float *isig_b, float ia) {
            tc::tmem_ld16(tl + col0, d32);
            tc::tmem_ld16(tl + col0 + 16, d32 + 16);
            tc::tmem_wait_ld();
#pragma unroll
            for (int s2 = 0; s2 < 32; ++s2) dst[l * CP + s2] = d32[s2] * ia * isig_b[s2];
        };
        if (warp == 0) {
            row(0, KX, isig, isig[64 + l]);
            row(32, KY, isig + 32, isig[64 + l]);
        } else if (warp == 4) {
            row(64, GK, isig + 64, isig[64 + l]);
        } else {
            row(96, VG, isig + 96, isig[128 + l]);
        }
    }
    tc::fence_before_sync();
    ok = __syncthreads_and(ok);
    if (warp == 1 || warp == 3) {
        // dbeta_j = sum_{s>=j} w_sj Phi[j][s] + (adjoint from later chunks), with
        //   Phi[j][s] = -y_s^T H_{j-1} x_s - c_s <H_s, H_{j-1}> + g_s^T M_{j-1} x_s
        // (H_s the state at token s, H_{j-1} the one before token j, H_{-1} = H_start),
        // through the prefix sums over i < j of its terms, as matrix products over the
        // chunk (warps 1 and 3, thread dt: rows 8r + dt / 8, columns 8q + dt % 8):
        //   Q  = (w o GK^2 o w)^T W,         Q[i][s] = sum_{l<=s} w_sl w_l w_i (k_l . k_i)^2,
        //   T1 = L (w o KY o KX),  T2 = L Q,  T3 = L (w o VG o KX),  L[j][i] = w_{j-1,i} (i < j),
        //   u1 = L (w o uk),  qe = L (w o qe),
        //   Phi[j][s] = -(b_{j-1} yhx_s + T1) - c_s (b_s b_{j-1} hs2 + b_s u1_j + b_{j-1} X1_s + T2)
        //               + (b_{j-1} gmx_s + T3)
        const int dt = (warp == 1 ? 0 : 32) + lane, r0 = dt >> 3, q0 = dt & 7;
        {
            float acc[4][4];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[r][q] = 0.f;
#pragma unroll 4
            for (int l = 0; l < C; ++l) {
                const float wl = s_w[l];
                float g2[4], wt[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const float g = GK[l * CP + r0 + 8 * r];
                    g2[r] = wl * g * g;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) wt[q] = Wt[l * CP + q0 + 8 * q];
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[r][q] = fmaf(g2[r], wt[q], acc[r][q]);
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int i = r0 + 8 * r;
#pragma unroll
                for (int q = 0; q < 4; ++q) Qm[i * CP + q0 + 8 * q] = s_w[i] * acc[r][q];
            }
        }
        named_barrier_sync(3, 64);
        {
            float t1[4][4], t2[4][4], t3[4][4], u1[4], qe[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                u1[r] = qe[r] = 0.f;
#pragma unroll
                for (int q = 0; q < 4; ++q) t1[r][q] = t2[r][q] = t3[r][q] = 0.f;
            }
#pragma unroll 2
            for (int i = 0; i < C; ++i) {
                const float wi = s_w[i];
                float lm[4], a1[4], a3[4], qm[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int j = r0 + 8 * r;
                    lm[r] = j >= 1 ? Wt[i * CP + j - 1] : 0.f;   // 0 unless i <= j - 1
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int s2 = q0 + 8 * q;
                    const float kx = KX[i * CP + s2];
                    a1[q] = wi * KY[i * CP + s2] * kx;
                    a3[q] = wi * VG[i * CP + s2] * kx;
                    qm[q] = Qm[i * CP + s2];
                }
                const float wuk = wi * s_uk[i], wqe = wi * s_qe[i];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    u1[r] = fmaf(lm[r], wuk, u1[r]);
                    qe[r] = fmaf(lm[r], wqe, qe[r]);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        t1[r][q] = fmaf(lm[r], a1[q], t1[r][q]);
                        t2[r][q] = fmaf(lm[r], qm[q], t2[r][q]);
                        t3[r][q] = fmaf(lm[r], a3[q], t3[r][q]);
                    }
                }
            }
            // w_sj Phi[j][s] over this thread's columns, summed along the row, then over
            // the 8 threads of the row (consecutive lanes)
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int j = r0 + 8 * r;
                const float bm = s_bm1[j];
                float rs = 0.f;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int s2 = q0 + 8 * q;
                    const float phi = -(bm * s_yhx[s2] + t1[r][q])
                                      - s_c[s2] * (s_b[s2] * bm * hs2 + s_b[s2] * u1[r] +
                                                   bm * s_X1[s2] + t2[r][q])
                                      + (bm * s_gmx[s2] + t3[r][q]);
                    rs += Wt[j * CP + s2] * phi;   // 0 for s < j
                }
                rs += __shfl_xor_sync(0xffffffffu, rs, 1);
                rs += __shfl_xor_sync(0xffffffffu, rs, 2);
                rs += __shfl_xor_sync(0xffffffffu, rs, 4);
                // the adjoint from later chunks: w_{C-1,j} (b_{j-1} eh + sum_{i<j} w_{j-1,i} w_i qe_i)
                if (q0 == 0 && ok) dbeta[tok0 + j] = fmaf(s_wend[j], fmaf(bm, eh, qe[r]), rs);
            }
        }
    } else {
        // warps 0, 2, 4..7: the coefficient tiles, two adjacent s per item, with the row
        // scales of the A operand folded in (B[l][s] = P[l][s] pi / sigma_s)
        constexpr int NT = kSimtThreads - 64;
        const int me = warp == 0 ? lane : (warp == 2 ? 32 + lane : tid - 64);
        auto coef = [&](int l, int s2, float *p4) {
            const float w = Wt[l * CP + s2];
            const float kx = KX[l * CP + s2];
            p4[0] = -w * kx * isig[32 + s2];                             // Py / sigma_y
            p4[1] = w * (VG[l * CP + s2] - KY[l * CP + s2]) * isig[s2];  // Px / sigma_x
            const int m = l > s2 ? l : s2;
            p4[2] = -2.f * s_R[m] * Wt[l * CP + m] * Wt[s2 * CP + m] * s_w[s2] * GK[l * CP + s2] *
                    isig[64 + s2];                                       // Pk / sigma_k
            p4[3] = w * kx * isig[96 + s2];                              // Pg / sigma_g
        };
        float ma = 0.f, mg = 0.f;
        for (int e = me; e < C * C / 2; e += NT) {
            const int l = e >> 4, s2 = 2 * (e & 15);
            float p0[4], p1[4];
            coef(l, s2, p0);
            coef(l, s2 + 1, p1);
            ma = fmaxf(ma, fmaxf(fmaxf(fabsf(p0[0]), fabsf(p0[1])), fabsf(p0[2])));
            ma = fmaxf(ma, fmaxf(fmaxf(fabsf(p1[0]), fabsf(p1[1])), fabsf(p1[2])));
            mg = fmaxf(mg, fmaxf(fabsf(p0[3]), fabsf(p1[3])));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, o));
            mg = fmaxf(mg, __shfl_xor_sync(0xffffffffu, mg, o));
        }
        if (lane == 0) {
            mred[warp * 2] = ma;
            mred[warp * 2 + 1] = mg;
        }
        named_barrier_sync(1, NT);
        ma = mg = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            if (w == 1 || w == 3) continue;
            ma = fmaxf(ma, mred[w * 2]);
            mg = fmaxf(mg, mred[w * 2 + 1]);
        }
        const float pa = inv_pow2_above(ma), pg = inv_pow2_above(mg);
        for (int e = me; e < C * C / 2; e += NT) {
            const int l = e >> 4, s2 = 2 * (e & 15);
            float p0[4], p1[4];
            coef(l, s2, p0);
            coef(l, s2 + 1, p1);
            // K-major tile row l, columns s2, s2 + 1 (one 4-byte word)
            const uint32_t off = (uint32_t)l * 128u + ((((uint32_t)s2 >> 3) ^ (uint32_t)l) & 7u) * 16u +
                                 ((uint32_t)s2 & 7u) * 2u;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float f = q == 3 ? pg : pa;
                *reinterpret_cast<uint32_t *>(sm + L::PT + q * 4096 + off) = pack_f16(p0[q] * f, p1[q] * f);
            }
        }
        if (tid == 0) {
            mred[16] = pa;   // read after the next block barrier
            mred[17] = pg;
        }
        fence_proxy_async_smem();
        named_barrier_sync(1, NT);
        if (tid == 0) {
            // A0 = [Y; X; K]^T-rows times (Py, Px, Pk), B0 = G rows times Pg: A MN-major
            // (rows s of the region, the halves HALF apart), B K-major (32 of 64 columns)
            tc::fence_after_sync();
            constexpr uint32_t ID = tc::idesc_f16(128, C, true, false);
            auto adesc = [&](int row0, int kk) {
                return tc::sdesc(sb + L::RGN + (uint32_t)row0 * 128u + kk * 2048, L::HALF, 1024);
            };
            auto bdesc = [&](int q, int kk) { return tc::sdesc(sb + L::PT + q * 4096 + kk * 32, 16, 1024); };
            if (ok) {
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk) {
                    tc::mma_f16(tmem + 128, adesc(32, kk), bdesc(0, kk), ID, kk > 0);   // Py y
                    tc::mma_f16(tmem + 128, adesc(0, kk), bdesc(1, kk), ID, true);      // Px x
                    tc::mma_f16(tmem + 128, adesc(64, kk), bdesc(2, kk), ID, true);     // Pk k
                    tc::mma_f16(tmem + 160, adesc(96, kk), bdesc(3, kk), ID, kk > 0);   // Pg g
                }
            }
            tc::commit(&bars[1]);
        }
    }
    ok = __syncthreads_and(ok);
    // epilogue: thread (column c = TMEM lane, tokens 16 wg .. 16 wg + 15); the row
    // products R1..R4 of 8 tokens at a time are loaded before they are used (the first 8
    // while the row outputs finish)
    const int quarter = warp & 3, wg = warp >> 2, c = quarter * 32 + lane;
    float rr[4][8];
    auto load_r = [&](int u0) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const size_t g = (tok0 + wg * 16 + u0 + u) * D + c;
#pragma unroll
            for (int p = 0; p < 4; ++p) rr[p][u] = R[p * RD + g];
        }
    };
    load_r(0);
    if (!mbar_wait_bounded(&bars[1], 0, kTcWaitProbes)) ok = false;
    tc::fence_after_sync();
    {
        const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(wg * 16);
        float a0[16], b0[16];
        tc::tmem_ld16(tl + 128, a0);
        tc::tmem_ld16(tl + 160, b0);
        tc::tmem_wait_ld();
        const float ua = 1.f / mred[16], ug = 1.f / mred[17];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            if (u == 8) load_r(8);
            const int l = wg * 16 + u;
            const size_t g = (tok0 + l) * D + c;
            const int ur = u & 7;
            float a = fmaf(-2.f * s_f[l], rr[0][ur], a0[u] * ua);
            a = fmaf(s_wend[l], rr[1][ur] + rr[2][ur], a);
            const float bb = fmaf(s_wend[l], rr[3][ur], b0[u] * ug);
            if (ok) {
                dk[g] = __float2bfloat16_rn(s_w[l] * a);
                dv[g] = __float2bfloat16_rn(s_w[l] * bb);
            }
            // write-gate gradient: (k . A + v . B) / 2 over the row (k, v from their
            // row tiles, exact for bf16 inputs)
            auto at = [&](int row) {
                const int cc = c & 63;
                const uint8_t *p = sm + L::RGN + (c >> 6) * L::HALF + row * 128 +
                                   ((((cc >> 3) ^ row) & 7) << 4) + (cc & 7) * 2;
                return __half2float(*reinterpret_cast<const __half *>(p));
            };
            const float kc = at(64 + l) * isig[64 + l], vc = at(128 + l) * isig[128 + l];
            const float dgp = warp_sum(fmaf(kc, a, vc * bb));
            if (lane == 0) red[l * 4 + quarter] = dgp;
        }
    }
    ok = __syncthreads_and(ok);
    if (dgate && tid < C && ok)
        dgate[tok0 + tid] = 0.5f * (red[tid * 4] + red[tid * 4 + 1] + red[tid * 4 + 2] + red[tid * 4 + 3]);
    if (!ok && tid == 0) {
        atomicExch(timeout_flag, 1);
        tc::commit(&bars[2]);
        mbar_wait_bounded(&bars[2], 0, kTcWaitProbes);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 256);
    }
}

}  // namespace gka
