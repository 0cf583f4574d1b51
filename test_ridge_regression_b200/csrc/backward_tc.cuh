// Tensor-core row products of the backward pass (bf16 inputs, D = 128, chunks
// of 32 tokens): the work of k_bwd_rows (backward_simt.cuh) as fp16 MMAs, and the
// right-hand side of the adjoint solve.
//
// Per chunk, with its chunk-start states H_s, M_s (the recompute's state pass writes
// them as fp16 copies scaled by 2^e, which arrive here by TMA), its adjoint states
// E^H, E^M arriving from later chunks (fp16 copies scaled by 2^e from the adjoint pass,
// adjoint_tc.cuh, also by TMA) and its rows k_t, v_t, g_t, x_t:
//   R1 = H_s K^T,  Hx = H_s X^T,  Mg = M_s^T G^T,
//   R2 = (E^H + E^H^T) K^T,  R3 = E^M^T V^T,  R4 = E^M K^T
// as 128 x 32 tiles (row c = TMEM lane, column t = token), then
//   R1, R2, R3, R4 to global (rows [B*H*T][128]), and per token
//   uk = k . R1,  yhx = y . Hx,  gmx = x . Mg,  qe = k . R2 / 2 + v . R4,
//   and per chunk hs2 = ||H_s||_F^2 (from the fp16 copy) and eh = <E^H, H_s> +
//   <E^M, M_s> (the adjoint pass forms both terms from its fp32 adjoints).
// Every copy's largest entry lies below 2^14 (states) or 1 (adjoints); k, v, g tiles
// are converted in shared memory with one power-of-two scale each, x with one per
// token.  The accumulators are fp32.  Two CTAs serve a chunk, one per matrix (H: R1,
// Hx, R2; M: Mg, R3, R4), each with one matrix tile: the state copy, then the adjoint
// copy loaded into it once the first products have read the state.
#pragma once

#include <cuda_fp16.h>

#include "backward_simt.cuh"
#include "common.cuh"
#include "ptx.cuh"
#include "solve_tc.cuh"
#include "state_tc.cuh"
#include "tcgen05.cuh"

namespace gka {

constexpr int kBrC = 32;   // tokens per chunk of this kernel

// Element (row t, column c) of a [2][32][64] fp16 row tile (128B swizzle).
__device__ __forceinline__ float f16_tile_at(const uint8_t *tile, int t, int c) {
    const int cc = c & 63;
    const uint8_t *p = tile + (c >> 6) * (kBrC * 128) + t * 128 + ((((cc >> 3) ^ t) & 7) << 4) +
                       (cc & 7) * 2;
    return __half2float(*reinterpret_cast<const __half *>(p));
}

struct BwdRowsTcSmem {
    static constexpr uint32_t MA = 0;              // [2][128][64] fp16: H_s or M_s, then E^H or E^M
    static constexpr uint32_t RK = MA + 32768;     // [2][32][64] fp16 rows of k
    static constexpr uint32_t RV = RK + 8192;      // v (M role)
    static constexpr uint32_t RG = RV + 8192;      // g (M role)
    static constexpr uint32_t RX = RG + 8192;      // x (per-token scales)
    static constexpr uint32_t XS = RX + 8192;      // float[32] x scales
    static constexpr uint32_t RED = XS + 128;      // float[2][32][4] per-token partial sums
    static constexpr uint32_t MRED = RED + 1024;   // float[24] block reductions
    static constexpr uint32_t BARS = MRED + 96;    // 5 mbarriers: products A, B; matrix;
                                                   // adjoint; drain
    static constexpr uint32_t TBASE = BARS + 40;
    static constexpr uint32_t END = TBASE + 16;
    static constexpr size_t bytes = END + 1024;    // + alignment slack
};

// One 128 x 128 fp16 chunk-start state copy (the state pass's output, scaled by
// 2^e) from `map` (rows [B*H*N*2*128][128], boxes 64 x 64, 128B swizzle) into a
// [2 column halves][128 rows][64] swizzled tile: four TMA loads completing on bar.
__device__ __forceinline__ void load_state_tile(const CUtensorMap *map, int row0, uint8_t *tile,
                                                uint64_t *bar) {
    for (int h = 0; h < 2; ++h)
        for (int rb = 0; rb < 2; ++rb)
            tc::tma_load_2d(tile + h * 16384 + rb * 8192, map, h * 64, row0 + rb * 64, bar);
}

// Sum of squares of the fp16 values of a [2][128][64] tile (all 256 threads; this
// thread's row r = tid / 2, column half tid % 2; the swizzle does not matter to a sum).
__device__ __forceinline__ float tile_f16_sumsq(uint32_t tile) {
    const int tid = threadIdx.x, r = tid >> 1, h = tid & 1;
    float s2 = 0.f;
#pragma unroll
    for (int c8 = 0; c8 < 8; ++c8) {
        const uint4 o = ld_shared_u4(tile + (uint32_t)h * 16384u + (uint32_t)r * 128u + c8 * 16u);
        const uint32_t w4[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w4[i]));
            s2 = fmaf(f.x, f.x, fmaf(f.y, f.y, s2));
        }
    }
    return s2;
}

// grid (N, B*H, 2), block 256, three CTAs per SM.  T = N * 32.  blockIdx.z = 0 (H role):
// H_s, then E^H: R1, uk, yhx, R2, the H part of qe (tokq plane 3), hs2 and eh; 1 (M role):
// M_s, then E^M: gmx, R3, R4, the M part of qe (tokq plane 4).  H_s, M_s: the fp16
// chunk-start state copies of the recompute's state pass (state_map, exponents sexp
// [B*H][N][2]); E^H, E^M: the fp16 adjoint copies of the adjoint pass (adj_map over adj_lp,
// same layout, exponents aexp) and its inner products eh_part [B*H][N][2].
__global__ void __launch_bounds__(kSimtThreads, 3)
k_bwd_rows_tc(const __grid_constant__ CUtensorMap state_map, const int *__restrict__ sexp,
              const __grid_constant__ CUtensorMap adj_map, const __half *__restrict__ adj_lp,
              const int *__restrict__ aexp, const float *__restrict__ eh_part,
              const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v,
              const __nv_bfloat16 *__restrict__ dout, const float *__restrict__ xs,
              const float *__restrict__ ys, float *__restrict__ R, float *__restrict__ tokq,
              float *__restrict__ chq, int T, int N, int *__restrict__ timeout_flag) {
    using L = BwdRowsTcSmem;
    constexpr int D = 128, C = kBrC;
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = smem_align1024(smraw);
    const uint32_t sb = smem_u32(sm);
    float *xsc = reinterpret_cast<float *>(sm + L::XS);
    float *red = reinterpret_cast<float *>(sm + L::RED);    // [2][32 tokens][4 quarters]
    float *mred = reinterpret_cast<float *>(sm + L::MRED);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BARS);
    uint32_t *tbase = reinterpret_cast<uint32_t *>(sm + L::TBASE);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, wg = warp >> 2;
    const int c = quarter * 32 + lane;       // matrix row = TMEM lane of this thread
    const int n = blockIdx.x, bh = blockIdx.y, m = blockIdx.z;   // m = 0: H role, 1: M role
    const bool mrole = m == 1;
    const size_t tok0 = (size_t)bh * T + (size_t)n * C;
    const size_t plane = (size_t)gridDim.y * T, RD = plane * D;
    const size_t e2 = ((size_t)bh * N + n) * 2;               // (chunk, matrix 0) entry
    const int mrow = (int)((e2 + m) * D);                       // this role's matrix in the maps

    if (tid == 0) {
        for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        // this role's chunk-start state (fp16 copy), read while the rows convert
        mbar_arrive_expect_tx(&bars[2], 32768);
        load_state_tile(&state_map, mrow, sm + L::MA, &bars[2]);
    }
    if (tid == 32) {
        // read after the rows: this role's adjoint copy (and the fp32 y rows in the H role)
        bulk_prefetch_l2(adj_lp + (size_t)mrow * D, D * D * 2);
        if (!mrole) bulk_prefetch_l2(ys + tok0 * D, C * D * 4);
    }
    if (warp == 0) {
        tc::tmem_alloc(tbase, 128);
        tc::tmem_relinquish();
    }
    // rows, thread (token t = tid / 8, columns c0 .. c0 + 15): k (and in the M role v, g)
    // in bf16 with one power-of-two scale per tile (one block reduction), x with one per
    // token; every load issued before any is used
    const int t8 = tid >> 3, c0 = (tid & 7) * 16;
    const uint32_t rhalf = (uint32_t)(c0 >> 6) * (kBrC * 128u), rcc = (uint32_t)(c0 & 63);
    float sK, sV = 1.f, sG = 1.f;
    {
        const size_t g0 = (tok0 + t8) * D + c0;
        uint4 ur[3][2];
        float4 xr[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            ur[0][h] = *reinterpret_cast<const uint4 *>(k + g0 + 8 * h);
            if (mrole) {
                ur[1][h] = *reinterpret_cast<const uint4 *>(v + g0 + 8 * h);
                ur[2][h] = *reinterpret_cast<const uint4 *>(dout + g0 + 8 * h);
            } else {
                ur[1][h] = ur[2][h] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) xr[i] = *reinterpret_cast<const float4 *>(xs + g0 + 4 * i);
        // x: one scale per token (its 8 threads)
        {
            float xv[16];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                xv[4 * i] = xr[i].x; xv[4 * i + 1] = xr[i].y; xv[4 * i + 2] = xr[i].z; xv[4 * i + 3] = xr[i].w;
            }
            float mxx = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) mxx = fmaxf(mxx, fabsf(xv[i]));
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) mxx = fmaxf(mxx, __shfl_xor_sync(0xffffffffu, mxx, o));
            const float sx = inv_pow2_above(mxx);
            if ((tid & 7) == 0) xsc[t8] = sx;
#pragma unroll
            for (int i = 0; i < 16; ++i) xv[i] *= sx;
            st_row8(sb + L::RX + rhalf, (uint32_t)t8, rcc, xv);
            st_row8(sb + L::RX + rhalf, (uint32_t)t8, rcc + 8, xv + 8);
        }
        float mx[3] = {0.f, 0.f, 0.f};
#pragma unroll
        for (int q = 0; q < 3; ++q) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t w4[4] = {ur[q][h].x, ur[q][h].y, ur[q][h].z, ur[q][h].w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    mx[q] = fmaxf(mx[q], fmaxf(fabsf(bf16_lo(w4[i])), fabsf(bf16_hi(w4[i]))));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx[q] = fmaxf(mx[q], __shfl_xor_sync(0xffffffffu, mx[q], o));
        }
        if (lane == 0) {
            mred[warp] = mx[0];
            mred[8 + warp] = mx[1];
            mred[16 + warp] = mx[2];
        }
        __syncthreads();
        float m3[3] = {0.f, 0.f, 0.f};
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            m3[0] = fmaxf(m3[0], mred[w]);
            m3[1] = fmaxf(m3[1], mred[8 + w]);
            m3[2] = fmaxf(m3[2], mred[16 + w]);
        }
        sK = inv_pow2_above(m3[0]);
        if (mrole) {
            sV = inv_pow2_above(m3[1]);
            sG = inv_pow2_above(m3[2]);
        }
        const float scl[3] = {sK, sV, sG};
        const uint32_t tiles[3] = {sb + L::RK, sb + L::RV, sb + L::RG};
#pragma unroll
        for (int q = 0; q < 3; ++q) {
            if (q > 0 && !mrole) break;
            float f[16];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t w4[4] = {ur[q][h].x, ur[q][h].y, ur[q][h].z, ur[q][h].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    f[8 * h + 2 * i] = bf16_lo(w4[i]) * scl[q];
                    f[8 * h + 2 * i + 1] = bf16_hi(w4[i]) * scl[q];
                }
            }
            st_row8(tiles[q] + rhalf, (uint32_t)t8, rcc, f);
            st_row8(tiles[q] + rhalf, (uint32_t)t8, rcc + 8, f + 8);
        }
    }
    // the copy holds 2^e S (exponents in [-120, 120])
    const float sS = pow2f(sexp[e2 + m]);
    bool ok = mbar_wait_bounded(&bars[2], 0, kTcWaitProbes);
    float hs2 = mrole ? 0.f : tile_f16_sumsq(sb + L::MA) * (pow2f(-sexp[e2]) * pow2f(-sexp[e2]));
    fence_proxy_async_smem();
    tc::fence_before_sync();
    ok = __syncthreads_and(ok);
    tc::fence_after_sync();
    const uint32_t tmem = *tbase;
    constexpr uint32_t ID_K = tc::idesc_f16(128, C, false, false);   // A K-major
    constexpr uint32_t ID_T = tc::idesc_f16(128, C, true, false);    // A MN-major (transposed)
    auto adesc_k = [&](int kk) { return tc::sdesc(sb + L::MA + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024); };
    auto adesc_t = [&](int kk) { return tc::sdesc(sb + L::MA + kk * 2048, 16384, 1024); };
    auto bdesc = [&](uint32_t b, int kk) { return tc::sdesc(b + (kk >> 2) * (C * 128) + (kk & 3) * 32, 16, 1024); };
    if (tid == 0) {
        if (ok) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                if (!mrole) {
                    tc::mma_f16(tmem + 0, adesc_k(kk), bdesc(sb + L::RK, kk), ID_K, kk > 0);    // R1
                    tc::mma_f16(tmem + 32, adesc_k(kk), bdesc(sb + L::RX, kk), ID_K, kk > 0);   // Hx
                } else {
                    tc::mma_f16(tmem + 0, adesc_t(kk), bdesc(sb + L::RG, kk), ID_T, kk > 0);    // Mg
                }
            }
        }
        tc::commit(&bars[0]);
    }
    if (!mbar_wait_bounded(&bars[0], 0, kTcWaitProbes)) ok = false;
    tc::fence_after_sync();
    bool e_loaded = false;
    if (tid == 0 && ok) {
        // the products have read the state: this role's adjoint copy into the same tile,
        // landing while the first results leave
        mbar_arrive_expect_tx(&bars[3], 32768);
        load_state_tile(&adj_map, mrow, sm + L::MA, &bars[3]);
        e_loaded = true;
    }
    // per-token sums over the 128 rows of `np` partial vectors: red[j][t][quarter], then
    // tokq planes p0 (+ 1)
    auto token_sums = [&](const float *pa, const float *pb, int np, int p0) {
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const float a = warp_sum(pa[u]);
            const float b = np > 1 ? warp_sum(pb[u]) : 0.f;
            if (lane == 0) {
                const int e = (wg * 16 + u) * 4 + quarter;
                red[e] = a;
                if (np > 1) red[128 + e] = b;
            }
        }
        __syncthreads();
        if (tid < np * C && ok) {
            const int j = tid >> 5, tt = tid & 31;
            const float *r4 = red + j * 128 + tt * 4;
            tokq[(p0 + j) * plane + tok0 + tt] = r4[0] + r4[1] + r4[2] + r4[3];
        }
        __syncthreads();
    };
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(wg * 16);
    const float iK = 1.f / sK;
    auto k_at = [&](int tt) { return f16_tile_at(sm + L::RK, tt, c) * iK; };
    {
        float acc[16], p1[16], p2[16];
        if (!mrole) {
            // R1 = H_s k -> R plane 0, uk = k . R1;  yhx = y . (H_s x)
            tc::tmem_ld16(tl + 0, acc);
            tc::tmem_wait_ld();
            const float u1 = 1.f / (sS * sK);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int tt = wg * 16 + u;
                const float a1 = acc[u] * u1;
                if (ok) R[(tok0 + tt) * D + c] = a1;
                p1[u] = a1 * k_at(tt);
            }
            tc::tmem_ld16(tl + 32, acc);
            tc::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int tt = wg * 16 + u;
                p2[u] = acc[u] / (sS * xsc[tt]) * ys[(tok0 + tt) * D + c];
            }
            token_sums(p1, p2, 2, 0);
        } else {
            // gmx = x . (M_s^T g), x as the products saw it
            tc::tmem_ld16(tl + 0, acc);
            tc::tmem_wait_ld();
            const float u3 = 1.f / (sS * sG);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int tt = wg * 16 + u;
                p1[u] = acc[u] * u3 * (f16_tile_at(sm + L::RX, tt, c) / xsc[tt]);
            }
            token_sums(p1, p1, 1, 2);
        }
    }
    // phase B: the adjoint copy (2^e E) in the same tile
    const float sE = pow2f(aexp[e2 + m]);
    if (!mbar_wait_bounded(&bars[3], 0, kTcWaitProbes)) ok = false;
    tc::fence_before_sync();
    ok = __syncthreads_and(ok);
    tc::fence_after_sync();
    if (tid == 0) {
        if (ok) {
            if (!mrole) {
                // R2 = (E^H + E^H^T) k
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_f16(tmem + 64, adesc_k(kk), bdesc(sb + L::RK, kk), ID_K, kk > 0);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_f16(tmem + 64, adesc_t(kk), bdesc(sb + L::RK, kk), ID_T, true);
            } else {
                // R3 = E^M^T v, R4 = E^M k
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    tc::mma_f16(tmem + 32, adesc_t(kk), bdesc(sb + L::RV, kk), ID_T, kk > 0);
                    tc::mma_f16(tmem + 64, adesc_k(kk), bdesc(sb + L::RK, kk), ID_K, kk > 0);
                }
            }
        }
        tc::commit(&bars[1]);
    }
    if (!mbar_wait_bounded(&bars[1], 0, kTcWaitProbes)) ok = false;
    tc::fence_after_sync();
    {
        float acc[16], part[16];
        if (!mrole) {
            // R2 -> plane 1, qe's H part = k . R2 / 2 -> tokq plane 3
            tc::tmem_ld16(tl + 64, acc);
            tc::tmem_wait_ld();
            const float u2 = 1.f / (sE * sK);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int tt = wg * 16 + u;
                const float a2 = acc[u] * u2;
                if (ok) R[RD + (tok0 + tt) * D + c] = a2;
                part[u] = 0.5f * a2 * k_at(tt);
            }
            token_sums(part, part, 1, 3);
        } else {
            // R3 -> plane 2, R4 -> plane 3, qe's M part = v . R4 -> tokq plane 4
            const float iV = 1.f / sV;
            tc::tmem_ld16(tl + 32, acc);
            tc::tmem_wait_ld();
            const float u3 = 1.f / (sE * sV), u4 = 1.f / (sE * sK);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int tt = wg * 16 + u;
                if (ok) R[2 * RD + (tok0 + tt) * D + c] = acc[u] * u3;
            }
            tc::tmem_ld16(tl + 64, acc);
            tc::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int tt = wg * 16 + u;
                const float a4 = acc[u] * u4;
                if (ok) R[3 * RD + (tok0 + tt) * D + c] = a4;
                part[u] = a4 * (f16_tile_at(sm + L::RV, tt, c) * iV);
            }
            token_sums(part, part, 1, 4);
        }
    }
    if (!mrole) {
        // chunk scalars: hs2, and eh from the adjoint pass's two inner products
        hs2 = warp_sum(hs2);
        if (lane == 0) mred[warp] = hs2;
        __syncthreads();
        if (tid == 0 && ok) {
            float s2 = 0.f;
            for (int w = 0; w < 8; ++w) s2 += mred[w];
            chq[e2] = s2;
            chq[e2 + 1] = eh_part[e2] + eh_part[e2 + 1];
        }
    }
    if (!ok && tid == 0) {
        // a wait gave up: flag it, and let every MMA this CTA issued finish before TMEM
        // is released (a commit after them, waited for with a bound)
        atomicExch(timeout_flag, 1);
        tc::commit(&bars[4]);
        mbar_wait_bounded(&bars[4], 0, kTcWaitProbes);
        mbar_wait_bounded(&bars[2], 0, kTcWaitProbes);   // the state tile's loads
        if (e_loaded) mbar_wait_bounded(&bars[3], 0, kTcWaitProbes);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 128);
    }
}

}  // namespace gka

namespace gka {

// ---------------------------------------------------------------------------
// k_bwd_u_tc: the right-hand side of the adjoint solve for one 32-token chunk
// (bf16 inputs, D = 128; the tensor-core solve then solves for y on it):
//   u_t = M_t^T g_t = b_t M_s^T g_t + sum_{i<=t} w_ti k~_i (v~_i . g_t),
// k~ = sqrt(w) k, v~ = sqrt(w) v the written keys and values.  Three fp16 MMA groups
// (operands with power-of-two scales, fp32 accumulators), row c = TMEM lane:
//   Q = G V~^T           (A = the 128-row operand region [G; V~; K~; -], only its
//                         first 32 lanes are used; B = the V~ rows),
//   A1 = M_s^T G^T       (the state pass's fp16 copy of M_s, MN-major),
//   A2 = K~^T P^T        after one warp forms P[t][i] = w_ti Q[t][i] (i <= t) in fp16,
// then u[t][c] = b_t A1[c][t] + A2[c][t], written in bf16 (the precision the
// tensor-core solve reads).  The rows arrive by bulk copies, M_s by TMA.
// grid (N, B*H), block 256.
// ---------------------------------------------------------------------------
struct BwdUTcSmem {
    static constexpr uint32_t MB = 0;              // [2][128][64] fp16 M_s
    static constexpr uint32_t AT = MB + 32768;     // [2][128][64] fp16: G, V~, K~ rows (32 each)
    static constexpr uint32_t PT = AT + 32768;     // [32][64] fp16 P (K-major, 32 columns used)
    static constexpr uint32_t RK = PT + 4096;      // bf16 [32][128] k rows
    static constexpr uint32_t RV = RK + 8192;      // v rows
    static constexpr uint32_t RG = RV + 8192;      // g rows
    static constexpr uint32_t SC = RG + 8192;      // float[32] beta, float[32] gate
    static constexpr uint32_t ELL = SC + 256;      // double[32] + double[8]
    static constexpr uint32_t SB = ELL + 320;      // float[32] b, float[32] sqrt(gate)
    static constexpr uint32_t MRED = SB + 256;     // float[8][4] maxima, float scale of P
    static constexpr uint32_t BARS = MRED + 144;   // 4 mbarriers: loads, Q and A1, A2, drain
    static constexpr uint32_t TBASE = BARS + 32;
    static constexpr uint32_t END = TBASE + 16;
    static constexpr size_t bytes = END + 1024;    // + alignment slack
};

__global__ void __launch_bounds__(kSimtThreads, 2)
k_bwd_u_tc(const __grid_constant__ CUtensorMap state_map, const int *__restrict__ sexp,
           const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v,
           const float *__restrict__ beta, const float *__restrict__ gate,
           const __nv_bfloat16 *__restrict__ dout,
           __nv_bfloat16 *__restrict__ u_out, int T, int N, int *__restrict__ timeout_flag) {
    using L = BwdUTcSmem;
    constexpr int D = 128, C = kBrC;
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = smem_align1024(smraw);
    const uint32_t sb = smem_u32(sm);
    float *s_beta = reinterpret_cast<float *>(sm + L::SC), *s_gate = s_beta + 32;
    double *ell = reinterpret_cast<double *>(sm + L::ELL), *wtot = ell + C;
    float *s_b = reinterpret_cast<float *>(sm + L::SB), *s_sg = s_b + 32;
    float *mred = reinterpret_cast<float *>(sm + L::MRED);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BARS);
    uint32_t *tbase = reinterpret_cast<uint32_t *>(sm + L::TBASE);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = blockIdx.x, bh = blockIdx.y;
    const size_t tok0 = (size_t)bh * T + (size_t)n * C;
    const int srow = (int)(((size_t)bh * N + n) * 2 * D);   // H_s row in the state map; M_s follows

    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&bars[0], 32768 + 3 * 8192);
        load_state_tile(&state_map, srow + D, sm + L::MB, &bars[0]);
        bulk_g2s(sm + L::RK, k + tok0 * D, 8192, &bars[0]);
        bulk_g2s(sm + L::RV, v + tok0 * D, 8192, &bars[0]);
        bulk_g2s(sm + L::RG, dout + tok0 * D, 8192, &bars[0]);
    }
    // beta and the gate by the first 32 threads, so that the decays are formed while the
    // tiles land
    float p_gate = 1.f;
    if (tid < C) {
        s_beta[tid] = beta[tok0 + tid];
        if (gate) p_gate = gate[tok0 + tid];
    }
    if (warp == 0) {
        tc::tmem_alloc(tbase, 128);
        tc::tmem_relinquish();
    }
    __syncthreads();
    chunk_log_prefix_f32log(s_beta, C, ell, wtot);
    if (tid < C) {
        s_b[tid] = decay_exp(ell[tid]);
        s_sg[tid] = gate ? sqrtf(p_gate) : 1.f;
    }
    bool ok = mbar_wait_bounded(&bars[0], 0, kTcWaitProbes);
    __syncthreads();
    // the operand rows: item (token t, 8 columns 8j..) of each of G, V~, K~
    float gv[2][8], vv[2][8], kv[2][8];
    float mg = 0.f, mv = 0.f, mk = 0.f;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int item = tid + r * kSimtThreads, t = item >> 4, j = item & 15;
        const uint32_t off = (uint32_t)(t * 256 + j * 16);
        const uint4 ug = *reinterpret_cast<const uint4 *>(sm + L::RG + off);
        const uint4 uv = *reinterpret_cast<const uint4 *>(sm + L::RV + off);
        const uint4 uk = *reinterpret_cast<const uint4 *>(sm + L::RK + off);
        const uint32_t wg4[4] = {ug.x, ug.y, ug.z, ug.w}, wv4[4] = {uv.x, uv.y, uv.z, uv.w},
                       wk4[4] = {uk.x, uk.y, uk.z, uk.w};
        const float sg = s_sg[t];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            gv[r][2 * q] = bf16_lo(wg4[q]);
            gv[r][2 * q + 1] = bf16_hi(wg4[q]);
            vv[r][2 * q] = bf16_lo(wv4[q]) * sg;
            vv[r][2 * q + 1] = bf16_hi(wv4[q]) * sg;
            kv[r][2 * q] = bf16_lo(wk4[q]) * sg;
            kv[r][2 * q + 1] = bf16_hi(wk4[q]) * sg;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            mg = fmaxf(mg, fabsf(gv[r][e]));
            mv = fmaxf(mv, fabsf(vv[r][e]));
            mk = fmaxf(mk, fabsf(kv[r][e]));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mg = fmaxf(mg, __shfl_xor_sync(0xffffffffu, mg, o));
        mv = fmaxf(mv, __shfl_xor_sync(0xffffffffu, mv, o));
        mk = fmaxf(mk, __shfl_xor_sync(0xffffffffu, mk, o));
    }
    if (lane == 0) {
        mred[warp * 4] = mg;
        mred[warp * 4 + 1] = mv;
        mred[warp * 4 + 2] = mk;
    }
    __syncthreads();
    mg = mv = mk = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        mg = fmaxf(mg, mred[w * 4]);
        mv = fmaxf(mv, mred[w * 4 + 1]);
        mk = fmaxf(mk, mred[w * 4 + 2]);
    }
    const float sG = inv_pow2_above(mg), sV = inv_pow2_above(mv), sK = inv_pow2_above(mk);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int item = tid + r * kSimtThreads, t = item >> 4, j = item & 15;
        // row t of the 32-row block at `row0` of the 128-row region, columns 8j..8j+7
        auto put = [&](int row0, const float *x, float sc) {
            const uint32_t row = (uint32_t)(row0 + t);
            st_shared_v4(sb + L::AT + (uint32_t)(j >> 3) * 16384u + row * 128u +
                             (((uint32_t)j ^ row) & 7u) * 16u,
                         pack_f16(x[0] * sc, x[1] * sc), pack_f16(x[2] * sc, x[3] * sc),
                         pack_f16(x[4] * sc, x[5] * sc), pack_f16(x[6] * sc, x[7] * sc));
        };
        put(0, gv[r], sG);
        put(32, vv[r], sV);
        put(64, kv[r], sK);
    }
    const float sM = pow2f(sexp[((size_t)bh * N + n) * 2 + 1]);
    fence_proxy_async_smem();
    tc::fence_before_sync();
    ok = __syncthreads_and(ok);
    tc::fence_after_sync();
    const uint32_t tmem = *tbase;
    // K-major operand rows at `row0` of the region (K = d in two 64-column halves)
    auto kdesc = [&](int row0, int kk) {
        return tc::sdesc(sb + L::AT + (uint32_t)row0 * 128u + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
    };
    if (tid == 0) {
        if (ok) {
            constexpr uint32_t ID_KK = tc::idesc_f16(128, C, false, false);
            constexpr uint32_t ID_TK = tc::idesc_f16(128, C, true, false);   // A = M_s^T (MN-major)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                tc::mma_f16(tmem, kdesc(0, kk), kdesc(32, kk), ID_KK, kk > 0);
                tc::mma_f16(tmem + 32, tc::sdesc(sb + L::MB + kk * 2048, 16384, 1024), kdesc(0, kk),
                            ID_TK, kk > 0);
            }
        }
        tc::commit(&bars[1]);
    }
    if (warp == 0) {
        // P[t][i] = w_ti Q[t][i] for i <= t (t = lane), in fp16 with one power-of-two scale
        if (!mbar_wait_bounded(&bars[1], 0, kTcWaitProbes)) ok = false;
        tc::fence_after_sync();
        float q[32];
        tc::tmem_ld16(tmem, q);
        tc::tmem_ld16(tmem + 16, q + 16);
        tc::tmem_wait_ld();
        const int t = lane;
        const float uq = 1.f / (sG * sV);
        const double lt = ell[t];
        float mp = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            q[i] = i <= t ? q[i] * uq * decay_exp(lt - ell[i]) : 0.f;
            mp = fmaxf(mp, fabsf(q[i]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mp = fmaxf(mp, __shfl_xor_sync(0xffffffffu, mp, o));
        const float sP = inv_pow2_above(mp);
#pragma unroll
        for (int c = 0; c < 4; ++c)
            st_shared_v4(sb + L::PT + (uint32_t)t * 128u + (uint32_t)((c ^ t) & 7) * 16u,
                         pack_f16(q[8 * c] * sP, q[8 * c + 1] * sP),
                         pack_f16(q[8 * c + 2] * sP, q[8 * c + 3] * sP),
                         pack_f16(q[8 * c + 4] * sP, q[8 * c + 5] * sP),
                         pack_f16(q[8 * c + 6] * sP, q[8 * c + 7] * sP));
        if (lane == 0) mred[32] = sP;
        fence_proxy_async_smem();
        tc::fence_before_sync();
        ok = __all_sync(0xffffffffu, ok);
        __syncwarp();
        if (lane == 0) {
            tc::fence_after_sync();
            if (ok) {
                // A2 = K~^T P^T: A MN-major (rows i of K~, the two column halves 16384 apart)
                constexpr uint32_t ID_TK = tc::idesc_f16(128, C, true, false);
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    tc::mma_f16(tmem + 64, tc::sdesc(sb + L::AT + 64 * 128 + kk * 2048, 16384, 1024),
                                tc::sdesc(sb + L::PT + kk * 32, 16, 1024), ID_TK, kk > 0);
            }
            tc::commit(&bars[2]);
        }
        __syncwarp();
    }
    ok = __syncthreads_and(ok);
    if (!mbar_wait_bounded(&bars[2], 0, kTcWaitProbes)) ok = false;
    tc::fence_after_sync();
    // thread (row c = TMEM lane, tokens 16 wg .. 16 wg + 15)
    const int quarter = warp & 3, wg = warp >> 2, c = quarter * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(wg * 16);
    float a1[16], a2[16];
    tc::tmem_ld16(tl + 32, a1);
    tc::tmem_ld16(tl + 64, a2);
    tc::tmem_wait_ld();
    const float u1 = 1.f / (sM * sG), u2 = 1.f / (sK * mred[32]);
#pragma unroll
    for (int u = 0; u < 16; ++u) {
        const int t = wg * 16 + u;
        const float x = fmaf(a1[u] * u1, s_b[t], a2[u] * u2);
        if (ok) u_out[(tok0 + t) * D + c] = __float2bfloat16_rn(x);
    }
    if (!ok && tid == 0) {
        atomicExch(timeout_flag, 1);
        tc::commit(&bars[3]);
        mbar_wait_bounded(&bars[3], 0, kTcWaitProbes);
        mbar_wait_bounded(&bars[0], 0, kTcWaitProbes);   // the loads
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 128);
    }
}

}  // namespace gka
