// Tensor-core chunk increments of the chunk-state scan (bf16 inputs, D = 128).
//
// Method: "Gated KalmaNet" (arXiv 2511.21016), ai.info page, Methodology:
// only the chunk-start states are carried sequentially.  The state after
// chunk n is  S_{n+1} = b_{C-1} S_n + dS_n  with
//   dH_n = sum_i w_{C-1,i} k_i k_i^T = K^T diag(w) K,
//   dM_n = sum_i w_{C-1,i} v_i k_i^T = V^T diag(w) K,
// two 128 x 128 x C products per chunk; the scan kernel adds them up.  With
// the write gate g (nullable) every weight w_{C-1,i} is w_{C-1,i} g_i.
//
// C = 64 or 128 in the forward (tensor maps of 64-row boxes), C = 32 in the
// backward's recompute of the chunk states (32-row boxes; no per-token decays
// or norm bounds: tokdec and bound_inc are NULL there).
//
// One CTA (4 warps) per chunk.  K and V arrive by TMA (bf16) and are turned
// into fp16 with a power-of-two scale below 1 (exact).  The weighted keys
// diag(w) K are split into fp16 hi + lo parts (hi + lo carries 22 mantissa
// bits, about fp32), so the increments come out at fp32 accuracy from fp16
// MMAs: dH = K^T (W K)_hi + K^T (W K)_lo, the same for dM with V^T.
// Thread d reads row d of each fp32 accumulator from TMEM and writes it to
// the state slot n + 1.  The CTA also writes the chunk decay b_{C-1} and the
// increments of the norm bounds used to scale the scan's fp16 state copies,
// and every token's decays for the solve: l_t log2(e), b_t = exp(l_t),
// beta_t and beta_t^2 (l_t the chunk-relative cumulative log, summed in double).
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "solve_tc.cuh"
#include "tcgen05.cuh"

namespace gka {

template <int C>
struct DeltaSmem {
    static constexpr uint32_t KT = 0;                 // 2 x [C][64] keys (bf16 -> fp16)
    static constexpr uint32_t VT = KT + C * 256;      // 2 x [C][64] values
    static constexpr uint32_t WH = VT + C * 256;      // 2 x [C][64] (w k)_hi
    static constexpr uint32_t WL = WH + C * 256;      // 2 x [C][64] (w k)_lo
    static constexpr uint32_t STAGE = WL + C * 256;   // 2 x [128][32] fp32 store staging (swizzled)
    static constexpr uint32_t ELL = STAGE + 32768;    // double[C] cumulative logs
    static constexpr uint32_t WT = ELL + 8 * C + 8 * (kTcThreads / 32);   // float[C] weights
    static constexpr uint32_t RED = WT + 4 * C;
    static constexpr uint32_t BARS = RED + 64;
    static constexpr uint32_t TBASE = BARS + 32;
    static constexpr uint32_t END = TBASE + 16;
    // at least 80 KB so that at most two CTAs (2 x 256 TMEM columns) share an SM
    static constexpr size_t bytes = END + 1024 > 81920 ? END + 1024 : 81920;
};

struct DeltaMaps {
    CUtensorMap k, v;    // [B*H*T][128] bf16, box 64 x min(C, 64), 128B swizzle
    CUtensorMap out;     // fp32 states [B*H*(N+1)*2*128][128], box 32 x 128, 128B swizzle
};

// grid (N, B*H), block 128.
template <int C>
__global__ void __launch_bounds__(kTcThreads, 1)
k_chunk_delta_tc(const __grid_constant__ DeltaMaps maps, const float *__restrict__ beta,
                 const float *__restrict__ gate, float *__restrict__ states, float *__restrict__ decay,
                 float *__restrict__ bound_inc, float *__restrict__ tokdec, size_t plane, int T,
                 int N, int *__restrict__ timeout_flag) {
    using L = DeltaSmem<C>;
    constexpr int D = kTcD;
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = smem_align1024(smraw);
    const uint32_t sb = smem_u32(sm);
    double *ell = reinterpret_cast<double *>(sm + L::ELL);
    double *wtot = ell + C;
    float *s_wt = reinterpret_cast<float *>(sm + L::WT);   // w_{C-1,i} g_i
    float *red = reinterpret_cast<float *>(sm + L::RED);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BARS);
    uint64_t *bar_load = &bars[0], *bar_mma = &bars[1];
    uint32_t *tbase = reinterpret_cast<uint32_t *>(sm + L::TBASE);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = blockIdx.x, bh = blockIdx.y;
    const size_t tok0 = (size_t)bh * T + (size_t)n * C;

    if (tid == 0) {
        mbar_init(bar_load, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
    }
    __syncthreads();
    constexpr int BOX = C < 64 ? C : 64;   // rows per TMA box
    if (tid == 0) {
        mbar_arrive_expect_tx(bar_load, 2 * C * 256);
        for (int h = 0; h < 2; ++h)
            for (int rb = 0; rb < C / BOX; ++rb) {
                tc::tma_load_2d(sm + L::KT + h * C * 128 + rb * BOX * 128, &maps.k, h * 64,
                                (int)tok0 + rb * BOX, bar_load);
                tc::tma_load_2d(sm + L::VT + h * C * 128 + rb * BOX * 128, &maps.v, h * 64,
                                (int)tok0 + rb * BOX, bar_load);
            }
    }
    if (warp == 0) {
        tc::tmem_alloc(tbase, 256);
        tc::tmem_relinquish();
    }
    chunk_log_prefix(beta + tok0, C, ell, wtot);
    if (tid < C) {
        if (tokdec) {
            const float bt = decay_exp(tid == 0 ? ell[0] : ell[tid] - ell[tid - 1]);
            tokdec[tok0 + tid] = (float)(ell[tid] * 1.4426950408889634);
            tokdec[plane + tok0 + tid] = decay_exp(ell[tid]);
            tokdec[2 * plane + tok0 + tid] = bt;
            tokdec[3 * plane + tok0 + tid] = bt * bt;
        }
        float w = decay_exp(ell[C - 1] - ell[tid]);
        if (gate) w *= gate[tok0 + tid];   // write gate of token tid
        s_wt[tid] = w;
    }
    bool ok = mbar_wait_bounded(bar_load, 0, kTcWaitProbes);
    const float sK = tile_bf16_to_f16_scaled<C * 256, kTcThreads>(sm + L::KT, red);
    const float sV = tile_bf16_to_f16_scaled<C * 256, kTcThreads>(sm + L::VT, red);

    // (w k)_hi and (w k)_lo tiles, same swizzled layout as the key tile: the
    // 16-byte chunk at byte c of half h belongs to key row (c % (C*128)) / 128
    const double lend = ell[C - 1];
    for (int c = tid * 16; c < C * 256; c += kTcThreads * 16) {
        const int row = (c % (C * 128)) >> 7;
        const float w = s_wt[row];
        const uint4 u = *reinterpret_cast<const uint4 *>(sm + L::KT + c);
        const __half *e = reinterpret_cast<const __half *>(&u);
        float hv[8], lv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float x = w * __half2float(e[i]);
            hv[i] = __half2float(__float2half_rn(x));
            lv[i] = x - hv[i];
        }
        uint4 hw, lw;
        hw.x = pack_f16(hv[0], hv[1]); hw.y = pack_f16(hv[2], hv[3]);
        hw.z = pack_f16(hv[4], hv[5]); hw.w = pack_f16(hv[6], hv[7]);
        lw.x = pack_f16(lv[0], lv[1]); lw.y = pack_f16(lv[2], lv[3]);
        lw.z = pack_f16(lv[4], lv[5]); lw.w = pack_f16(lv[6], lv[7]);
        *reinterpret_cast<uint4 *>(sm + L::WH + c) = hw;
        *reinterpret_cast<uint4 *>(sm + L::WL + c) = lw;
    }
    fence_proxy_async_smem();
    tc::fence_before_sync();
    ok = __syncthreads_and(ok);
    tc::fence_after_sync();
    const uint32_t tmem = *tbase;
    if (tid == 0 && ok) {
        constexpr uint32_t ID = tc::idesc_f16(128, 128, true, true);
        const uint32_t a_k = sb + L::KT, a_v = sb + L::VT, b_h = sb + L::WH, b_l = sb + L::WL;
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) {
            const uint64_t bh_d = tc::sdesc(b_h + kk * 2048, C * 128, 1024);
            const uint64_t bl_d = tc::sdesc(b_l + kk * 2048, C * 128, 1024);
            const uint64_t ak_d = tc::sdesc(a_k + kk * 2048, C * 128, 1024);
            const uint64_t av_d = tc::sdesc(a_v + kk * 2048, C * 128, 1024);
            tc::mma_f16(tmem + 0, ak_d, bh_d, ID, kk > 0);
            tc::mma_f16(tmem + 0, ak_d, bl_d, ID, true);
            tc::mma_f16(tmem + 128, av_d, bh_d, ID, kk > 0);
            tc::mma_f16(tmem + 128, av_d, bl_d, ID, true);
        }
        tc::commit(bar_mma);
    }
    // chunk decay and the norm-bound increments sum_i w_i ||k_i||^2, sum_i w_i ||v_i|| ||k_i||
    if (bound_inc) {
        float bhs = 0.f, bms = 0.f;
        for (int i = tid; i < C; i += kTcThreads) {
            const float w = s_wt[i];
            float kk2 = 0.f, vv2 = 0.f;
            for (int h = 0; h < 2; ++h) {
                const __half *kr = reinterpret_cast<const __half *>(sm + L::KT + h * C * 128 + i * 128);
                const __half *vr = reinterpret_cast<const __half *>(sm + L::VT + h * C * 128 + i * 128);
                for (int e = 0; e < 64; ++e) {
                    const float kx = __half2float(kr[(e + i) & 63]);
                    const float vx = __half2float(vr[(e + i) & 63]);
                    kk2 = fmaf(kx, kx, kk2);
                    vv2 = fmaf(vx, vx, vv2);
                }
            }
            kk2 /= sK * sK;
            vv2 /= sV * sV;
            bhs = fmaf(w, kk2, bhs);
            bms = fmaf(w, sqrtf(kk2) * sqrtf(vv2), bms);
        }
        bhs = warp_sum(bhs);
        bms = warp_sum(bms);
        if (lane == 0) {
            red[8 + warp] = bhs;
            red[12 + warp] = bms;
        }
    }
    if (!mbar_wait_bounded(bar_mma, 0, kTcWaitProbes)) ok = false;
    tc::fence_after_sync();
    ok = __syncthreads_and(ok);
    if (ok) {
        if (tid == 0) {
            decay[(size_t)bh * N + n] = decay_exp(lend);
            if (bound_inc) {
                bound_inc[((size_t)bh * N + n) * 2] = red[8] + red[9] + red[10] + red[11];
                bound_inc[((size_t)bh * N + n) * 2 + 1] = red[12] + red[13] + red[14] + red[15];
            }
        }
        // row d of dH and dM (thread d = TMEM lane d) -> swizzled staging -> TMA store
        // into state slot n + 1, 64 columns (two 32-column boxes) per round
        const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
        const float uh = 1.f / (sK * sK), um = 1.f / (sV * sK);
        const int orow = (int)(((size_t)bh * (N + 1) + n + 1) * 2 * D);
#pragma unroll 1
        for (int round = 0; round < 4; ++round) {
            const int m = round >> 1, cb0 = (round & 1) * 64;
            const float us = m == 0 ? uh : um;
#pragma unroll
            for (int bx = 0; bx < 2; ++bx) {
                float v0[16], v1[16];
                tc::tmem_ld16(tl + m * 128 + cb0 + bx * 32, v0);
                tc::tmem_ld16(tl + m * 128 + cb0 + bx * 32 + 16, v1);
                tc::tmem_wait_ld();
                const uint32_t rowb = sb + L::STAGE + bx * 16384 + tid * 128;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float *vv = j < 4 ? v0 + 4 * j : v1 + 4 * (j - 4);
                    st_shared_v4(rowb + ((j ^ tid) & 7) * 16, __float_as_uint(vv[0] * us),
                                 __float_as_uint(vv[1] * us), __float_as_uint(vv[2] * us),
                                 __float_as_uint(vv[3] * us));
                }
            }
            fence_proxy_async_smem();
            __syncthreads();
            if (tid == 0) {
                tc::tma_store_2d(&maps.out, cb0, orow + m * D, sm + L::STAGE);
                tc::tma_store_2d(&maps.out, cb0 + 32, orow + m * D, sm + L::STAGE + 16384);
                tc::bulk_commit();
                tc::bulk_wait_read0();
            }
            __syncthreads();
        }
        if (tid == 0) tc::bulk_wait0();
    } else if (tid == 0) {
        atomicExch(timeout_flag, 1);
        tc::commit(bar_mma);   // drain: a second arrival after whatever is still in flight
        mbar_wait_bounded(bar_mma, 1, kTcWaitProbes);
        mbar_wait_bounded(bar_load, 0, kTcWaitProbes);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 256);
    }
}

}  // namespace gka
