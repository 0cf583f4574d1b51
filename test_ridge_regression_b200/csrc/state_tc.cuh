// Tensor-core chunk-state pass: the sequential part of the chunk-wise GKA
// forward in one kernel, bf16 inputs, D = 128.
//
// Method: "Gated KalmaNet" (arXiv 2511.21016), ai.info page, Methodology:
// only the chunk-start states are carried across chunks,
//   S_0 = 0,   S_{n+1} = b_n S_n + dS_n,
//   dH_n = K^T diag(w) K,   dM_n = V^T diag(w) K,   w_i = exp(l_{C-1} - l_i),
// with l the chunk-relative cumulative log of beta and b_n = exp(l_{C-1}).
//
// One CTA per (head, matrix): blockIdx.x = 0 carries H, 1 carries M.  The
// fp32 state lives in registers for the whole sequence (thread (h, d) owns
// row d, columns 64h..64h+63), so no state ever goes through memory in fp32.
// Per chunk:
//   - K (and V) arrive by TMA, bf16, two chunks ahead; beta with them;
//   - every warp forms the chunk's log-decay prefix (fp32 logs summed in
//     double) in registers; the H CTA writes the per-token decays the solve
//     reads and the chunk decay;
//   - the weighted keys w_i k_i are split into bf16 parts (three for 64-token
//     chunks, about fp32; two for 128-token chunks, 16 mantissa bits) in the
//     swizzled layout of the key tile; dS = A^T (wK) with A = K or V as loaded
//     (bf16 is exact) accumulates the parts on tcgen05 into one of two TMEM
//     buffers, while the threads write the fp16 copy of S_n and fold in
//     dS_{n-1} from the other buffer;
//   - the fp16 copy is scaled by 2^e_n with e_n from the running bound
//     ||S_n||_F <= bound_n, bound_{n+1} = b_n bound_n + sum_i w_i |k_i|^2 (H)
//     or sum_i w_i |v_i| |k_i| (M), so that every copied value is <= 2^14.
// The state after the last chunk goes to final_state (nullable).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "tcgen05.cuh"

namespace gka {

constexpr int kStateThreads = 256;
constexpr uint32_t kStateWaitProbes = 1u << 22;

// Exponent e such that |value| <= bound implies |value * 2^e| <= 2^14.
__device__ __forceinline__ int lp_exponent_tc(float bound) {
    if (!(bound > 0.f)) return 0;
    const int e = 14 - (ilogbf(bound) + 1);
    return e < -120 ? -120 : (e > 120 ? 120 : e);
}

template <int C>
struct StateSmem {
    static constexpr int NP = C == 64 ? 3 : 2;              // bf16 parts of w k
    static constexpr uint32_t TILE = C * 256;               // one [C][128] bf16 tile (2 halves)
    static constexpr uint32_t KS = 0;                       // 2 stages of keys
    static constexpr uint32_t VS = KS + 2 * TILE;           // 2 stages of values (M CTA)
    static constexpr uint32_t PARTS = VS + 2 * TILE;        // NP tiles of (w k) parts
    static constexpr uint32_t BETA = PARTS + NP * TILE;     // 2 stages of beta [C] floats
    static constexpr uint32_t WW = BETA + 2 * 4 * C;        // per-warp w [8][C] floats
    static constexpr uint32_t RED = WW + 8 * 4 * C;         // per-warp partial bound increments
    static constexpr uint32_t BARS = RED + 64;              // load[2], mma[2], fin
    static constexpr uint32_t TBASE = BARS + 8 * 8;
    static constexpr uint32_t END = TBASE + 16;
    static constexpr size_t bytes = END + 1024;             // + alignment slack
};

struct StateMaps {
    CUtensorMap k, v;    // [B*H*T][128] bf16, box 64 x 64, 128B swizzle
};

// Pairs of consecutive values as packed bf16x2 / fp16x2 words (low half first).
__device__ __forceinline__ uint32_t pack_bf16(__nv_bfloat16 lo, __nv_bfloat16 hi) {
    return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    const __half2 p = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&p);
}

// grid (2, B*H), block 256.  T = N * C.
template <int C>
__global__ void __launch_bounds__(kStateThreads, 1)
k_state_pass_tc(const __grid_constant__ StateMaps maps, const float *__restrict__ beta,
                __half *__restrict__ slp, int *__restrict__ state_exp,
                float *__restrict__ decay, float *__restrict__ tokdec, size_t plane,
                float *__restrict__ final_state, int T, int N, int *__restrict__ timeout_flag) {
    using L = StateSmem<C>;
    constexpr int D = 128, NP = L::NP, PER = C / 32;
    constexpr uint32_t TILE = L::TILE;
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smraw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BARS);
    uint64_t *bar_load = bars, *bar_mma = bars + 2, *bar_fin = bars + 4;
    uint32_t *tbase = reinterpret_cast<uint32_t *>(sm + L::TBASE);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const int d = quarter * 32 + lane;          // state row of this thread = its TMEM lane
    const int m = blockIdx.x, bh = blockIdx.y;  // m = 0: H, 1: M
    const bool is_m = m == 1;
    const size_t tokbase = (size_t)bh * T;
    float *s_beta = reinterpret_cast<float *>(sm + L::BETA);       // [2][C]
    float *s_ww = reinterpret_cast<float *>(sm + L::WW) + warp * C;  // this warp's w [C]
    float *s_red = reinterpret_cast<float *>(sm + L::RED);         // [2][8]

    if (tid == 0) {
        for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    __syncthreads();

    int last_load[2] = {-1, -1};   // thread 0: chunk last loaded into each stage
    // thread 0: chunk c (keys, values for M, beta) into stage c & 1
    auto issue_load = [&](int c) {
        const int st = c & 1;
        uint64_t *bar = &bar_load[st];
        mbar_arrive_expect_tx(bar, TILE * (is_m ? 2u : 1u) + 4u * C);
        const int row0 = (int)(tokbase + (size_t)c * C);
        for (int h = 0; h < 2; ++h)
            for (int rb = 0; rb < C / 64; ++rb) {
                const uint32_t o = st * TILE + h * C * 128 + rb * 8192;
                tc::tma_load_2d(sm + L::KS + o, &maps.k, h * 64, row0 + rb * 64, bar);
                if (is_m) tc::tma_load_2d(sm + L::VS + o, &maps.v, h * 64, row0 + rb * 64, bar);
            }
        bulk_g2s(s_beta + st * C, beta + tokbase + (size_t)c * C, 4 * C, bar);
        last_load[st] = c;
    };
    if (tid == 0) {
        issue_load(0);
        if (N > 1) issue_load(1);
    }
    if (warp == 0) {
        tc::tmem_alloc(tbase, 256);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tbase;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(half * 64);

    // Log-decay prefix of chunk c, by every warp for itself: w_t into s_ww, the
    // chunk decay into bn.  The H CTA's warp 0 also writes the per-token decays
    // (l_t log2 e, exp(l_t), beta_t, beta_t^2) and the chunk decay.
    auto prefix = [&](int c, float &bn) {
        const float *bt = s_beta + (c & 1) * C;
        double x[PER];
        double run = 0.0;
#pragma unroll
        for (int p = 0; p < PER; ++p) {
            run += fmax((double)logf(bt[lane * PER + p]), kLogBetaMin);
            x[p] = run;
        }
        double tot = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double y = __shfl_up_sync(0xffffffffu, tot, o);
            if (lane >= o) tot += y;
        }
        const double excl = tot - run;
#pragma unroll
        for (int p = 0; p < PER; ++p) x[p] += excl;   // l of token lane*PER + p
        const double lend = __shfl_sync(0xffffffffu, tot, 31);
#pragma unroll
        for (int p = 0; p < PER; ++p) s_ww[lane * PER + p] = decay_exp(lend - x[p]);
        bn = decay_exp(lend);
        if (!is_m && warp == 0) {
            double prev = __shfl_up_sync(0xffffffffu, x[PER - 1], 1);
            if (lane == 0) prev = 0.0;
#pragma unroll
            for (int p = 0; p < PER; ++p) {
                const size_t g = tokbase + (size_t)c * C + lane * PER + p;
                const float b1 = decay_exp(x[p] - (p == 0 ? prev : x[p - 1]));
                tokdec[g] = (float)(x[p] * 1.4426950408889634);
                tokdec[plane + g] = decay_exp(x[p]);
                tokdec[2 * plane + g] = b1;
                tokdec[3 * plane + g] = b1 * b1;
            }
            if (lane == 0) decay[(size_t)bh * N + c] = bn;
        }
        __syncwarp();
    };

    // B operand of chunk c: the parts of w_i k_i (bf16, the key tile's swizzled
    // layout: the 16-byte chunk at a byte offset holds the same elements in
    // every tile), and this CTA's bound increment into s_red[c & 1][warp].
    // 16 consecutive threads take the 16 chunks of one key row.
    auto prep = [&](int c) {
        const uint8_t *kt = sm + L::KS + (c & 1) * TILE;
        const uint8_t *vt = sm + L::VS + (c & 1) * TILE;
        float acc = 0.f;
#pragma unroll 1
        for (int item = tid; item < C * 16; item += kStateThreads) {
            const int r = item >> 4, l16 = item & 15;
            const uint32_t off = (uint32_t)((l16 >> 3) * (C * 128) + r * 128 + (l16 & 7) * 16);
            const uint4 u = *reinterpret_cast<const uint4 *>(kt + off);
            const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&u);
            const float w = s_ww[r];
            float kk = 0.f;
            __nv_bfloat16 h0[8], h1[8], h2[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float x = __bfloat162float(e[i]);
                kk = fmaf(x, x, kk);
                const float y = w * x;
                h0[i] = __float2bfloat16_rn(y);
                const float r1 = y - __bfloat162float(h0[i]);
                h1[i] = __float2bfloat16_rn(r1);
                if (NP == 3) h2[i] = __float2bfloat16_rn(r1 - __bfloat162float(h1[i]));
            }
            uint4 p0, p1;
            p0.x = pack_bf16(h0[0], h0[1]); p0.y = pack_bf16(h0[2], h0[3]);
            p0.z = pack_bf16(h0[4], h0[5]); p0.w = pack_bf16(h0[6], h0[7]);
            p1.x = pack_bf16(h1[0], h1[1]); p1.y = pack_bf16(h1[2], h1[3]);
            p1.z = pack_bf16(h1[4], h1[5]); p1.w = pack_bf16(h1[6], h1[7]);
            *reinterpret_cast<uint4 *>(sm + L::PARTS + off) = p0;
            *reinterpret_cast<uint4 *>(sm + L::PARTS + TILE + off) = p1;
            if (NP == 3) {
                uint4 p2;
                p2.x = pack_bf16(h2[0], h2[1]); p2.y = pack_bf16(h2[2], h2[3]);
                p2.z = pack_bf16(h2[4], h2[5]); p2.w = pack_bf16(h2[6], h2[7]);
                *reinterpret_cast<uint4 *>(sm + L::PARTS + 2 * TILE + off) = p2;
            }
            float vv = 0.f;
            if (is_m) {
                const uint4 uv = *reinterpret_cast<const uint4 *>(vt + off);
                const __nv_bfloat16 *ev = reinterpret_cast<const __nv_bfloat16 *>(&uv);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float x = __bfloat162float(ev[i]);
                    vv = fmaf(x, x, vv);
                }
            }
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) {
                kk += __shfl_xor_sync(0xffffffffu, kk, o);
                vv += __shfl_xor_sync(0xffffffffu, vv, o);
            }
            if (l16 == 0) acc += is_m ? w * sqrtf(kk) * sqrtf(vv) : w * kk;
        }
        acc = warp_sum(acc);
        if (lane == 0) s_red[(c & 1) * 8 + warp] = acc;
    };

    // thread 0: dS_c = A^T (w K) into TMEM buffer c & 1 (A = K or V of stage c & 1)
    auto issue_mma = [&](int c) {
        constexpr uint32_t ID = tc::idesc_bf16(128, 128, true, true);
        const uint32_t a = sb + (is_m ? L::VS : L::KS) + (c & 1) * TILE;
#pragma unroll
        for (int p = 0; p < NP; ++p)
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                tc::mma_f16(tmem + (c & 1) * 128, tc::sdesc(a + kk * 2048, C * 128, 1024),
                            tc::sdesc(sb + L::PARTS + p * TILE + kk * 2048, C * 128, 1024), ID,
                            (p | kk) != 0);
        tc::commit(&bar_mma[c & 1]);
    };

    // ---- prologue: chunk 0's operands and product ----
    bool ok = mbar_wait_bounded(&bar_load[0], 0, kStateWaitProbes);
    float b_next = 0.f;
    prefix(0, b_next);
    prep(0);
    fence_proxy_async_smem();
    ok = __syncthreads_and(ok);
    float binc_next = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) binc_next += s_red[w];
    if (tid == 0 && ok) issue_mma(0);

    float st[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) st[i] = 0.f;
    float bound = 0.f;
    const size_t DD = (size_t)D * D;

#pragma unroll 1
    for (int n = 0; n < N && ok; ++n) {
        const float bn = b_next, bincn = binc_next;   // chunk n's decay and bound increment
        // dS_n is ready; stage n & 1 and the parts are free again
        if (!mbar_wait_bounded(&bar_mma[n & 1], (n >> 1) & 1, kStateWaitProbes)) ok = false;
        tc::fence_after_sync();
        if (tid == 0 && n + 2 < N) issue_load(n + 2);
        if (n + 1 < N) {
            // chunk n + 1's operands; its product runs during this chunk's update
            if (!mbar_wait_bounded(&bar_load[(n + 1) & 1], ((n + 1) >> 1) & 1, kStateWaitProbes))
                ok = false;
            prefix(n + 1, b_next);
            prep(n + 1);
            fence_proxy_async_smem();
            tc::fence_before_sync();
            ok = __syncthreads_and(ok);
            tc::fence_after_sync();
            binc_next = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) binc_next += s_red[((n + 1) & 1) * 8 + w];
            if (tid == 0 && ok) issue_mma(n + 1);
        }
        // fp16 copy of the chunk-start state S_n, scaled by 2^e_n
        const int ex = lp_exponent_tc(bound);
        {
            const float sc = ldexpf(1.f, ex);
            __half *dst = slp + (((size_t)bh * N + n) * 2 + m) * DD + (size_t)d * D + half * 64;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                uint4 w4;
                w4.x = pack_h2(st[8 * j] * sc, st[8 * j + 1] * sc);
                w4.y = pack_h2(st[8 * j + 2] * sc, st[8 * j + 3] * sc);
                w4.z = pack_h2(st[8 * j + 4] * sc, st[8 * j + 5] * sc);
                w4.w = pack_h2(st[8 * j + 6] * sc, st[8 * j + 7] * sc);
                *reinterpret_cast<uint4 *>(dst + 8 * j) = w4;
            }
            if (tid == 0) state_exp[((size_t)bh * N + n) * 2 + m] = ex;
        }
        // S_{n+1} = b_n S_n + dS_n
        {
            float dl[64];
#pragma unroll
            for (int cb = 0; cb < 64; cb += 16) tc::tmem_ld16(tl + (n & 1) * 128 + cb, dl + cb);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 64; ++i) st[i] = fmaf(bn, st[i], dl[i]);
        }
        bound = fmaf(bn, bound, bincn);
    }

    if (ok && final_state) {
        float *dst = final_state + ((size_t)bh * 2 + m) * DD + (size_t)d * D + half * 64;
#pragma unroll
        for (int j = 0; j < 16; ++j)
            *reinterpret_cast<float4 *>(dst + 4 * j) =
                make_float4(st[4 * j], st[4 * j + 1], st[4 * j + 2], st[4 * j + 3]);
    }

    // teardown: no MMA or copy of this CTA may be in flight when TMEM is freed
    tc::fence_before_sync();
    ok = __syncthreads_and(ok);
    if (!ok && tid == 0) {
        atomicExch(timeout_flag, 1);
        tc::commit(bar_fin);
        mbar_wait_bounded(bar_fin, 0, kStateWaitProbes);
        for (int s2 = 0; s2 < 2; ++s2)
            if (last_load[s2] >= 0)
                mbar_wait_bounded(&bar_load[s2], (last_load[s2] >> 1) & 1, kStateWaitProbes);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 256);
    }
}

}  // namespace gka
