// Chunk states for few heads: the sequence of every head is cut into S
// segments of whole chunks, so that S times more CTAs share the sequential
// work of the one-pass state kernel.
//
// Method: "Gated KalmaNet" (arXiv 2511.21016), ai.info page, Methodology:
// only the chunk-start states are carried across chunks, and the carry is
// linear, S_{n+1} = b_n S_n + dS_n.  Over a segment of tokens [t0, t1) the
// same carry composes to
//   S(t1) = b_seg S(t0) + A_seg,   b_seg = prod_{t0 <= m < t1} beta_m,
//   A_seg = sum_{t0 <= i < t1} w_i a_i k_i^T,  w_i = g_i prod_{i < m < t1} beta_m,
// with a = k for H and a = v for M (g the write gate, NULL = 1): the segment's
// aggregate is one product over all its tokens, A_seg = A^T diag(w) K, with no
// sequential chain inside it.  Three steps:
//   1. k_seg_delta_tc: A_seg of every segment (fp32), b_seg and the segment's
//      norm-bound increment, one CTA per (segment, head) running through the
//      segment's tokens in 64-token pieces on tcgen05, both matrices at once;
//   2. k_seg_scan: the segment-start states S(t0) by the composed carry, in
//      place of the aggregates (segments in order, element-wise), and the
//      segment-start norm bounds;
//   3. k_state_pass_tc from each segment's start state and bound, one CTA per
//      (matrix, head, segment), writing every chunk's fp16 state copy exactly
//      as the single pass over the whole sequence would.
//
// Step 1's operands: A = K or V as loaded (bf16 is exact) and the weighted
// keys w_i k_i split into two bf16 parts (hi + lo, 16 mantissa bits), as in
// the one-pass kernel; accumulation in fp32 (TMEM).  The weights are products of
// beta from the segment's end backwards: fp32 suffix products inside each
// 64-token piece, times the product over the later pieces carried in double.  Step 1 may cut the sequences finer than step 3 (S1 = K S3
// segments, so that it too fills the SMs); step 3 then starts its segment s
// from step 2's start of segment K s.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "state_tc.cuh"
#include "tcgen05.cuh"

namespace gka {

constexpr int kSegPrepWarps = 8;                          // warps forming the (w k) parts
constexpr int kSegPrepThreads = 32 * kSegPrepWarps;
constexpr int kSegThreads = kSegPrepThreads + 32;         // + the control warp
constexpr int kSegSub = 64;    // tokens per piece
constexpr int kSegStages = 4;  // stages of loaded pieces

struct SegSmem {
    static constexpr uint32_t TILE = kSegSub * 256;                // [64][128] bf16, 2 halves
    static constexpr uint32_t KS = 0;                              // stages of keys
    static constexpr uint32_t VS = KS + kSegStages * TILE;         // stages of values
    static constexpr uint32_t PARTS = VS + kSegStages * TILE;      // 2 buffers x (hi, lo)
    static constexpr uint32_t BETA = PARTS + 2 * 2 * TILE;         // [stages][64] floats
    static constexpr uint32_t GATE = BETA + kSegStages * 4 * kSegSub;
    static constexpr uint32_t W = GATE + kSegStages * 4 * kSegSub; // [2][64] weights
    static constexpr uint32_t RED = W + 2 * 4 * kSegSub;           // [2][prep warps] bound partials
    static constexpr uint32_t BARS = RED + 8 * kSegPrepWarps;    // load[stages] mma[2] wrdy[2] pdone[2] fin
    static constexpr uint32_t TBASE = BARS + 8 * (kSegStages + 7);
    static constexpr uint32_t END = TBASE + 16;
    static constexpr size_t bytes = END + 1024;
};

// Chunks [n0, n1) of segment s of S over N chunks (every segment non-empty
// when S <= N).
__host__ __device__ __forceinline__ int seg_begin(int s, int S, int N) {
    return (int)(((long long)s * N) / S);
}

// grid (S, B*H), block kSegThreads.  agg: fp32 [B*H][S][2][128][128] (H then M
// of each segment); segdec: [B*H][S]; seginc: [B*H][S][2].
//
// Warps 0-7 form the (w k) parts of each piece; warp 8 computes each piece's
// weights as soon as the piece has landed, issues the TMA loads (kSegStages
// pieces in flight) and the MMAs.  Per piece c (counted from the segment's end):
//   load(c) -> weights(c) [warp 8] -> parts(c) [warps 0-7] -> MMA(c) [warp 8],
// with parts(c) overlapping MMA(c - 1) and weights(c + 1) overlapping parts(c).
__global__ void __launch_bounds__(kSegThreads, 1)
k_seg_delta_tc(const __grid_constant__ StateMaps maps, const float *__restrict__ beta,
               const float *__restrict__ gate, float *__restrict__ agg, float *__restrict__ segdec,
               float *__restrict__ seginc, int T, int N, int C, int S,
               int *__restrict__ timeout_flag) {
    using L = SegSmem;
    constexpr int D = 128;
    constexpr uint32_t TILE = L::TILE;
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = smem_align1024(smraw);
    const uint32_t sb = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BARS);
    uint64_t *bar_load = bars, *bar_mma = bars + kSegStages, *bar_wrdy = bar_mma + 2,
             *bar_pdone = bar_wrdy + 2, *bar_fin = bar_pdone + 2;
    uint32_t *tbase = reinterpret_cast<uint32_t *>(sm + L::TBASE);
    float *s_beta = reinterpret_cast<float *>(sm + L::BETA);
    float *s_gate = reinterpret_cast<float *>(sm + L::GATE);
    float *s_w = reinterpret_cast<float *>(sm + L::W);
    float *s_red = reinterpret_cast<float *>(sm + L::RED);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool control = warp == kSegPrepWarps;
    const int s = blockIdx.x, bh = blockIdx.y;
    const int n0 = seg_begin(s, S, N), n1 = seg_begin(s + 1, S, N);
    const int nsub = (n1 - n0) * C / kSegSub;   // pieces, processed from the last one back
    const size_t tokbase = (size_t)bh * T + (size_t)n0 * C;

    if (tid == 0) {
        for (int i = 0; i < kSegStages; ++i) mbar_init(&bar_load[i], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar_mma[i], 1);
            mbar_init(&bar_wrdy[i], 1);
            mbar_init(&bar_pdone[i], kSegPrepWarps);
        }
        mbar_init(bar_fin, 1);
        fence_mbar_init();
    }
    __syncthreads();
    // control lane 0: piece c (counted from the segment's end) into stage c % kSegStages
    auto issue_load = [&](int c) {
        const int st = c % kSegStages;
        uint64_t *bar = &bar_load[st];
        mbar_arrive_expect_tx(bar, 2 * TILE + (gate ? 8u : 4u) * kSegSub);
        const size_t t = tokbase + (size_t)(nsub - 1 - c) * kSegSub;
        for (int h = 0; h < 2; ++h) {
            tc::tma_load_2d(sm + L::KS + st * TILE + h * 8192, &maps.k, h * 64, (int)t, bar);
            tc::tma_load_2d(sm + L::VS + st * TILE + h * 8192, &maps.v, h * 64, (int)t, bar);
        }
        bulk_g2s(s_beta + st * kSegSub, beta + t, 4 * kSegSub, bar);
        if (gate) bulk_g2s(s_gate + st * kSegSub, gate + t, 4 * kSegSub, bar);
    };
    // control lane 0: dS += A^T (w k) of piece c into TMEM (H: columns 0-127, M: 128-255)
    auto issue_mma = [&](uint32_t tmem, int c) {
        constexpr uint32_t ID = tc::idesc_bf16(128, 128, true, true);
        const int st = c % kSegStages;
        const uint32_t ak = sb + L::KS + st * TILE, av = sb + L::VS + st * TILE;
        const uint32_t ph = sb + L::PARTS + (c & 1) * 2 * TILE;
#pragma unroll
        for (int kk = 0; kk < kSegSub / 16; ++kk)
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                const uint64_t bd = tc::sdesc(ph + p * TILE + kk * 2048, 8192, 1024);
                const bool acc = (c | kk | p) != 0;
                tc::mma_f16(tmem + 0, tc::sdesc(ak + kk * 2048, 8192, 1024), bd, ID, acc);
                tc::mma_f16(tmem + 128, tc::sdesc(av + kk * 2048, 8192, 1024), bd, ID, acc);
            }
        tc::commit(&bar_mma[c & 1]);
    };
    // pieces 0 and 1 now; piece c + 2 once the product of piece c - 2 has freed its
    // stage (kSegStages = 4)
    static_assert(kSegStages == 4, "load schedule");
    if (control && lane == 0)
        for (int c = 0; c < 2 && c < nsub; ++c) issue_load(c);
    if (warp == 0) {
        tc::tmem_alloc(tbase, 256);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tbase;

    bool ok = true;
    double suf = 1.0;   // control warp: product of beta over the pieces after this one
    float binc_h = 0.f, binc_m = 0.f;   // prep threads: shares of the bound increments
    int last_load[kSegStages];   // control lane 0: piece last loaded into each stage
    for (int i = 0; i < kSegStages; ++i) last_load[i] = i < nsub && i < 2 ? i : -1;
    if (control) {
#pragma unroll 1
        for (int c = 0; c < nsub; ++c) {
            const int st = c % kSegStages;
            // (every wait's outcome is made warp-uniform, so the warp leaves together)
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bar_load[st], (c / kSegStages) & 1,
                                                           kStateWaitProbes))) {
                ok = false;
                break;
            }
            // weights(c) -> s_w[c & 1]: w_i = g_i prod_{m > i in the segment} beta_m,
            // as fp32 suffix products inside the piece (as the one-pass kernel forms
            // its chunk weights) times the product over the pieces after it, carried in
            // double; lane l holds tokens 2l, 2l + 1.  The buffer's last reader,
            // parts(c - 2), finished before MMA(c - 2) was issued.
            const float *bt = s_beta + st * kSegSub;
            const float b0 = bt[2 * lane], b1 = bt[2 * lane + 1];
            float tot = b0 * b1;   // -> product over the tokens of this lane and the lanes above
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_down_sync(0xffffffffu, tot, o);
                if (lane + o < 32) tot *= y;
            }
            float after = __shfl_down_sync(0xffffffffu, tot, 1);   // the lanes above
            if (lane == 31) after = 1.f;
            const float later = (float)suf;   // the pieces after this one
            float w1 = later * after, w0 = later * (after * b1);
            if (gate) {
                w0 *= s_gate[st * kSegSub + 2 * lane];
                w1 *= s_gate[st * kSegSub + 2 * lane + 1];
            }
            s_w[(c & 1) * kSegSub + 2 * lane] = w0;
            s_w[(c & 1) * kSegSub + 2 * lane + 1] = w1;
            suf *= (double)__shfl_sync(0xffffffffu, tot, 0);
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_wrdy[c & 1]);
            // MMA(c - 1) once its parts are formed
            if (c >= 1) {
                if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bar_pdone[(c - 1) & 1],
                                                               ((c - 1) >> 1) & 1, kStateWaitProbes))) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    tc::fence_after_sync();
                    issue_mma(tmem, c - 1);
                }
            }
            // MMA(c - 2) done: its stage takes piece c + 2
            if (c >= 2 && !__all_sync(0xffffffffu, mbar_wait_bounded(&bar_mma[c & 1], ((c - 2) >> 1) & 1,
                                                                     kStateWaitProbes))) {
                ok = false;
                break;
            }
            if (lane == 0 && c + 2 < nsub) {
                issue_load(c + 2);
                last_load[(c + 2) % kSegStages] = c + 2;
            }
            __syncwarp();
        }
        // the last piece's product, then every product is done
        if (ok && nsub > 0) {
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bar_pdone[(nsub - 1) & 1],
                                                           ((nsub - 1) >> 1) & 1, kStateWaitProbes)))
                ok = false;
            if (ok && lane == 0) {
                tc::fence_after_sync();
                issue_mma(tmem, nsub - 1);
            }
            __syncwarp();
            if (ok && !__all_sync(0xffffffffu, mbar_wait_bounded(&bar_mma[(nsub - 1) & 1],
                                                                 ((nsub - 1) >> 1) & 1, kStateWaitProbes)))
                ok = false;
        }
    } else {
        // parts(c): the (w k) parts of piece c in the swizzled layout of the key tile,
        // and this thread's share of the bound increments
#pragma unroll 1
        for (int c = 0; c < nsub; ++c) {
            const int st = c % kSegStages;
            const bool got =
                mbar_wait_bounded(&bar_load[st], (c / kSegStages) & 1, kStateWaitProbes) &&
                mbar_wait_bounded(&bar_wrdy[c & 1], (c >> 1) & 1, kStateWaitProbes) &&
                (c < 2 || mbar_wait_bounded(&bar_mma[c & 1], ((c - 2) >> 1) & 1, kStateWaitProbes));
            if (!__all_sync(0xffffffffu, got)) {   // warp-uniform: the warp leaves together
                ok = false;
                break;
            }
            const uint8_t *kt = sm + L::KS + st * TILE;
            const uint8_t *vt = sm + L::VS + st * TILE;
            uint8_t *pb = sm + L::PARTS + (c & 1) * 2 * TILE;
            const float *wc = s_w + (c & 1) * kSegSub;
#pragma unroll
            for (int j = 0; j < kSegSub * 16 / kSegPrepThreads; ++j) {
                const int item = tid + j * kSegPrepThreads;   // 64 rows x 16 pieces of 16 bytes
                const int r = item >> 4, l16 = item & 15;
                const uint32_t off = (uint32_t)((l16 >> 3) * 8192 + r * 128 + (l16 & 7) * 16);
                const uint4 u = *reinterpret_cast<const uint4 *>(kt + off);
                const uint4 uv = *reinterpret_cast<const uint4 *>(vt + off);
                const uint32_t uw[4] = {u.x, u.y, u.z, u.w}, vw[4] = {uv.x, uv.y, uv.z, uv.w};
                const float w = wc[r];
                float sq = 0.f, sv = 0.f;
                uint32_t p0[4], p1[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float x0 = bf16_lo(uw[q]), x1 = bf16_hi(uw[q]);
                    sq = fmaf(x0, x0, fmaf(x1, x1, sq));
                    const float y0 = w * x0, y1 = w * x1;
                    p0[q] = bf16x2_bits(y0, y1);
                    p1[q] = bf16x2_bits(y0 - bf16_lo(p0[q]), y1 - bf16_hi(p0[q]));
                    const float z0 = bf16_lo(vw[q]), z1 = bf16_hi(vw[q]);
                    sv = fmaf(z0, z0, fmaf(z1, z1, sv));
                }
                *reinterpret_cast<uint4 *>(pb + off) = make_uint4(p0[0], p0[1], p0[2], p0[3]);
                *reinterpret_cast<uint4 *>(pb + TILE + off) = make_uint4(p1[0], p1[1], p1[2], p1[3]);
                binc_h = fmaf(w, sq, binc_h);
                binc_m = fmaf(0.5f * w, sq + sv, binc_m);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_pdone[c & 1]);
        }
        binc_h = warp_sum(binc_h);
        binc_m = warp_sum(binc_m);
        if (lane == 0) {
            s_red[warp] = binc_h;
            s_red[kSegPrepWarps + warp] = binc_m;
        }
    }
    tc::fence_before_sync();
    ok = __syncthreads_and(ok);
    tc::fence_after_sync();
    if (ok) {
        if (control) {
            if (lane == 0) {
                float bh_ = 0.f, bm_ = 0.f;
                for (int w = 0; w < kSegPrepWarps; ++w) {
                    bh_ += s_red[w];
                    bm_ += s_red[kSegPrepWarps + w];
                }
                segdec[(size_t)bh * S + s] = (float)suf;
                seginc[((size_t)bh * S + s) * 2] = bh_;
                seginc[((size_t)bh * S + s) * 2 + 1] = bm_;
            }
        } else {
            // rows of the two accumulators: warp w reads lane quarter w % 4, columns
            // (w / 4) * CW .. + CW - 1 of H and of M
            constexpr int CW = 128 / (kSegPrepWarps / 4);
            const int quarter = warp & 3, half = warp >> 2;
            const int d = quarter * 32 + lane;
            const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
            float *dst = agg + ((size_t)bh * S + s) * 2 * D * D + (size_t)d * D;
#pragma unroll 1
            for (int m = 0; m < 2; ++m)
#pragma unroll
                for (int cb = 0; cb < CW; cb += 16) {
                    float v[16];
                    tc::tmem_ld16(tl + m * 128 + half * CW + cb, v);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        *reinterpret_cast<float4 *>(dst + (size_t)m * D * D + half * CW + cb + 4 * j) =
                            make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                }
        }
    } else if (control && lane == 0) {
        // a wait gave up: flag it, then drain the products and copies this lane issued
        atomicExch(timeout_flag, 1);
        tc::commit(bar_fin);
        mbar_wait_bounded(bar_fin, 0, kStateWaitProbes);
        for (int st = 0; st < kSegStages; ++st)
            if (last_load[st] >= 0)
                mbar_wait_bounded(&bar_load[st], (last_load[st] / kSegStages) & 1, kStateWaitProbes);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 256);
    }
}

// Step 2: segment-start states in place of the aggregates, element-wise over
// the segments of a head in order: start_0 = 0, start_{s+1} = b_s start_s + A_s.
// grid (2*D*D / (4 * 256), B*H), block 256 (four elements per thread).
// Block (0, bh) also scans the two norm bounds into segbound [B*H][S][2].
__global__ void __launch_bounds__(256)
k_seg_scan(float *__restrict__ agg, const float *__restrict__ segdec,
           const float *__restrict__ seginc, float *__restrict__ segbound, int S) {
    constexpr int DD2 = 2 * 128 * 128;
    const int bh = blockIdx.y;
    const int e = (blockIdx.x * 256 + threadIdx.x) * 4;
    float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
    float *base = agg + (size_t)bh * S * DD2 + e;
    // eight segments at a time: their loads go out before any store into the same
    // array (which would otherwise order every load behind the previous store)
    constexpr int kB = 8;
#pragma unroll 1
    for (int s0 = 0; s0 < S; s0 += kB) {
        float4 av[kB];
        float bv[kB];
#pragma unroll
        for (int j = 0; j < kB; ++j)
            if (s0 + j < S) {
                av[j] = *reinterpret_cast<const float4 *>(base + (size_t)(s0 + j) * DD2);
                bv[j] = segdec[(size_t)bh * S + s0 + j];
            }
#pragma unroll
        for (int j = 0; j < kB; ++j)
            if (s0 + j < S) {
                *reinterpret_cast<float4 *>(base + (size_t)(s0 + j) * DD2) = run;
                const float bb = bv[j];
                run = make_float4(fmaf(bb, run.x, av[j].x), fmaf(bb, run.y, av[j].y),
                                  fmaf(bb, run.z, av[j].z), fmaf(bb, run.w, av[j].w));
            }
    }
    if (blockIdx.x == 0 && threadIdx.x < 2) {
        float bd = 0.f;
        for (int s = 0; s < S; ++s) {
            segbound[((size_t)bh * S + s) * 2 + threadIdx.x] = bd;
            bd = fmaf(segdec[(size_t)bh * S + s], bd, seginc[((size_t)bh * S + s) * 2 + threadIdx.x]);
        }
    }
}

}  // namespace gka
