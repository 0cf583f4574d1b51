// Tensor-core chunk-state pass: the sequential part of the chunk-wise GKA
// forward in one kernel, bf16 inputs, D = 128.
//
// Method: "Gated KalmaNet" (arXiv 2511.21016), ai.info page, Methodology:
// only the chunk-start states are carried across chunks,
//   S_0 = 0,   S_{n+1} = b_n S_n + dS_n,
//   dH_n = K^T diag(w) K,   dM_n = V^T diag(w) K,   w_i = g_i prod_{m > i} beta_m,
// with b_n = prod_m beta_m over chunk n (the exp of the chunk's summed log decay)
// and g_i the write gate of token i (the paper's beta_t-augmented variant,
// ai.info page, Main Findings; `gate` nullable, NULL = 1).
//
// One CTA per (head, matrix): blockIdx.x = 0 carries H, 1 carries M.  The
// fp32 state lives in registers for the whole sequence (arithmetic thread
// (g, d) owns row d, columns 32g..32g+31), so no state goes through memory in
// fp32.  Warps 0-15 do the arithmetic; warp 16 issues the TMA loads, the MMAs
// and the TMA stores; warp 17 forms each chunk's decays as soon as the chunk
// has landed, so that neither waiting on the tensor core nor that bookkeeping
// stalls an arithmetic warp.
// Per chunk:
//   - K (and V) arrive by TMA, bf16, two chunks ahead; beta with them;
//   - the decay warp forms w (suffix products of beta) and b_n, published
//     through an mbarrier; in the H CTA it also writes the per-token decays the
//     solve reads (from fp32 logs summed in double) and the chunk decay;
//   - the weighted keys w_i k_i are split into two bf16 parts (hi + lo, 16
//     mantissa bits; the final state stays within a few 1e-6 of the float64
//     oracle) in the swizzled layout of the key tile; dS = A^T (wK) with A = K or V as loaded
//     (bf16 is exact) accumulates the parts on tcgen05 into one of two TMEM
//     buffers, while the arithmetic warps stage the fp16 copy of S_n in shared
//     memory (written out by one TMA store) and fold in dS_{n-1} from the
//     other buffer; with 64-token chunks the parts are double-buffered too, so
//     the next chunk's parts are formed while the current product runs;
//   - the fp16 copy is scaled by 2^e_n with e_n from a running bound
//     ||S_n||_F <= bound_n, bound_{n+1} = b_n bound_n + inc_n, with
//     inc_n = sum_i w_i |k_i|^2 >= ||dH_n||_F for H and
//     inc_n = sum_i w_i (|v_i|^2 + |k_i|^2) / 2 >= sum_i w_i |v_i| |k_i| >= ||dM_n||_F
//     for M (both linear in the elements, so no per-row reduction), which keeps
//     every copied value <= 2^14.
// The state after the last chunk goes to final_state (nullable).
//
// C = 32 serves the backward's recompute (32-row TMA boxes; tokdec may be NULL:
// then no per-token decays, the chunk decays as always).
//
// With S > 1 the sequence of every head is cut into S segments of whole chunks
// (seg_tc.cuh): CTA (m, bh * S + s) runs segment s from its start state
// seg_start[bh][K s] and norm bound seg_bound[bh][K s] (fp32, from the scan over
// the K S finer segments of the aggregates) instead of from zero, and only the
// last segment writes final_state.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "tcgen05.cuh"

namespace gka {

constexpr int kStateEpiThreads = 512;                    // arithmetic warps 0-15
constexpr int kStateBarThreads = kStateEpiThreads + 32;  // + the issuing warp 16
constexpr int kStateThreads = kStateBarThreads + 32;     // + the decay warp 17
constexpr uint32_t kStateWaitProbes = 1u << 22;

// Exponent e such that |value| <= bound implies |value * 2^e| <= 2^14.
__device__ __forceinline__ int lp_exponent_tc(float bound) {
    if (!(bound > 0.f)) return 0;
    const int e = 14 - (ilogbf(bound) + 1);
    return e < -120 ? -120 : (e > 120 ? 120 : e);
}

template <int C>
struct StateSmem {
    static constexpr int NP = 2;                            // bf16 parts of w k (hi, lo)
    static constexpr int NPB = C <= 64 ? 2 : 1;             // buffers of parts
    static constexpr uint32_t TILE = C * 256;               // one [C][128] bf16 tile (2 halves)
    static constexpr uint32_t KS = 0;                       // 2 stages of keys
    static constexpr uint32_t VS = KS + 2 * TILE;           // 2 stages of values (M CTA)
    static constexpr uint32_t PARTS = VS + 2 * TILE;        // NPB x NP tiles of (w k) parts
    // fp16 staging of one state copy, [2 column halves][128 rows][64], 128B-swizzled:
    // own space for chunks of up to 64 tokens; with 128-token chunks the H CTA stages
    // in its (unused) value stages and the M CTA in the key stage of the chunk it has
    // just prepared (free until that stage is loaded again)
    static constexpr uint32_t OUTB = C <= 64 ? 32768 : 0;
    static constexpr uint32_t OUT = PARTS + NPB * NP * TILE;
    static constexpr uint32_t BETA = OUT + OUTB;            // [2][C]
    static constexpr uint32_t GATE = BETA + 2 * 4 * C;      // [2][C] write gates
    static constexpr uint32_t W = GATE + 2 * 4 * C;         // [2][C] w of the chunks in flight
    static constexpr uint32_t BN = W + 2 * 4 * C;           // [2] chunk decays (16 bytes)
    static constexpr uint32_t RED = BN + 16;                // [2][16] partial bound increments
    static constexpr uint32_t BARS = RED + 128;             // load[2] mma[2] fin w[2] out
    static constexpr uint32_t TBASE = BARS + 8 * 8;
    static constexpr uint32_t END = TBASE + 16;
    static constexpr size_t bytes = END + 1024;             // + alignment slack
};

struct StateMaps {
    CUtensorMap k, v;    // [B*H*T][128] bf16, box 64 x 64, 128B swizzle
    CUtensorMap out;     // fp16 state copies [B*H*N*2*128][128], box 64 x 128, 128B swizzle
};

// A pair of floats as packed bf16x2 (first value in the low half), and back.
__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&p);
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    const __half2 p = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&p);
}

// grid (2, B*H*S), block kStateThreads.  T = N * C.  seg_start: fp32
// [B*H][K*S][2][128][128], seg_bound: [B*H][K*S][2] (both unused when S == 1).
template <int C>
__global__ void __launch_bounds__(kStateThreads, 1)
k_state_pass_tc(const __grid_constant__ StateMaps maps, const float *__restrict__ beta,
                const float *__restrict__ gate, int *__restrict__ state_exp, float *__restrict__ decay,
                float *__restrict__ tokdec, size_t plane, float *__restrict__ final_state,
                int T, int N, int S, int K, const float *__restrict__ seg_start,
                const float *__restrict__ seg_bound, int *__restrict__ timeout_flag, int tdc) {
    // tdc: the per-token decays are relative to groups of tdc chunks (1: to this kernel's
    // chunks; 2 with S == 1: to chunks twice as long, for a solve at that size)
    constexpr int BOXR = C < 64 ? C : 64;   // rows per TMA box of k and v
    using L = StateSmem<C>;
    constexpr int D = 128, NP = L::NP, PER = C / 32;
    constexpr uint32_t TILE = L::TILE;
    // the solve launched after this kernel may start its state-independent set-up on
    // the SMs this grid leaves free (it waits for this grid before reading its output)
    griddep_launch_dependents();
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = smem_align1024(smraw);
    const uint32_t sb = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BARS);
    uint64_t *bar_load = bars, *bar_mma = bars + 2, *bar_fin = bars + 4, *bar_w = bars + 5,
             *bar_out = bars + 7;
    uint32_t *tbase = reinterpret_cast<uint32_t *>(sm + L::TBASE);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool arith = warp < 16;
    const int quarter = warp & 3, cg = (warp >> 2) & 3;   // lane quarter, 32-column group
    const int d = quarter * 32 + lane;          // state row of this thread = its TMEM lane
    const int m = blockIdx.x, bh = blockIdx.y / S, seg = blockIdx.y % S;  // m = 0: H, 1: M
    const bool is_m = m == 1;
    // this CTA's chunks: n0 .. n0 + NL - 1 (the whole sequence when S == 1)
    const int n0 = (int)(((long long)seg * N) / S);
    const int NL = (int)(((long long)(seg + 1) * N) / S) - n0;
    const size_t tokbase = (size_t)bh * T + (size_t)n0 * C;
    float *s_beta = reinterpret_cast<float *>(sm + L::BETA);   // [2][C]
    float *s_gate = reinterpret_cast<float *>(sm + L::GATE);   // [2][C], with a gate
    float *s_w = reinterpret_cast<float *>(sm + L::W);         // [2][C]
    float *s_bn = reinterpret_cast<float *>(sm + L::BN);       // [2]
    float *s_red = reinterpret_cast<float *>(sm + L::RED);     // [2][16]
    // parts buffer of chunk c
    auto parts = [&](int c) -> uint32_t { return L::PARTS + (c & (L::NPB - 1)) * NP * TILE; };
    // staging of chunk n's fp16 state copy
    auto out_stage = [&](int n) -> uint32_t {
        return C <= 64 ? L::OUT : (is_m ? L::KS + ((n + 1) & 1) * TILE : L::VS);
    };

    if (tid == kStateEpiThreads) {
        for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
        mbar_init(&bar_w[0], 32);
        mbar_init(&bar_w[1], 32);
        mbar_init(bar_out, kStateEpiThreads);
        fence_mbar_init();
    }
    __syncthreads();

    int last_load[2] = {-1, -1};   // issuer: chunk last loaded into each stage
    // issuer: chunk c (keys, values for M, beta, gates) into stage c & 1
    auto issue_load = [&](int c) {
        const int st = c & 1;
        uint64_t *bar = &bar_load[st];
        mbar_arrive_expect_tx(bar, TILE * (is_m ? 2u : 1u) + (gate ? 8u : 4u) * C);
        const int row0 = (int)(tokbase + (size_t)c * C);
        for (int h = 0; h < 2; ++h)
            for (int rb = 0; rb < C / BOXR; ++rb) {
                const uint32_t o = st * TILE + h * C * 128 + rb * BOXR * 128;
                tc::tma_load_2d(sm + L::KS + o, &maps.k, h * 64, row0 + rb * BOXR, bar);
                if (is_m) tc::tma_load_2d(sm + L::VS + o, &maps.v, h * 64, row0 + rb * BOXR, bar);
            }
        bulk_g2s(s_beta + st * C, beta + tokbase + (size_t)c * C, 4 * C, bar);
        if (gate) bulk_g2s(s_gate + st * C, gate + tokbase + (size_t)c * C, 4 * C, bar);
        last_load[st] = c;
    };
    // issuer: dS_c = A^T (w K) into TMEM buffer c & 1 (A = K or V of stage c & 1)
    auto issue_mma = [&](uint32_t tmem, int c) {
        constexpr uint32_t ID = tc::idesc_bf16(128, 128, true, true);
        const uint32_t a = sb + (is_m ? L::VS : L::KS) + (c & 1) * TILE;
#pragma unroll
        for (int p = 0; p < NP; ++p)
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                tc::mma_f16(tmem + (c & 1) * 128, tc::sdesc(a + kk * 2048, C * 128, 1024),
                            tc::sdesc(sb + parts(c) + p * TILE + kk * 2048, C * 128, 1024), ID,
                            (p | kk) != 0);
        tc::commit(&bar_mma[c & 1]);
    };
    if (tid == kStateEpiThreads) {
        issue_load(0);
        if (NL > 1) issue_load(1);
    }
    if (warp == 0) {
        tc::tmem_alloc(tbase, 256);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tbase;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(cg * 32);

    // Decay warp: chunk c's weights w_t = g_t prod_{m>t} beta_m (suffix products;
    // lane l holds tokens l*PER..) into s_w[c & 1], b_c into s_bn[c & 1], then
    // every lane arrives on bar_w[c & 1].
    auto decays = [&](int c) {
        const float *bt = s_beta + (c & 1) * C;
        float bv[PER], sfx[PER];
        float run = 1.f;
#pragma unroll
        for (int p = 0; p < PER; ++p) bv[p] = bt[lane * PER + p];
#pragma unroll
        for (int p = PER - 1; p >= 0; --p) {
            sfx[p] = run;          // product over this lane's tokens after p
            run *= bv[p];
        }
        float tot = run;           // -> product over the tokens of lanes >= this lane
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_down_sync(0xffffffffu, tot, o);
            if (lane + o < 32) tot *= y;
        }
        float above = __shfl_down_sync(0xffffffffu, tot, 1);   // lanes > this lane
        if (lane == 31) above = 1.f;
#pragma unroll
        for (int p = 0; p < PER; ++p) {
            float w = sfx[p] * above;
            if (gate) w *= s_gate[(c & 1) * C + lane * PER + p];
            s_w[(c & 1) * C + lane * PER + p] = w;
        }
        if (lane == 0) s_bn[c & 1] = tot;
        __syncwarp();
        mbar_arrive(&bar_w[c & 1]);
    };

    // Decay warp of the H CTA: chunk c's per-token decays for the solve
    // (l_t log2 e, exp(l_t), beta_t, beta_t^2; l from fp32 logs summed in
    // double, relative to the start of the chunk's group of tdc chunks) and the
    // chunk decay.
    double goff = 0.0;   // summed log of the group's earlier chunks
    auto token_decays = [&](int c) {
        const float *bt = s_beta + (c & 1) * C;
        double x[PER];
        double acc = 0.0;
#pragma unroll
        for (int p = 0; p < PER; ++p) {
            acc += fmax((double)logf(bt[lane * PER + p]), kLogBetaMin);
            x[p] = acc;
        }
        double t2 = acc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double y = __shfl_up_sync(0xffffffffu, t2, o);
            if (lane >= o) t2 += y;
        }
        const double excl = t2 - acc + goff;
        double prev = __shfl_up_sync(0xffffffffu, t2, 1) + goff;
        if (lane == 0) prev = goff;
#pragma unroll
        for (int p = 0; p < PER; ++p) {
            const double l = x[p] + excl;
            const size_t g = tokbase + (size_t)c * C + lane * PER + p;
            const float b1 = decay_exp(l - prev);
            if (tokdec) {
                tokdec[g] = (float)(l * 1.4426950408889634);
                tokdec[plane + g] = decay_exp(l);
                tokdec[2 * plane + g] = b1;
                tokdec[3 * plane + g] = b1 * b1;
            }
            prev = l;
        }
        const double lend = __shfl_sync(0xffffffffu, t2, 31);
        if (lane == 0) decay[(size_t)bh * N + n0 + c] = decay_exp(lend);
        goff = (n0 + c + 1) % tdc == 0 ? 0.0 : goff + lend;
        __syncwarp();
    };

    // Arithmetic warps: B operand of chunk c, the bf16 parts of w_i k_i, in the
    // swizzled layout of the key tile (the 16-byte chunk at a byte offset holds
    // the same elements in every tile), and this warp's share of the bound
    // increment into s_red[c & 1][warp].
    auto prep = [&](int c) {
        const uint8_t *kt = sm + L::KS + (c & 1) * TILE;
        const uint8_t *vt = sm + L::VS + (c & 1) * TILE;
        const float *wc = s_w + (c & 1) * C;
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < C * 16 / kStateEpiThreads; ++j) {
            const int item = tid + j * kStateEpiThreads;   // C rows x 16 chunks of 16 bytes
            const int r = item >> 4, l16 = item & 15;
            const uint32_t off = (uint32_t)((l16 >> 3) * (C * 128) + r * 128 + (l16 & 7) * 16);
            const uint4 u = *reinterpret_cast<const uint4 *>(kt + off);
            const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
            const float w = wc[r];
            float sq = 0.f;
            uint32_t p0[4], p1[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float x0 = bf16_lo(uw[q]), x1 = bf16_hi(uw[q]);
                sq = fmaf(x0, x0, fmaf(x1, x1, sq));
                const float y0 = w * x0, y1 = w * x1;
                p0[q] = bf16x2_bits(y0, y1);
                const float r0 = y0 - bf16_lo(p0[q]), r1 = y1 - bf16_hi(p0[q]);
                p1[q] = bf16x2_bits(r0, r1);
            }
            uint8_t *pb = sm + parts(c);
            *reinterpret_cast<uint4 *>(pb + off) = make_uint4(p0[0], p0[1], p0[2], p0[3]);
            *reinterpret_cast<uint4 *>(pb + TILE + off) = make_uint4(p1[0], p1[1], p1[2], p1[3]);
            if (is_m) {
                const uint4 uv = *reinterpret_cast<const uint4 *>(vt + off);
                const uint32_t vw[4] = {uv.x, uv.y, uv.z, uv.w};
                float sv = 0.f;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float x0 = bf16_lo(vw[q]), x1 = bf16_hi(vw[q]);
                    sv = fmaf(x0, x0, fmaf(x1, x1, sv));
                }
                acc = fmaf(0.5f * w, sq + sv, acc);
            } else {
                acc = fmaf(w, sq, acc);
            }
        }
        acc = warp_sum(acc);
        if (lane == 0) s_red[(c & 1) * 16 + warp] = acc;
    };
    auto bound_inc = [&](int c) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < 16; ++w) s += s_red[(c & 1) * 16 + w];
        return s;
    };

    // ---- prologue: chunk 0's operands and product ----
    const bool issuer_warp = warp == 16, decay_warp = warp == 17;
    constexpr bool kDblParts = L::NPB == 2;
    bool ok = true;
    float b_next = 1.f;   // arithmetic warps: decay of the next chunk to fold in
    if (arith) {
        ok = mbar_wait_bounded(&bar_w[0], 0, kStateWaitProbes);
        ok = mbar_wait_bounded(&bar_load[0], 0, kStateWaitProbes) && ok;
        b_next = s_bn[0];
        prep(0);
        fence_proxy_async_smem();
    } else if (decay_warp) {
        ok = mbar_wait_bounded(&bar_load[0], 0, kStateWaitProbes);
        decays(0);
        if (!is_m) token_decays(0);
    }
    ok = __syncthreads_and(ok);
    if (tid == kStateEpiThreads && ok) issue_mma(tmem, 0);

    float st[32];
    float bound = 0.f;
    const size_t DD = (size_t)D * D;
    if (S > 1 && arith) {
        // the segment's start state and norm bound (zero for the first segment)
        const size_t e0 = (size_t)bh * S * K + (size_t)seg * K;   // this segment's start entry
        const float *src = seg_start + (e0 * 2 + m) * DD + (size_t)d * D + cg * 32;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 x = *reinterpret_cast<const float4 *>(src + 4 * j);
            st[4 * j] = x.x; st[4 * j + 1] = x.y; st[4 * j + 2] = x.z; st[4 * j + 3] = x.w;
        }
        bound = seg_bound[e0 * 2 + m];
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) st[i] = 0.f;
    }

    // Decay warp: chunk c's decays as soon as it has landed.  Stage c & 1 is
    // reloaded only after the product of chunk c - 2 is done, which comes after
    // every read of the w and b_n buffers this overwrites.
    if (decay_warp) {
#pragma unroll 1
        for (int c = 1; c < NL && ok; ++c) {
            if (!mbar_wait_bounded(&bar_load[c & 1], (c >> 1) & 1, kStateWaitProbes)) ok = false;
            decays(c);
            if (!is_m) token_decays(c);
        }
    }

    // Arithmetic and issuing warps.  `ok` changes only at barriers, so they
    // leave the loop together; a wait that gives up sets `fail`, which the next
    // barrier folds into `ok`.
    bool fail = false;
#pragma unroll 1
    for (int n = 0; n < NL && ok && !decay_warp; ++n) {
        const int ph = (n >> 1) & 1, ph1 = ((n + 1) >> 1) & 1;
        if (issuer_warp) {
            // stage n & 1 is free once dS_n is done and the previous TMA store has
            // read its staging; chunk n + 1's product once its operands are ready;
            // chunk n's fp16 copy once it is staged
            if (lane == 0) {
                if (!mbar_wait_bounded(&bar_mma[n & 1], ph, kStateWaitProbes)) fail = true;
                tc::bulk_wait_read0();
                if (n + 2 < NL) issue_load(n + 2);
            }
            __syncwarp();
            ok = named_barrier_and(2, kStateBarThreads, ok && !fail);
            if (!ok) break;
            if (lane == 0) {
                tc::fence_after_sync();
                if (n + 1 < NL) issue_mma(tmem, n + 1);
                if (!mbar_wait_bounded(bar_out, n & 1, kStateWaitProbes)) fail = true;
                if (!fail) {
                    const int row = (int)(((size_t)bh * N + n0 + n) * 2 + m) * D;
                    tc::tma_store_2d(&maps.out, 0, row, sm + out_stage(n));
                    tc::tma_store_2d(&maps.out, 64, row, sm + out_stage(n) + 16384);
                    tc::bulk_commit();
                }
            }
            __syncwarp();
            continue;
        }
        const float bn = b_next, bincn = bound_inc(n);   // chunk n's decay and bound increment
        if (n + 1 < NL) {
            // chunk n + 1's operands (with double-buffered parts, formed while
            // chunk n's product still runs)
            if (!mbar_wait_bounded(&bar_w[(n + 1) & 1], ph1, kStateWaitProbes)) fail = true;
            if (!mbar_wait_bounded(&bar_load[(n + 1) & 1], ph1, kStateWaitProbes)) fail = true;
            b_next = s_bn[(n + 1) & 1];
            if (kDblParts) {
                prep(n + 1);
                fence_proxy_async_smem();
            }
        }
        // dS_n is ready (and, with single-buffered parts, the parts are free)
        if (!mbar_wait_bounded(&bar_mma[n & 1], ph, kStateWaitProbes)) fail = true;
        tc::fence_after_sync();
        if (!kDblParts && n + 1 < NL) {
            prep(n + 1);
            fence_proxy_async_smem();
        }
        tc::fence_before_sync();
        ok = named_barrier_and(2, kStateBarThreads, ok && !fail);
        if (!ok) break;
        {
            // fp16 copy of the chunk-start state S_n, scaled by 2^e_n, staged in the TMA
            // box layout: [column half][row][64], 16-byte chunk j of row d at j ^ (d % 8)
            const int ex = lp_exponent_tc(bound);
            const float sc = ldexpf(1.f, ex);
            uint8_t *row = sm + out_stage(n) + (cg >> 1) * 16384 + d * 128;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int chunk = ((cg & 1) * 4 + j) ^ (d & 7);
                *reinterpret_cast<uint4 *>(row + chunk * 16) = make_uint4(
                    pack_h2(st[8 * j] * sc, st[8 * j + 1] * sc),
                    pack_h2(st[8 * j + 2] * sc, st[8 * j + 3] * sc),
                    pack_h2(st[8 * j + 4] * sc, st[8 * j + 5] * sc),
                    pack_h2(st[8 * j + 6] * sc, st[8 * j + 7] * sc));
            }
            fence_proxy_async_smem();
            mbar_arrive(bar_out);
            if (tid == 0) state_exp[((size_t)bh * N + n0 + n) * 2 + m] = ex;
        }
        // S_{n+1} = b_n S_n + dS_n
        {
            float dl[32];
#pragma unroll
            for (int cb = 0; cb < 32; cb += 16) tc::tmem_ld16(tl + (n & 1) * 128 + cb, dl + cb);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) st[i] = fmaf(bn, st[i], dl[i]);
        }
        bound = fmaf(bn, bound, bincn);
    }

    ok = ok && !fail;
    if (arith && ok && final_state && seg == S - 1) {
        float *dst = final_state + ((size_t)bh * 2 + m) * DD + (size_t)d * D + cg * 32;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            *reinterpret_cast<float4 *>(dst + 4 * j) =
                make_float4(st[4 * j], st[4 * j + 1], st[4 * j + 2], st[4 * j + 3]);
    }

    // teardown: no MMA or copy of this CTA may be in flight when TMEM or shared
    // memory is released
    tc::fence_before_sync();
    ok = __syncthreads_and(ok);
    if (tid == kStateEpiThreads) {
        tc::bulk_wait0();
        if (!ok) {
            atomicExch(timeout_flag, 1);
            tc::commit(bar_fin);
            mbar_wait_bounded(bar_fin, 0, kStateWaitProbes);
            for (int s2 = 0; s2 < 2; ++s2)
                if (last_load[s2] >= 0)
                    mbar_wait_bounded(&bar_load[s2], (last_load[s2] >> 1) & 1, kStateWaitProbes);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 256);
    }
}

}  // namespace gka
