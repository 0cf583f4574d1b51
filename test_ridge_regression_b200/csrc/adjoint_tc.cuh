// Tensor-core adjoint-state pass of the backward (bf16 inputs, D = 128, chunks of
// 32 tokens): the adjoint increments of every chunk and their reverse scan in one
// sequential pass per (head, matrix).
//
// Method: "Gated KalmaNet" (arXiv 2511.21016), ai.info page, Key Contributions 3 and
// Methodology (implicit differentiation of the chunk-wise solve, reusing the chunked
// state recursion in reverse).  With G^H_t = -y_t x_t^T - c_t H_t, G^M_t = g_t x_t^T
// the per-token gradients of the loss with respect to the states, the adjoint E_n
// that reaches chunk n's last token from later chunks obeys
//   E_{N-1} = 0,   E_{n-1} = b_n E_n + dE_n,
//   dE^H_n = -(b o Y)^T X - (e o K~)^T K~ - c1 H_s,   dE^M_n = (b o G)^T X,
// b_s the chunk-relative decays, K~ the written keys sqrt(w_s) k_s, e_i =
// sum_{s>=i} b_s c_s w_si, c1 = sum_s b_s^2 c_s and H_s the chunk-start state.
//
// One CTA per (head, matrix), blockIdx.x = 0 for E^H, 1 for E^M, over the chunks from
// last to first.  The fp32 adjoint lives in registers (arithmetic thread (cg, d) owns
// row d, columns 32cg..32cg+31), so neither the increments nor the adjoints go through
// memory in fp32.  Warps 0-15 do the arithmetic, warp 16 issues the TMA loads, the MMAs
// and the TMA stores, warp 17 forms each chunk's decay weights when its rows land.
// Per chunk:
//   - the y, x (fp32) and k (bf16) rows, or the g and x rows, arrive by TMA two chunks
//     ahead with beta, c and the write gate; the chunk-start state copy (fp16, scaled
//     by 2^e, from the recompute's state pass) two chunks ahead as well;
//   - the arithmetic warps convert the rows, weighted, into fp16 operand tiles with
//     power-of-two scales from the tile maxima (the two products of dE^H with one
//     common scale, so that they share an accumulator); the issuing warp then runs
//     dE_n = A^T B as 128 x 128 x 32 MMAs into TMEM;
//   - while that runs, E_n leaves as an fp16 copy scaled by 2^e (e from the exact
//     maximum of |E_n|, so the largest entry lies in [1/2, 1)), staged over the state
//     copy it is read against: <E_n, S_n> (S_n = H_s or M_s, for dbeta) is formed from
//     the fp32 E_n first, and E becomes b_n E_n - c1 H_s (H) or b_n E_n (M);
//   - then E += dE_n from TMEM.
// Outputs: the copies [B*H][N][2][128][128] fp16 (2^e E_n), their exponents
// [B*H][N][2] and the inner products [B*H][N][2].
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "solve_tc.cuh"
#include "state_tc.cuh"
#include "tcgen05.cuh"

namespace gka {

constexpr int kAdjC = 32;                               // tokens per chunk
constexpr int kAdjEpiThreads = 512;                     // arithmetic warps 0-15
constexpr int kAdjBarThreads = kAdjEpiThreads + 32;     // + the issuing warp 16
constexpr int kAdjThreads = kAdjBarThreads + 32;        // + the weights warp 17

struct AdjMaps {
    CUtensorMap y, x;    // fp32 rows [B*H*T][128], box 32 x 32, 128B swizzle
    CUtensorMap k, g;    // bf16 rows [B*H*T][128], box 64 x 32
    CUtensorMap state;   // fp16 chunk-start state copies [B*H*N*2*128][128], box 64 x 64
    CUtensorMap out;     // fp16 adjoint copies, same shape, box 64 x 128
};

struct AdjSmem {
    // row stages: [Y 32 x 128 fp32 | X 32 x 128 fp32 | K (or G) 32 x 128 bf16]
    static constexpr uint32_t RY = 0, RX = 16384, RK = 32768;
    static constexpr uint32_t STAGE = 40960;
    static constexpr uint32_t ROWS = 0;                     // 2 stages
    static constexpr uint32_t SBUF = ROWS + 2 * STAGE;      // 2 x [2][128][64] fp16 state copies
    static constexpr uint32_t OPS = SBUF + 2 * 32768;       // operand tiles [2][32][64] fp16
    static constexpr uint32_t TY = OPS, TX = OPS + 8192, TE = OPS + 16384, TK = OPS + 24576;
    static constexpr uint32_t SCAL = OPS + 32768;           // [2][beta 32 | c 32 | gate 32]
    static constexpr uint32_t WTS = SCAL + 2 * 384;         // [2][b 32 | ek 32 | sg 32 | bn, c1]
    static constexpr uint32_t WSTR = 448;                   // bytes per stage of WTS
    static constexpr uint32_t RED = WTS + 2 * WSTR;         // mx[16][4], emx[16], eh[16]
    static constexpr uint32_t BARS = RED + 384;             // rows[2] S[2] w[2] mma out fin
    static constexpr uint32_t TBASE = BARS + 9 * 8;
    static constexpr uint32_t END = TBASE + 16;
    static constexpr size_t bytes = END + 1024;             // + alignment slack
};

// Largest of a non-negative float over the warp: the bit patterns of non-negative
// floats order like unsigned integers, so one integer reduction does it.
__device__ __forceinline__ float warp_max_nonneg(float x) {
    return __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(x)));
}

// Exponent e of the power of two inv_pow2_above returns (x * 2^e lies in [1/2, 1)).
__device__ __forceinline__ int inv_pow2_exponent(float x) {
    return ((__float_as_int(inv_pow2_above(x)) >> 23) & 0xff) - 127;
}

// grid (2, B*H), block kAdjThreads.  T = N * 32.  ys, xs: the solves' fp32 rows (read
// through the maps); cvec: c_t; state_exp: the state copies' exponents [B*H][N][2];
// adj_exp, eh_part: outputs [B*H][N][2].
__global__ void __launch_bounds__(kAdjThreads, 1)
k_adjoint_pass_tc(const __grid_constant__ AdjMaps maps, const float *__restrict__ beta,
                  const float *__restrict__ gate, const float *__restrict__ cvec,
                  const int *__restrict__ state_exp, int *__restrict__ adj_exp,
                  float *__restrict__ eh_part, int T, int N, int *__restrict__ timeout_flag) {
    using L = AdjSmem;
    constexpr int D = 128, C = kAdjC;
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = smem_align1024(smraw);
    const uint32_t sb = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BARS);
    uint64_t *bar_rows = bars, *bar_s = bars + 2, *bar_w = bars + 4, *bar_mma = bars + 6,
             *bar_out = bars + 7, *bar_fin = bars + 8;
    uint32_t *tbase = reinterpret_cast<uint32_t *>(sm + L::TBASE);
    float *s_mx = reinterpret_cast<float *>(sm + L::RED);   // [16][4] tile maxima per warp
    float *s_emx = s_mx + 64;                               // [16] max |E| per warp
    float *s_eh = s_emx + 16;                               // [16] <E, S> per warp
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool arith = warp < 16, issuer_warp = warp == 16, weights_warp = warp == 17;
    const int quarter = warp & 3, cg = (warp >> 2) & 3;
    const int d = quarter * 32 + lane;                      // adjoint row = TMEM lane
    const int m = blockIdx.x, bh = blockIdx.y;              // m = 0: E^H, 1: E^M
    const bool is_m = m == 1;
    auto scal = [&](int st) { return reinterpret_cast<float *>(sm + L::SCAL + st * 384); };
    auto wts = [&](int st) { return reinterpret_cast<float *>(sm + L::WTS + st * L::WSTR); };
    // chunk of iteration i (last chunk first)
    auto chunk_of = [&](int i) { return N - 1 - i; };
    auto copy_row = [&](int n) { return (int)(((size_t)bh * N + n) * 2 + m) * D; };

    if (tid == kAdjEpiThreads) {
        for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
        mbar_init(&bar_w[0], 32);
        mbar_init(&bar_w[1], 32);
        mbar_init(bar_mma, 1);
        mbar_init(bar_out, kAdjEpiThreads);
        mbar_init(bar_fin, 1);
        fence_mbar_init();
    }
    if (tid < 16) s_emx[tid] = 0.f;   // E_{N-1} = 0
    __syncthreads();

    // issuer: chunk rows (y, x, k or g, x) and scalars of iteration i into stage i & 1
    int last_rows[2] = {-1, -1}, last_s[2] = {-1, -1};
    auto load_rows = [&](int i) {
        const int st = i & 1, n = chunk_of(i);
        uint64_t *bar = &bar_rows[st];
        const uint32_t bytes = is_m ? (16384u + 8192u + 128u)
                                    : (2 * 16384u + 8192u + 256u + (gate ? 128u : 0u));
        mbar_arrive_expect_tx(bar, bytes);
        const int row0 = (int)((size_t)bh * T + (size_t)n * C);
        uint8_t *base = sm + L::ROWS + st * L::STAGE;
        for (int q = 0; q < 4; ++q) {
            tc::tma_load_2d(base + L::RX + q * 4096, &maps.x, q * 32, row0, bar);
            if (!is_m) tc::tma_load_2d(base + L::RY + q * 4096, &maps.y, q * 32, row0, bar);
        }
        for (int h = 0; h < 2; ++h)
            tc::tma_load_2d(base + L::RK + h * 4096, is_m ? &maps.g : &maps.k, h * 64, row0, bar);
        float *sc = scal(st);
        const size_t t0 = (size_t)bh * T + (size_t)n * C;
        bulk_g2s(sc, beta + t0, 4 * C, bar);
        if (!is_m) {
            bulk_g2s(sc + 32, cvec + t0, 4 * C, bar);
            if (gate) bulk_g2s(sc + 64, gate + t0, 4 * C, bar);
        }
        last_rows[st] = i;
    };
    // issuer: the chunk-start state copy of iteration i into state buffer i & 1
    auto load_state = [&](int i) {
        const int st = i & 1;
        mbar_arrive_expect_tx(&bar_s[st], 32768);
        uint8_t *tile = sm + L::SBUF + st * 32768;
        const int row0 = copy_row(chunk_of(i));
        for (int h = 0; h < 2; ++h)
            for (int rb = 0; rb < 2; ++rb)
                tc::tma_load_2d(tile + h * 16384 + rb * 8192, &maps.state, h * 64, row0 + rb * 64,
                                &bar_s[st]);
        last_s[st] = i;
    };
    if (tid == kAdjEpiThreads) {
        load_rows(0);
        load_state(0);
        if (N > 1) {
            load_rows(1);
            load_state(1);
        }
    }
    if (warp == 0) {
        tc::tmem_alloc(tbase, 128);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tbase;

    bool ok = true;
    if (weights_warp) {
        // chunk weights as each stage lands: lane t = token t.  l_t: inclusive prefix of
        // the clamped log(beta) in double; b_t = exp(l_t); e by a suffix scan of the
        // linear recurrence e_t = b_t c_t + w_{t+1,t} e_{t+1}.
#pragma unroll 1
        for (int i = 0; i < N && ok; ++i) {
            const int st = i & 1;
            if (!mbar_wait_bounded(&bar_rows[st], (i >> 1) & 1, kStateWaitProbes)) {
                ok = false;
                break;
            }
            const float *sc = scal(st);
            float *w = wts(st);
            double l = fmax(log((double)sc[lane]), kLogBetaMin);
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double y = __shfl_up_sync(0xffffffffu, l, o);
                if (lane >= o) l += y;
            }
            const float b = decay_exp(l);
            w[lane] = b;
            const double lend = __shfl_sync(0xffffffffu, l, 31);
            if (!is_m) {
                const double lnext = __shfl_down_sync(0xffffffffu, l, 1);
                float A = lane < 31 ? decay_exp(lnext - l) : 0.f;
                const float ct = sc[32 + lane];
                float B = b * ct;
                const float c1 = warp_sum(b * B);
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float A2 = __shfl_down_sync(0xffffffffu, A, o);
                    const float B2 = __shfl_down_sync(0xffffffffu, B, o);
                    if (lane + o < 32) {
                        B = fmaf(A, B2, B);
                        A *= A2;
                    }
                }
                const float sg = gate ? sqrtf(sc[64 + lane]) : 1.f;
                w[32 + lane] = B * sg;   // e_t sqrt(w_t)
                w[64 + lane] = sg;
                if (lane == 0) w[97] = c1;
            }
            if (lane == 0) w[96] = decay_exp(lend);
            __syncwarp();
            mbar_arrive(&bar_w[st]);
        }
    }

    // arithmetic warps: item (token t, columns 8j..8j+7) of the conversions
    const int ct = tid >> 4, cj = tid & 15;
    float E[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) E[i] = 0.f;
    bool fail = false;
#pragma unroll 1
    for (int i = 0; i < N && ok && !weights_warp; ++i) {
        const int st = i & 1, ph = (i >> 1) & 1, n = chunk_of(i);
        if (issuer_warp) {
            ok = named_barrier_and(2, kAdjBarThreads, ok && !fail);
            if (!ok) break;
            if (lane == 0) {
                tc::fence_after_sync();
                constexpr uint32_t ID = tc::idesc_f16(128, 128, true, true);
                auto desc = [&](uint32_t t, int kk) { return tc::sdesc(t + kk * 2048, C * 128, 1024); };
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk) {
                    tc::mma_f16(tmem, desc(sb + L::TY, kk), desc(sb + L::TX, kk), ID, kk > 0);
                    if (!is_m) tc::mma_f16(tmem, desc(sb + L::TE, kk), desc(sb + L::TK, kk), ID, true);
                }
                tc::commit(bar_mma);
                // the rows of stage st were converted before the barrier
                if (i + 2 < N) load_rows(i + 2);
                // E_n's copy, staged over its state copy, then that buffer's next load
                if (!mbar_wait_bounded(bar_out, i & 1, kStateWaitProbes)) fail = true;
                if (!fail) {
                    const uint8_t *tile = sm + L::SBUF + st * 32768;
                    tc::tma_store_2d(&maps.out, 0, copy_row(n), tile);
                    tc::tma_store_2d(&maps.out, 64, copy_row(n), tile + 16384);
                    tc::bulk_commit();
                    tc::bulk_wait_read0();
                    if (i + 2 < N) load_state(i + 2);
                }
            }
            __syncwarp();
            continue;
        }
        // ---- arithmetic warps ----
        if (!mbar_wait_bounded(&bar_w[st], ph, kStateWaitProbes)) fail = true;
        if (!mbar_wait_bounded(&bar_rows[st], ph, kStateWaitProbes)) fail = true;
        const float *w = wts(st);
        const float bn = w[96], c1 = is_m ? 0.f : w[97];
        const int eS = state_exp[((size_t)bh * N + n) * 2 + m];
        // pass 1: this item's rows and the tile maxima
        const uint8_t *rs = sm + L::ROWS + st * L::STAGE;
        float xv[8], yv[8], kv[8];
        {
            const int sw = ct & 7;
            const uint8_t *xr = rs + L::RX + (cj >> 2) * 4096 + ct * 128;
            const float4 x0 = *reinterpret_cast<const float4 *>(xr + ((2 * (cj & 3)) ^ sw) * 16);
            const float4 x1 = *reinterpret_cast<const float4 *>(xr + ((2 * (cj & 3) + 1) ^ sw) * 16);
            xv[0] = x0.x; xv[1] = x0.y; xv[2] = x0.z; xv[3] = x0.w;
            xv[4] = x1.x; xv[5] = x1.y; xv[6] = x1.z; xv[7] = x1.w;
            if (!is_m) {
                const uint8_t *yr = rs + L::RY + (cj >> 2) * 4096 + ct * 128;
                const float4 y0 = *reinterpret_cast<const float4 *>(yr + ((2 * (cj & 3)) ^ sw) * 16);
                const float4 y1 = *reinterpret_cast<const float4 *>(yr + ((2 * (cj & 3) + 1) ^ sw) * 16);
                yv[0] = y0.x; yv[1] = y0.y; yv[2] = y0.z; yv[3] = y0.w;
                yv[4] = y1.x; yv[5] = y1.y; yv[6] = y1.z; yv[7] = y1.w;
            }
            const uint4 u = *reinterpret_cast<const uint4 *>(rs + L::RK + (cj >> 3) * 4096 +
                                                             ct * 128 + ((cj & 7) ^ sw) * 16);
            const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                kv[2 * q] = bf16_lo(uw[q]);
                kv[2 * q + 1] = bf16_hi(uw[q]);
            }
        }
        // H: mX, mY (b y), mK (sg k), mE (ek k);  M: mX, mG (b g) in the mY slot
        const float bt = w[ct], ekt = is_m ? 0.f : w[32 + ct], sgt = is_m ? 0.f : w[64 + ct];
        float mx4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            mx4[0] = fmaxf(mx4[0], fabsf(xv[e]));
            if (is_m) {
                mx4[1] = fmaxf(mx4[1], fabsf(bt * kv[e]));
            } else {
                mx4[1] = fmaxf(mx4[1], fabsf(bt * yv[e]));
                mx4[2] = fmaxf(mx4[2], fabsf(sgt * kv[e]));
                mx4[3] = fmaxf(mx4[3], fabsf(ekt * kv[e]));
            }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) mx4[q] = warp_max_nonneg(mx4[q]);
        if (lane == 0)
            *reinterpret_cast<float4 *>(s_mx + warp * 4) = make_float4(mx4[0], mx4[1], mx4[2], mx4[3]);
        named_barrier_sync(1, kAdjEpiThreads);
        // the previous chunk's <E, S> (complete since this barrier)
        if (tid == 0 && i > 0) {
            float s = 0.f;
            for (int q = 0; q < 16; ++q) s += s_eh[q];
            eh_part[((size_t)bh * N + n + 1) * 2 + m] = s;
        }
        // the 16 warps' maxima: lane l reads warp l % 16's, one reduction each
        float MX, MY, MK, ME, EM;
        {
            const float4 v = *reinterpret_cast<const float4 *>(s_mx + (lane & 15) * 4);
            MX = warp_max_nonneg(v.x);
            MY = warp_max_nonneg(v.y);
            MK = warp_max_nonneg(v.z);
            ME = warp_max_nonneg(v.w);
            EM = warp_max_nonneg(s_emx[lane & 15]);
        }
        // pass 2: the fp16 operand tiles (single-buffered: the previous chunk's products
        // were waited for before its update)
        float unscale;
        {
            const float sX = inv_pow2_above(MX);
            const uint32_t off = (uint32_t)(cj >> 3) * 4096u + (uint32_t)ct * 128u +
                                 (uint32_t)(((cj & 7) ^ (ct & 7)) * 16);
            auto put = [&](uint32_t tile, const float *o8) {
                st_shared_v4(tile + off, pack_f16(o8[0], o8[1]), pack_f16(o8[2], o8[3]),
                             pack_f16(o8[4], o8[5]), pack_f16(o8[6], o8[7]));
            };
            float o8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) o8[e] = xv[e] * sX;
            put(sb + L::TX, o8);
            if (is_m) {
                const float sG = inv_pow2_above(MY);
                const float f = bt * sG;
#pragma unroll
                for (int e = 0; e < 8; ++e) o8[e] = kv[e] * f;
                put(sb + L::TY, o8);
                unscale = 1.f / (sG * sX);
            } else {
                // both products of dE^H carry the scale S = min(sY sX, sE sK)
                const float sK = inv_pow2_above(MK);
                const float S = fminf(inv_pow2_above(MY) * sX, inv_pow2_above(ME) * sK);
                const float sY = S / sX, sE = S / sK;
                float f = -bt * sY;
#pragma unroll
                for (int e = 0; e < 8; ++e) o8[e] = yv[e] * f;
                put(sb + L::TY, o8);
                f = sgt * sK;
#pragma unroll
                for (int e = 0; e < 8; ++e) o8[e] = kv[e] * f;
                put(sb + L::TK, o8);
                f = -ekt * sE;
#pragma unroll
                for (int e = 0; e < 8; ++e) o8[e] = kv[e] * f;
                put(sb + L::TE, o8);
                unscale = 1.f / S;
            }
        }
        fence_proxy_async_smem();
        tc::fence_before_sync();
        ok = named_barrier_and(2, kAdjBarThreads, ok && !fail);
        if (!ok) break;
        // E_n: <E_n, S_n>, its fp16 copy over S_n's, then E <- b_n E_n - c1 H_s
        const int eE = inv_pow2_exponent(EM);
        {
            if (!mbar_wait_bounded(&bar_s[st], ph, kStateWaitProbes)) fail = true;
            const float scE = pow2f(eE), c1s = c1 * pow2f(-eS);
            uint8_t *row = sm + L::SBUF + st * 32768 + (cg >> 1) * 16384 + d * 128;
            float dot = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint4 *p = reinterpret_cast<uint4 *>(row + ((((cg & 1) * 4 + j) ^ (d & 7)) * 16));
                const uint4 u = *p;
                const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
                float s8[8];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&uw[q]));
                    s8[2 * q] = f.x;
                    s8[2 * q + 1] = f.y;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) dot = fmaf(E[8 * j + e], s8[e], dot);
                *p = make_uint4(pack_f16(E[8 * j] * scE, E[8 * j + 1] * scE),
                                pack_f16(E[8 * j + 2] * scE, E[8 * j + 3] * scE),
                                pack_f16(E[8 * j + 4] * scE, E[8 * j + 5] * scE),
                                pack_f16(E[8 * j + 6] * scE, E[8 * j + 7] * scE));
#pragma unroll
                for (int e = 0; e < 8; ++e) E[8 * j + e] = fmaf(-c1s, s8[e], bn * E[8 * j + e]);
            }
            fence_proxy_async_smem();
            mbar_arrive(bar_out);
            dot = warp_sum(dot) * pow2f(-eS);
            if (lane == 0) s_eh[warp] = dot;
            if (tid == 0) adj_exp[((size_t)bh * N + n) * 2 + m] = eE;
        }
        // E += dE_n
        if (!mbar_wait_bounded(bar_mma, i & 1, kStateWaitProbes)) fail = true;
        tc::fence_after_sync();
        {
            const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(cg * 32);
            float dl[32];
            tc::tmem_ld16(tl, dl);
            tc::tmem_ld16(tl + 16, dl + 16);
            tc::tmem_wait_ld();
            float mx = 0.f;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                E[e] = fmaf(dl[e], unscale, E[e]);
                mx = fmaxf(mx, fabsf(E[e]));
            }
            mx = warp_max_nonneg(mx);
            if (lane == 0) s_emx[warp] = mx;
        }
        tc::fence_before_sync();
    }
    // the first chunk's <E, S>
    ok = ok && !fail;
    if (arith) {
        named_barrier_sync(1, kAdjEpiThreads);
        if (tid == 0 && ok) {
            float s = 0.f;
            for (int q = 0; q < 16; ++q) s += s_eh[q];
            eh_part[((size_t)bh * N + 0) * 2 + m] = s;
        }
    }

    // teardown: no MMA or copy of this CTA may be in flight when TMEM or shared memory
    // is released
    tc::fence_before_sync();
    ok = __syncthreads_and(ok);
    if (tid == kAdjEpiThreads) {
        tc::bulk_wait0();
        if (!ok) {
            atomicExch(timeout_flag, 1);
            tc::commit(bar_fin);
            mbar_wait_bounded(bar_fin, 0, kStateWaitProbes);
            for (int s2 = 0; s2 < 2; ++s2) {
                if (last_rows[s2] >= 0)
                    mbar_wait_bounded(&bar_rows[s2], (last_rows[s2] >> 1) & 1, kStateWaitProbes);
                if (last_s[s2] >= 0)
                    mbar_wait_bounded(&bar_s[s2], (last_s[s2] >> 1) & 1, kStateWaitProbes);
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 128);
    }
}

}  // namespace gka
