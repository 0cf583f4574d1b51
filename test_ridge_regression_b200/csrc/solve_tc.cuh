// Tensor-core (tcgen05 + TMEM + TMA) Chebyshev solve and readout of the
// chunk-wise GKA forward, bf16 inputs, head dimension 128.
//
// Method: "Gated KalmaNet" (arXiv 2511.21016), ai.info page, Key
// Contributions 2-3 and Methodology: the Chebyshev iteration needs only
// products with H_t, and inside a chunk H_t x = b_t H_s x + sum_{i<=t}
// w_{ti} (k_i . x) k_i, so every iteration of all tokens of a chunk is three
// small GEMMs against the chunk-start state and the chunk's keys.
//
// One CTA (8 warps) solves one chunk of TOK = MG = C tokens (64 or 128).  Work is
// kept transposed so that every accumulator has M = 128 rows, one TMEM lane per
// thread:
//   S^T = K X^T           (keys x tokens, K = 128)                    -> TMEM S
//   Z1  = H_s X^T         (M = 128, N = TOK, K = 128)                  -> TMEM Z1
//   P^T = W o S^T         (registers -> fp16 in shared memory, W_{ij} = w_{ji},
//                          with each token's factor c3_j folded in)
//   Z3  = K^T P^T         (M = 128, N = TOK, K = MG)                   -> TMEM Z3
//   the three-term Chebyshev update in fp32 registers (thread d owns element d of
//   its warpgroup's TOK/2 iterates); the new iterate goes back to shared memory as
//   fp16 (MN-major, 128B-swizzled), the B operand of the next round.
// The readout is the same three GEMMs with M_s in place of H_s and V in place of
// K for the final product: o_j = b_j M_s x_j + sum_i w_{ji} (k_i.x_j) v_i.  H_s, K,
// V and q arrive by TMA or bulk copies and stay in shared memory for all r rounds;
// M_s replaces H_s for the readout.
//
// Operand precision: every MMA operand is fp16 with a scale, fp32 accumulation.
// bf16 keys and values convert exactly (scaled by 2^-e so that |k|, |v| < 1); the
// chunk-start states come from the state kernels already in fp16, scaled by 2^e
// from a bound on their Frobenius norm; token j's iterate is kept as sigma x / invd_j
// with sigma a power of two per chunk from the bound ||x_i|| <= ||q|| (1+2a) / (a d)
// that every Chebyshev iterate satisfies, which makes the coefficient of q the same
// for every token.  All scales are undone in fp32.  fp16 keeps 3 more mantissa
// bits than bf16 at the same tensor-core rate; rounding the iterate to bf16 instead
// would cost about 1e-2 relative error at a = 0.1 (condition number 11).
#pragma once

#include <cuda_fp16.h>

#include <type_traits>

#include "common.cuh"
#include "ptx.cuh"
#include "tcgen05.cuh"

namespace gka {

constexpr int kTcThreads = 128;
constexpr int kSolveThreads = 256;   // solve kernel: two warpgroups
constexpr int kTcD = 128;         // head dimension of the tensor-core path
constexpr uint32_t kTcWaitProbes = 1u << 22;
// waits inside the solve suspend for up to kTcSleepNs per probe (a waiting warp
// then takes no issue slots); kTcSleepProbes probes bound a wait at about a second
constexpr uint32_t kTcSleepNs = 1000;
constexpr uint32_t kTcSleepProbes = 1u << 20;

template <int MG, int TOK>
struct TcSmem {
    // byte offsets from a 1024-aligned base
    static constexpr uint32_t HM = 0;                        // H_s, later M_s: 2 x [128][64] fp16
    static constexpr uint32_t VT = HM + 32768;               // values: 2 x [MG][64]
    static constexpr uint32_t KT = VT + MG * 256;            // keys:   2 x [MG][64]
    static constexpr uint32_t XT = KT + MG * 256;            // X^T: TOK/64 x [128][64], MN-major
    static constexpr uint32_t PT = XT + TOK * 256;           // P^T: TOK/64 x [MG][64], MN-major
    static constexpr uint32_t QS = PT + TOK * MG * 2;        // q: [TOK][128] bf16, then q^T
    static constexpr uint32_t SCAL = QS + TOK * 256;         // per-token scalars [3][TOK]
    static constexpr uint32_t RED = SCAL + 8 * 4 * TOK;      // float[16]
    static constexpr uint32_t NRM = RED + 64;                // u, E, X, Gjj [4][MG]
    static constexpr uint32_t NRM2 = NRM + 16 * MG;          // second warpgroup's E, X [2][MG]
    static constexpr uint32_t UPART = NRM2 + 8 * MG;         // [4 lane quarters][MG] partial u
    static constexpr uint32_t QPART = UPART + 16 * MG;       // [4 lane quarters][TOK] |q_j|^2
    static constexpr uint32_t DEC = QPART + 16 * TOK;        // l2, b, beta, beta^2: [4][MG] floats
    // [2 rounds][TOK] -w c1, then [2 rounds][TOK] -w / s_j of the rounds: over UPART
    // and QPART, set-up scratch that is dead once the rounds start
    static constexpr uint32_t COEF = UPART;
    static_assert(16 * TOK <= DEC - UPART, "coefficient tables overrun the set-up scratch");
    static constexpr uint32_t BARS = DEC + 16 * MG;
    static constexpr uint32_t TBASE = BARS + 8 * 8;
    static constexpr uint32_t END = TBASE + 16;
    static constexpr size_t bytes = END + 1024;              // + alignment slack
};
// two 64-token CTAs must fit one SM (228 KiB, of which 1 KiB per CTA is reserved)
static_assert(TcSmem<64, 64>::bytes <= 233472 / 2 - 1024, "64-token solve: two CTAs per SM");

struct TcMaps {
    CUtensorMap k;       // [B*H*T rows][128] bf16, box 64 x 64, 128B swizzle
    CUtensorMap v;       // same for v
    CUtensorMap state;   // [B*H*N*2*128 rows][128] fp16 scaled chunk-start states, box 64 x 64
};

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

__device__ __forceinline__ uint4 ld_shared_u4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    const __half2 p = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&p);
}

// 2^-(floor(log2 x) + 1) for x > 0 (so that x * result < 1), else 1; built from
// x's exponent field (x below the normal range counts as 2^-127, and the result is
// at least 2^-126).
__device__ __forceinline__ float inv_pow2_above(float x) {
    if (!(x > 0.f)) return 1.f;
    const int eb = (__float_as_int(x) >> 23) & 0xff;   // biased exponent of x
    const int rb = 253 - eb;                           // biased exponent of 2^(126 - eb)
    return __int_as_float((rb < 1 ? 1 : rb) << 23);
}

// 2^e exactly, from the exponent field: e in [-126, 127] (float), [-1022, 1023] (double).
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((e + 127) << 23); }
__device__ __forceinline__ double pow2d(int e) {
    return __longlong_as_double((long long)(e + 1023) << 52);
}

// 16 consecutive fp32 values from shared memory (16-byte aligned), as 4 vector loads.
__device__ __forceinline__ void ld_f32x16(const float *p, float *v) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 t = reinterpret_cast<const float4 *>(p)[i];
        v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
    }
}

// Tokens 16c..16c+15 of row `row` of the 128B-swizzled bf16 q^T tile, as fp32.
__device__ __forceinline__ void load_qrow16(uint32_t tile, uint32_t row, int c, float *v) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t ch = ((uint32_t)(2 * c + h) ^ row) & 7u;
        uint32_t a, b, cc, d;
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(a), "=r"(b), "=r"(cc), "=r"(d)
                     : "r"(tile + row * 128u + ch * 16u));
        const uint32_t w4[4] = {a, b, cc, d};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[8 * h + 2 * i] = __uint_as_float(w4[i] << 16);
            v[8 * h + 2 * i + 1] = __uint_as_float(w4[i] & 0xffff0000u);
        }
    }
}

// In place: bf16 tile of BYTES bytes -> fp16, scaled so that every |value| < 1.
// Returns the scale.  All NTHR threads of the block call it (red: NTHR/32 floats);
// each thread keeps the 16-byte pieces it reads for the max and converts them from
// registers.
template <int BYTES, int NTHR>
__device__ __forceinline__ float tile_bf16_to_f16_scaled(uint8_t *tile, float *red) {
    constexpr int PER = BYTES / (NTHR * 16);   // 16-byte pieces per thread
    static_assert(BYTES % (NTHR * 16) == 0, "tile size");
    const int tid = threadIdx.x, nw = NTHR >> 5;
    uint4 u[PER];
    float mx = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        u[i] = *reinterpret_cast<const uint4 *>(tile + (i * NTHR + tid) * 16);
        const uint32_t w4[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
            mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(w4[e] << 16)),
                                 fabsf(__uint_as_float(w4[e] & 0xffff0000u))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    __syncthreads();
    if ((tid & 31) == 0) red[tid >> 5] = mx;
    __syncthreads();
    mx = 0.f;
    for (int w = 0; w < nw; ++w) mx = fmaxf(mx, red[w]);
    const float sc = inv_pow2_above(mx);
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const uint32_t w4[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
        uint32_t o4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            o4[e] = pack_f16(__uint_as_float(w4[e] << 16) * sc,
                             __uint_as_float(w4[e] & 0xffff0000u) * sc);
        *reinterpret_cast<uint4 *>(tile + (i * NTHR + tid) * 16) =
            make_uint4(o4[0], o4[1], o4[2], o4[3]);
    }
    return sc;
}

// The same conversion for a tile of two 64-column halves of ROWS rows each
// (TMA box layout: the 16-byte piece at byte offset o belongs to row
// (o mod ROWS*128) / 128), with row r first multiplied by sqrt(g[r]) (g: the
// write gates of the tile's tokens; nullptr: the plain conversion above).
template <int BYTES, int NTHR, int ROWS>
__device__ __forceinline__ float tile_bf16_to_f16_rows_scaled(uint8_t *tile, float *red,
                                                              const float *__restrict__ g) {
    if (g == nullptr) return tile_bf16_to_f16_scaled<BYTES, NTHR>(tile, red);
    constexpr int PER = BYTES / (NTHR * 16);
    static_assert(BYTES % (NTHR * 16) == 0 && BYTES == 2 * ROWS * 128, "tile size");
    const int tid = threadIdx.x, nw = NTHR >> 5;
    float rs[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) rs[i] = sqrtf(__ldg(g + (((i * NTHR + tid) % (ROWS * 8)) >> 3)));
    uint4 u[PER];
    float mx = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        u[i] = *reinterpret_cast<const uint4 *>(tile + (i * NTHR + tid) * 16);
        const uint32_t w4[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
        float m = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e)
            m = fmaxf(m, fmaxf(fabsf(__uint_as_float(w4[e] << 16)),
                               fabsf(__uint_as_float(w4[e] & 0xffff0000u))));
        mx = fmaxf(mx, m * rs[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    __syncthreads();
    if ((tid & 31) == 0) red[tid >> 5] = mx;
    __syncthreads();
    mx = 0.f;
    for (int w = 0; w < nw; ++w) mx = fmaxf(mx, red[w]);
    const float sc = inv_pow2_above(mx);
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const uint32_t w4[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
        const float f = rs[i] * sc;
        uint32_t o4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            o4[e] = pack_f16(__uint_as_float(w4[e] << 16) * f,
                             __uint_as_float(w4[e] & 0xffff0000u) * f);
        *reinterpret_cast<uint4 *>(tile + (i * NTHR + tid) * 16) =
            make_uint4(o4[0], o4[1], o4[2], o4[3]);
    }
    return sc;
}

// Writes 8 consecutive values (columns c0..c0+7, c0 % 8 == 0) of `row` of a
// 128B-swizzled [rows][64] fp16 tile as one 16-byte chunk.
__device__ __forceinline__ void st_row8(uint32_t tile, uint32_t row, uint32_t c0, const float *v) {
    st_shared_v4(tile + row * 128u + (((c0 >> 3) ^ row) & 7u) * 16u, pack_f16(v[0], v[1]),
                 pack_f16(v[2], v[3]), pack_f16(v[4], v[5]), pack_f16(v[6], v[7]));
}

// Writes 16 consecutive values (columns c0..c0+15, c0 % 16 == 0) of `row` of a
// 128B-swizzled [rows][64] fp16 tile as two 16-byte chunks.
__device__ __forceinline__ void st_row16(uint32_t tile, uint32_t row, uint32_t c0, const float *v) {
    const uint32_t base = tile + row * 128u;
    const uint32_t ch0 = ((c0 >> 3) ^ row) & 7u, ch1 = ((c0 >> 3) + 1u ^ row) & 7u;
    st_shared_v4(base + ch0 * 16u, pack_f16(v[0], v[1]), pack_f16(v[2], v[3]),
                 pack_f16(v[4], v[5]), pack_f16(v[6], v[7]));
    st_shared_v4(base + ch1 * 16u, pack_f16(v[8], v[9]), pack_f16(v[10], v[11]),
                 pack_f16(v[12], v[13]), pack_f16(v[14], v[15]));
}

// Sums each of the N per-lane values v[0..N) over the 32 lanes of the warp by
// recursive halving (N - N/32 shuffles).  Afterwards lane l holds, in
// v[0..N/32), the totals of the original indices l*N/32 .. l*N/32 + N/32 - 1.
template <int N>
__device__ __forceinline__ void reduce_scatter32(float (&v)[N], int lane) {
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int o = 16 >> step, h = N >> (step + 1);
        const bool up = lane & o;
#pragma unroll
        for (int s = 0; s < h; ++s) {
            const float send = up ? v[s] : v[s + h];
            const float keep = up ? v[s + h] : v[s];
            v[s] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
}

// grid (N, B*H).  A CTA solves the TOK = MG tokens of one chunk (64, or 128 so that
// every MMA has N = 128).  8 warps: warpgroup wg (warps 4wg..4wg+3) owns tokens
// wg*TOK/2 .. (wg+1)*TOK/2 - 1; warp w reads TMEM lane quarter w % 4, so thread
// (wg, d) owns element d of the iterates of its TOK/2 tokens.
template <int MG, int TOK, bool XOUT = false>
__global__ void __launch_bounds__(kSolveThreads, TOK == 64 ? 2 : 1)
k_chunk_solve_tc(const __grid_constant__ TcMaps maps, const __nv_bfloat16 *__restrict__ q,
                 const float *__restrict__ gate, const float *__restrict__ tokdec, size_t plane, float *__restrict__ norms,
                 const int *__restrict__ state_exp, __nv_bfloat16 *__restrict__ o,
                 float *__restrict__ x_out, int T, int N, int C, const ChebParams P,
                 int *__restrict__ timeout_flag, int sstride) {
    // sstride: chunk stride of the state copies and exponents (1: one copy per chunk of
    // this kernel; 2: copies at half-size chunks, this chunk's start at every second)
    using L = TcSmem<MG, TOK>;
    constexpr int HALF = MG / 2;       // keys per warpgroup in the norm reductions
    constexpr int TPT = TOK / 2;       // tokens per thread
    constexpr int NCH = TPT / 16;      // 16-token chunks per thread
    constexpr uint32_t TMEM_COLS = 4 * TOK;
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = smem_align1024(smraw);
    const uint32_t sb = smem_u32(sm);
    float *s_c1 = reinterpret_cast<float *>(sm + L::SCAL);   // coefficient of Z1 (scaled domain)
    float *s_c3 = s_c1 + TOK;                                // c3_j
    float *s_o1 = s_c3 + TOK;                                // readout coefficient of Z1
    float *s_t3 = s_o1 + TOK;                                // 1 / s_j, undoes s_j on Z3
    float *s_mn = s_t3 + TOK;                                // per-warp minima of c3 (set-up)
    float *s_coef = reinterpret_cast<float *>(sm + L::COEF);   // -w c1 per token
    float *s_coef3 = s_coef + 2 * TOK;                         // -w / s_j per token
    float *red = reinterpret_cast<float *>(sm + L::RED);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BARS);
    uint64_t *bar_load = &bars[0], *bar_v = &bars[1], *bar_m = &bars[2], *bar_s = &bars[3],
             *bar_z = &bars[4], *bar_fin = &bars[5], *bar_n = &bars[6], *bar_z1 = &bars[7];
    uint32_t *tbase = reinterpret_cast<uint32_t *>(sm + L::TBASE);

    // the warp index read through a shuffle is known to be warp-uniform, so TMEM
    // addresses and warp-role branches derived from it stay in uniform registers
    const int tid = threadIdx.x, warp = __shfl_sync(0xffffffffu, tid >> 5, 0), lane = tid & 31;
    const int wg = warp >> 2, quarter = warp & 3;
    const int d = quarter * 32 + lane;        // head-dimension row = TMEM lane of this thread
    const int tcol = wg * TPT;                // first token (TMEM column) of this thread
    const int n = blockIdx.x, bh = blockIdx.y;
    const size_t tok0 = (size_t)bh * T + (size_t)n * C;    // first token of the chunk
    const size_t scopy = ((size_t)bh * N + n) * sstride;        // this chunk's state copy
    const int srow = (int)(scopy * 2 * kTcD);                   // H_s row in the state map

    if (tid == 0) {
        for (int i = 0; i < 8; ++i) mbar_init(&bars[i], i == 5 ? 2 : 1);   // bar_fin: 2
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        // the inputs first; the state pass's outputs (state copy, decays) after the wait
        // for it (with programmatic dependent launch this set-up overlaps that pass)
        mbar_arrive_expect_tx(bar_load, 32768 + MG * 256 + TOK * kTcD * 2 + 16 * MG);
        for (int h = 0; h < 2; ++h)
            for (int rb = 0; rb < MG / 64; ++rb)
                tc::tma_load_2d(sm + L::KT + h * MG * 128 + rb * 8192, &maps.k, h * 64,
                                (int)tok0 + rb * 64, bar_load);
        bulk_g2s(sm + L::QS, q + tok0 * kTcD, TOK * kTcD * 2, bar_load);
        if constexpr (!XOUT) {
            // the values, read by the readout only
            mbar_arrive_expect_tx(bar_v, MG * 256);
            for (int h = 0; h < 2; ++h)
                for (int rb = 0; rb < MG / 64; ++rb)
                    tc::tma_load_2d(sm + L::VT + h * MG * 128 + rb * 8192, &maps.v, h * 64,
                                    (int)tok0 + rb * 64, bar_v);
        }
    }
    if (warp == 0) {
        tc::tmem_alloc(tbase, TMEM_COLS);
        tc::tmem_relinquish();
    }
    griddep_wait();
    if (tid == 0) {
        for (int h = 0; h < 2; ++h)
            for (int rb = 0; rb < 2; ++rb)
                tc::tma_load_2d(sm + L::HM + h * 16384 + rb * 8192, &maps.state, h * 64,
                                srow + rb * 64, bar_load);
        for (int pl = 0; pl < 4; ++pl)
            bulk_g2s(sm + L::DEC + pl * 4 * MG, tokdec + pl * plane + tok0, 4 * MG, bar_load);
    }
    // decays of every position (from the state pass): l2_t = l_t log2(e) with l_t
    // the chunk-relative cumulative log (w_ti = exp2(l2_t - l2_i)), b_t = exp(l_t),
    // beta_t and beta_t^2.  Runs of weights w_ti over consecutive i or t are
    // products of beta: w_{t,i-1} = w_ti beta_i and w_{t+1,i} = w_ti beta_{t+1}.
    float *s_l2 = reinterpret_cast<float *>(sm + L::DEC);
    float *s_bt = s_l2 + MG, *s_bet = s_bt + MG, *s_beta2 = s_bet + MG;
    const int eHexp = state_exp[scopy * 2];
    const int eMexp = state_exp[scopy * 2 + 1];
    bool ok = mbar_wait_sleep(bar_load, 0, kTcSleepProbes, kTcSleepNs);
    // keys: bf16 -> fp16 in place, scaled below 1 (the values follow while the norm
    // products run); with the write gate, key and value rows of token i are taken
    // times sqrt(g_i), which puts g_i into every product that pairs them
    const float *gate_rows = gate ? gate + tok0 : nullptr;
    const float sK = tile_bf16_to_f16_rows_scaled<MG * 256, kSolveThreads, MG>(sm + L::KT, red,
                                                                               gate_rows);
    const __nv_bfloat16 *qs = reinterpret_cast<const __nv_bfloat16 *>(sm + L::QS);
    fence_proxy_async_smem();
    tc::fence_before_sync();
    ok = __syncthreads_and(ok);
    tc::fence_after_sync();
    const uint32_t tmem = *tbase;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);   // this warp's lane quarter
    // TMEM columns: Z1 | S, then Z3 (S is consumed before MMA3 writes Z3) | W | x_prev
    const uint32_t T_Z1 = 0, T_S = TOK, T_Z3 = TOK, T_W = 2 * TOK, T_XP = 3 * TOK;
    const uint32_t a_hm = sb + L::HM, a_kt = sb + L::KT, a_vt = sb + L::VT, b_xt = sb + L::XT,
                   b_pt = sb + L::PT;

    // Rows of S = K X^T (keys) held by this thread.  With MG = 64 the S product is
    // issued with M = 128 and an A operand that starts 32 rows (4 KB) before the key
    // tile: key t lands in TMEM lane 32 + t (lane quarters 1 and 2), and lanes 0-31
    // and 96-127 receive products of the neighbouring tiles (values, X^T: finite fp16
    // data not written meanwhile), which nothing reads.  This costs the same tensor
    // time as M = 64 and leaves lane quarters 0 and 3 out of the P phase.  MG = 128:
    // key t in lane t.
    constexpr bool kSOffset = (MG == 64);
    const bool s_owner = kSOffset ? (quarter == 1 || quarter == 2) : true;
    const int key = kSOffset ? d - 32 : d;
    // rows of G = K K^T (norm set-up, M = MG): M = 64 puts key 16w + l in lane
    // 32w + l (l < 16); M = 128 puts key t in lane t.
    const bool g_owner = (MG == 128) || (lane < 16);
    const int gkey = (MG == 128) ? d : quarter * 16 + lane;

    // ---- per-token ||H_j||_F (ai.info, Methodology: closed form through the
    // key Gram matrix).  Zn = H_s K^T gives u_i = k_i^T H_s k_i, G = K K^T the
    // intra-chunk terms:  ||H_j||^2 = b_j^2 ||H_s||^2 + 2 b_j X_j + R_j with
    // X_j = sum_{i<=j} w_ji u_i and R_j = beta_j^2 R_{j-1} + 2 E_j + G_jj^2,
    // E_j = sum_{i<j} w_ji G_ij^2 (R_j = sum_{i,l<=j} w_ji w_jl G_il^2).
    // Zn = H_s K^T in columns [0, MG), G = K K^T in [kGcol, kGcol + MG)
    constexpr uint32_t kGcol = 128;
    if (tid == 0 && ok) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint64_t kdesc = tc::sdesc(a_kt + (kk >> 2) * (MG * 128) + (kk & 3) * 32, 16, 1024);
            tc::mma_f16(tmem + 0, tc::sdesc(a_hm + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                        kdesc, tc::idesc_f16(128, MG, false, false), kk > 0);
            tc::mma_f16(tmem + kGcol, kdesc, kdesc, tc::idesc_f16(MG, MG, false, false), kk > 0);
        }
        tc::commit(bar_n);
    }
    // values: bf16 -> fp16 in place, scaled below 1 (first read by the readout; with
    // XOUT there is no readout, and the value tile is neither loaded nor converted)
    float sV = 1.f;
    if constexpr (!XOUT) {
        ok = mbar_wait_sleep(bar_v, 0, kTcSleepProbes, kTcSleepNs) && ok;
        sV = tile_bf16_to_f16_rows_scaled<MG * 256, kSolveThreads, MG>(sm + L::VT, red, gate_rows);
    }
    float *s_u = reinterpret_cast<float *>(sm + L::NRM);
    float *s_E = s_u + MG, *s_X = s_E + MG, *s_G = s_X + MG;   // [MG] each; E and X: wg 0 part
    float *s_E1 = reinterpret_cast<float *>(sm + L::NRM2), *s_X1 = s_E1 + MG;   // wg 1 part
    float *upart = reinterpret_cast<float *>(sm + L::UPART);
    {
        // ||H_s||_F^2 from the (scaled) fp16 copy
        float hs = 0.f;
        for (int c = tid * 16; c < 32768; c += kSolveThreads * 16) {
            const uint4 u4 = *reinterpret_cast<const uint4 *>(sm + L::HM + c);
            const __half *e = reinterpret_cast<const __half *>(&u4);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float x = __half2float(e[i]);
                hs = fmaf(x, x, hs);
            }
        }
        hs = warp_sum(hs);
        if (lane == 0) red[8 + warp] = hs;
    }
    // While the norm products run: the q column of this thread's tokens (token-major tile), kept packed for the
    // transpose below; |q_j|^2 = sum_d q_j[d]^2 by a reduce-scatter over the warp
    uint32_t qcol[TPT / 2];
    {
        float sq[TPT];
#pragma unroll
        for (int jj = 0; jj < TPT; jj += 2) {
            const __nv_bfloat16 lo = qs[(tcol + jj) * kTcD + d], hi = qs[(tcol + jj + 1) * kTcD + d];
            qcol[jj / 2] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
            const float a0 = __bfloat162float(lo), a1 = __bfloat162float(hi);
            sq[jj] = a0 * a0;
            sq[jj + 1] = a1 * a1;
        }
        reduce_scatter32<TPT>(sq, lane);
#pragma unroll
        for (int s2 = 0; s2 < TPT / 32; ++s2)
            reinterpret_cast<float *>(sm + L::QPART)[quarter * TOK + tcol + lane * (TPT / 32) + s2] =
                sq[s2];
    }
    if (!mbar_wait_sleep(bar_n, 0, kTcSleepProbes, kTcSleepNs)) ok = false;
    tc::fence_after_sync();
    {
        // u_i: thread (wg, d) forms k_i[d] (H_s k_i)[d] for its half of the keys,
        // then a sum over d (warp reduce-scatter, then the four lane quarters)
        const __half *kt = reinterpret_cast<const __half *>(sm + L::KT);
        const int hoff = (d >> 6) * (MG * 64), c = d & 63;
        float pv[HALF];
#pragma unroll
        for (int cb = 0; cb < HALF; cb += 16) {
            float zn[16];
            tc::tmem_ld16(tl + wg * HALF + cb, zn);
            tc::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 16; ++u)
                pv[cb + u] = zn[u] * __half2float(
                                         kt[hoff + tc::sw128_offset(wg * HALF + cb + u, c) / 2]);
        }
        reduce_scatter32<HALF>(pv, lane);
#pragma unroll
        for (int s2 = 0; s2 < HALF / 32; ++s2)
            upart[quarter * MG + wg * HALF + lane * (HALF / 32) + s2] = pv[s2];
    }
    __syncthreads();
    const float inv_uscale = pow2f(-eHexp) / (sK * sK);   // state exponents lie in [-120, 120]
    if (tid < MG) s_u[tid] = (upart[tid] + upart[MG + tid] + upart[2 * MG + tid] +
                              upart[3 * MG + tid]) * inv_uscale;
    __syncthreads();
    {
        // row `gkey` of G over this warpgroup's half of the columns: E, X, G_gkey,gkey
        const float gs = 1.f / (sK * sK);
        float es = 0.f, xs = 0.f, gjj = 0.f;
        bool has_diag = false;
        float g[HALF];
#pragma unroll
        for (int cb = 0; cb < HALF; cb += 16) tc::tmem_ld16(tl + kGcol + wg * HALF + cb, g + cb);
        tc::tmem_wait_ld();
        if (g_owner) {
            // i from the top of this half down: w = w_{gkey,i}, zero while i > gkey
            const int lo = wg * HALF, hi = lo + HALF - 1;
            float w = gkey > hi ? exp2f(s_l2[gkey] - s_l2[hi + 1]) : 0.f;
#pragma unroll
            for (int u = HALF - 1; u >= 0; --u) {
                const int i = lo + u;
                w = (i == gkey) ? 1.f : w * s_bet[min(i + 1, MG - 1)];   // w = 0 when i + 1 == MG
                const float gi = g[u] * gs;
                xs = fmaf(w, s_u[i], xs);
                if (i < gkey) es = fmaf(w * gi, gi, es);
                if (i == gkey) {
                    gjj = gi;
                    has_diag = true;
                }
            }
        }
        if (g_owner) {
            (wg == 0 ? s_E : s_E1)[gkey] = es;
            (wg == 0 ? s_X : s_X1)[gkey] = xs;
            if (has_diag) s_G[gkey] = gjj;
        }
    }
    __syncthreads();
    // R_j = beta_j^2 R_{j-1} + (2 E_j + G_jj^2), R_{-1} = 0: an affine recurrence,
    // scanned by warp 0 (lane l owns MG/32 consecutive positions) into s_u (free now)
    float *s_R = s_u;
    if (warp == 0) {
        constexpr int PER = MG / 32;
        float ca[PER], cb2[PER];
        float A = 1.f, Bc = 0.f;   // this lane's positions composed: R_out = A R_in + Bc
#pragma unroll
        for (int p = 0; p < PER; ++p) {
            const int j = lane * PER + p;
            ca[p] = s_beta2[j];
            cb2[p] = fmaf(2.f, s_E[j] + s_E1[j], s_G[j] * s_G[j]);
            Bc = fmaf(ca[p], Bc, cb2[p]);
            A *= ca[p];
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {   // inclusive scan of the compositions
            const float Ap = __shfl_up_sync(0xffffffffu, A, o);
            const float Bp = __shfl_up_sync(0xffffffffu, Bc, o);
            if (lane >= o) {
                Bc = fmaf(A, Bp, Bc);
                A *= Ap;
            }
        }
        float R = __shfl_up_sync(0xffffffffu, Bc, 1);   // R just before this lane's positions
        if (lane == 0) R = 0.f;
#pragma unroll
        for (int p = 0; p < PER; ++p) {
            R = fmaf(ca[p], R, cb2[p]);
            s_R[lane * PER + p] = R;
        }
    }
    __syncthreads();
    if (tid < TOK) {
        const int j = tid;
        float hs2s = 0.f;   // ||H_s||^2 of the scaled fp16 copy
#pragma unroll
        for (int w = 0; w < kSolveThreads / 32; ++w) hs2s += red[8 + w];
        // in double: after long runs of strong decay without writes b_j^2 ||H_s||^2
        // falls below the fp32 range while ||H_j|| itself (and, since the layer is
        // invariant to scaling H and M together, the output) is still well defined
        const double hs2 = (double)hs2s * pow2d(-2 * eHexp);
        const float b = s_bt[j];
        const double bj = b;
        const double n2 = bj * bj * hs2 + 2.0 * bj * (double)(s_X[j] + s_X1[j]) + (double)s_R[j];
        // a norm below 2^-120 (a state decayed that far since its last write) counts
        // as a zero state, whose output is 0: 1 / ||H_j|| would leave the fp32 range
        const float nj = n2 > 0x1p-240 ? (float)sqrt(n2) : 0.f;
        norms[tok0 + j] = nj;
        const float invd = nj > 0.f ? 1.f / (P.half_1p2a * nj) : 0.f;
        const float *qpart = reinterpret_cast<const float *>(sm + L::QPART);
        const float qn = sqrtf(qpart[j] + qpart[TOK + j] + qpart[2 * TOK + j] + qpart[3 * TOK + j]);
        const float eH = pow2f(-eHexp);
        const float eM = pow2f(-eMexp);
        // The iterate of token j is kept as x~ = (sigma / invd_j) x with sigma a power of
        // two common to the CTA.  Every Chebyshev iterate obeys ||x|| <= ||q|| (1+2a) /
        // (a d), so ||x~|| <= sigma ||q|| (1+2a) / a for every token, and in the scaled
        // domain (q - A x) / d reads sigma q - c1 Z1 - c3 Z3 - cl x~: the coefficient of
        // q is the same for all tokens.  c3 is folded into the decay weights below,
        // times a power of two s_j (s3_of below).
        const float c3 = invd / (sK * sK);
        s_c1[j] = b * invd * eH;
        s_c3[j] = c3;
        s_o1[j] = b * eM * invd;   // readout coefficient of Z1, times 1 / sigma below
        float mq = qn, mc = c3, mn = c3 > 0.f ? c3 : INFINITY;
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) {
            mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, o2));
            mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, o2));
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o2));
        }
        if (lane == 0) {
            red[warp] = mq;
            red[4 + warp] = mc;
            s_mn[warp] = mn;
        }
    }
    __syncthreads();
    // sigma puts every ||x~|| below 2^12
    float qmax = 0.f, c3max = 0.f, c3min = INFINITY;
#pragma unroll
    for (int w = 0; w < TOK / 32; ++w) {
        qmax = fmaxf(qmax, red[w]);
        c3max = fmaxf(c3max, red[4 + w]);
        c3min = fminf(c3min, s_mn[w]);
    }
    const float sigma = inv_pow2_above(qmax * (2.f * P.half_1p2a / P.a)) * 4096.f;
    // The weighted products c3_j w S go to fp16 as s_j c3_j w S, and Z3's column j
    // carries s_j, which the update and the readout take out again (exactly: s_j is a
    // power of two).  Normally one s_j = sc3 serves the whole chunk, scaling its
    // largest c3 below 1, and the update's Z3 coefficient is common to all tokens;
    // when the chunk's norms spread so far that the smallest c3 sc3 would lose fp16
    // precision (a state decayed far below its tokens' writes), every token takes its
    // own s_j with c3_j s_j in [1/2, 1).  Both give the same bits where both apply.
    // With 64-token chunks every token takes its own s_j always (measured faster than
    // carrying both update loops; with 128-token chunks the common loop is faster).
    constexpr bool kPerTokenAlways = TOK == 64;
    const float sc3 = inv_pow2_above(c3max);
    const bool s3_common = !kPerTokenAlways && c3max <= 0x1p12f * c3min;
    auto s3_of = [&](float c3j) { return s3_common ? sc3 : inv_pow2_above(c3j); };
    if (tid < TOK) {
        s_o1[tid] *= 1.f / sigma;
        s_t3[tid] = 1.f / s3_of(s_c3[tid]);
    }

    // q^T: this thread's tokens of row d, written into the (now free) tile as
    // [128 d][64 tokens] with 128B-swizzled rows: 8 tokens per 16-byte load later
#pragma unroll
    for (int ch = 0; ch < TPT / 8; ++ch) {
        const int t = tcol + ch * 8;             // first of 8 tokens
        st_shared_v4(sb + L::QS + (t >> 6) * 16384u + d * 128u + ((((t & 63) >> 3) ^ d) & 7u) * 16u,
                     qcol[4 * ch], qcol[4 * ch + 1], qcol[4 * ch + 2], qcol[4 * ch + 3]);
    }
    const float cl = 2.f * P.a / (1.f + 2.f * P.a);   // lambda / d for every token with H != 0

    // W^T rows: W[i][j] = s_j c3_j w_{ji}, w_{ji} = exp(l_j - l_i) for i <= j, else 0
    // (this thread's tokens); Z3 then carries s_j c3_j and its update coefficient is
    // -w / s_j
    {
        // w = w_{j,key} along this thread's tokens j (zero while j < key)
        const int js = tcol;
        float w = (s_owner && key <= js) ? exp2f(s_l2[js] - s_l2[key]) : 0.f;
        float wv[16];
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int j = js + c * 16 + u;
                if (c * 16 + u > 0) w = (j == key && s_owner) ? 1.f : w * s_bet[j];
                const float c3j = s_c3[tcol + c * 16 + u];
                wv[u] = w * (c3j * s3_of(c3j));   // s_j c3_j w_ji
            }
            tc::tmem_st16(tl + T_W + tcol + c * 16, wv);
        }
    }

    // x_1 = q / d, x_0 = 0 (x~_1 = sigma q): thread (wg, d) keeps element d of its 32
    // current iterates in registers and of the previous ones in TMEM
    float xc[TPT];
    {
        const float zero16[16] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f,
                                  0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        __syncthreads();   // q^T complete
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int t0 = tcol + c * 16;
            float qv[16];
            load_qrow16(sb + L::QS + (t0 >> 6) * 16384u, d, (t0 & 63) >> 4, qv);
#pragma unroll
            for (int u = 0; u < 16; ++u) xc[c * 16 + u] = qv[u] * sigma;
            st_row16(sb + L::XT + (t0 >> 6) * 16384u, d, t0 & 63, &xc[c * 16]);
            tc::tmem_st16(tl + T_XP + t0, zero16);
        }
        tc::tmem_wait_st();
    }
    if (P.r > 1) {   // the first Chebyshev round's tables: -w c1 and -w / s_j per token
        for (int e = tid; e < TOK; e += kSolveThreads) {
            s_coef[TOK + e] = -P.omega[1] * s_c1[e];
            if (!s3_common) s_coef3[TOK + e] = -P.omega[1] * s_t3[e];
        }
    }
    fence_proxy_async_smem();
    tc::fence_before_sync();
    ok = __syncthreads_and(ok);

    constexpr uint32_t IDESC_S = tc::idesc_f16(kSOffset ? 128 : MG, TOK, false, true);
    const uint32_t a_s = a_kt - (kSOffset ? 4096u : 0u);   // A operand start of S
    constexpr uint32_t IDESC_Z1 = tc::idesc_f16(128, TOK, false, true);
    constexpr uint32_t IDESC_Z3 = tc::idesc_f16(128, TOK, true, true);
    constexpr uint32_t PT_BLOCK = MG * 128;   // bytes between 64-token blocks of P^T
    // P-phase warps and the issuer of the intra-chunk product Z3
    constexpr int kZ3Issuer = kSOffset ? 96 : 128;   // lane 0 of warp 3 (MG 64) or 4 (MG 128)
    constexpr int kPBarThreads = kSOffset ? 5 * 32 : kSolveThreads - 32;
    const bool p_warp = kSOffset ? s_owner : (warp != 0);
    const bool in_pbar = p_warp || warp == kZ3Issuer / 32;
    bool m_requested = false;
    uint32_t ph = 0;   // phase parity of bar_s / bar_z1 / bar_z (each completes once per round)

    // Round structure.  Thread 0 issues S = K X^T (commit bar_s) and Z1 = H_s X^T
    // (commit bar_z1); issuing blocks it for about as long as the tensor core works,
    // so warp 0 takes no part in the P phase.  MG = 64: the key rows of S sit in
    // lane quarters 1-2, so warps 1, 2, 5, 6 form P and warp 3 issues Z3.  MG = 128:
    // warps 1-7 form P, warp 4 also covering warp 0's lane quarter, and warp 4
    // issues Z3.  The P warps and the Z3 issuer meet at a named barrier, so Z3 =
    // K^T P^T (commit bar_z) need not wait for the Z1 issue to finish.
    // XOUT (x_out: fp32 [B*H*T][128]): the rounds stop before the readout pass and the
    // iterates x_j themselves are written (the backward recomputes them this way).
    const int last_it = XOUT ? P.r - 1 : P.r;
#pragma unroll 1
    for (int it = 1; it <= last_it && ok; ++it) {
        const bool out_pass = (it == P.r);
        const float w_next = P.omega[it + 1 < kMaxSteps ? it + 1 : 0];   // next round's weight
        if (tid == 0) {
            tc::fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                tc::mma_f16(tmem + T_S,
                            tc::sdesc(a_s + (kk >> 2) * (MG * 128) + (kk & 3) * 32, 16, 1024),
                            tc::sdesc(b_xt + kk * 2048, 16384, 1024), IDESC_S, kk > 0);
            tc::commit(bar_s);
            if (out_pass) {
                if (!m_requested) {
                    mbar_arrive_expect_tx(bar_m, 32768);
                    for (int h = 0; h < 2; ++h)
                        for (int rb = 0; rb < 2; ++rb)
                            tc::tma_load_2d(sm + L::HM + h * 16384 + rb * 8192, &maps.state, h * 64,
                                            srow + kTcD + rb * 64, bar_m);
                    m_requested = true;
                }
                if (!mbar_wait_bounded(bar_m, 0, kTcWaitProbes)) ok = false;
            }
            // Z1 = H_s X^T (M_s X^T on the readout pass)
            if (ok) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_f16(tmem + T_Z1,
                                tc::sdesc(a_hm + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                                tc::sdesc(b_xt + kk * 2048, 16384, 1024), IDESC_Z1, kk > 0);
            }
            tc::commit(bar_z1);
        }
        // the issuing lane's warp reconverges before anyone in it waits on a barrier
        // that this lane's issue completes (a suspended wait would stall the issue)
        if (warp == 0) __syncwarp();
        if (in_pbar) {
            if (p_warp) {
                // P^T = W o S^T -> fp16, MN-major tile of MG rows
                if (!mbar_wait_sleep(bar_s, ph, kTcSleepProbes, kTcSleepNs)) ok = false;
                tc::fence_after_sync();
                const bool both = !kSOffset && warp == 4;
#pragma unroll 1
                for (int hh = 0; hh < (both ? 2 : 1); ++hh) {
                    const int tb = both ? hh * TPT : tcol;
#pragma unroll
                    for (int c = 0; c < NCH; ++c) {
                        const int t0 = tb + c * 16;
                        float sv[16], wv[16];
                        tc::tmem_ld16(tl + T_S + t0, sv);
                        tc::tmem_ld16(tl + T_W + t0, wv);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int u = 0; u < 16; u += 2) {
                            const float2 p2 = __fmul2_rn(make_float2(sv[u], sv[u + 1]),
                                                         make_float2(wv[u], wv[u + 1]));
                            sv[u] = p2.x;
                            sv[u + 1] = p2.y;
                        }
                        st_row16(b_pt + (t0 >> 6) * PT_BLOCK, key, t0 & 63, sv);
                    }
                }
                fence_proxy_async_smem();
                tc::fence_before_sync();
            }
            named_barrier_sync(1, kPBarThreads);
            if (tid == kZ3Issuer) {
                tc::fence_after_sync();
                const uint32_t a3 = out_pass ? a_vt : a_kt;
#pragma unroll
                for (int kk = 0; kk < MG / 16; ++kk)
                    tc::mma_f16(tmem + T_Z3, tc::sdesc(a3 + kk * 2048, MG * 128, 1024),
                                tc::sdesc(b_pt + kk * 2048, PT_BLOCK, 1024), IDESC_Z3, kk > 0);
                tc::commit(bar_z);
            }
            if (warp == kZ3Issuer / 32) __syncwarp();
        }
        // x_new = (1 - w) x_prev + w (1 - lambda/d) x + w cq q - w c1 Z1 - w c3 Z3 (the
        // three-term update with the residual (q - A x)/d written out; the per-token
        // products -w c1 and -w / s_j of this round come from the tables; the q
        // coefficient w sigma is common to all tokens), in two parts:
        // A, as soon as Z1 = H_s X^T is done (while the P phase and the intra-chunk
        // product run): part = (1 - w) x_prev + w (1 - lambda/d) x + w cq q - w c1 Z1,
        // kept in the x_prev columns of TMEM; B, once Z3 is done: x_new = part - w c3 Z3.
        // Pairs of tokens go through the packed f32x2 FMA pipe.
        const float cAs = 1.f - P.omega[it], cBs = P.omega[it] * (1.f - cl);
        const float kqs = P.omega[it] * sigma, k3s = -P.omega[it] / sc3;
        const float2 cA = make_float2(cAs, cAs), cB = make_float2(cBs, cBs);
        const float2 kq = make_float2(kqs, kqs);
        const float *k1 = s_coef + (it & 1) * TOK, *k3t = s_coef3 + (it & 1) * TOK;
        if (!mbar_wait_sleep(bar_z1, ph, kTcSleepProbes, kTcSleepNs)) ok = false;
        tc::fence_after_sync();
        if (!out_pass) {
            if (tid == 0 && it == P.r - 1 && !XOUT) {
                // H_s is no longer read: fetch M_s for the readout into the same buffer
                mbar_arrive_expect_tx(bar_m, 32768);
                for (int h = 0; h < 2; ++h)
                    for (int rb = 0; rb < 2; ++rb)
                        tc::tma_load_2d(sm + L::HM + h * 16384 + rb * 8192, &maps.state, h * 64,
                                        srow + kTcD + rb * 64, bar_m);
                m_requested = true;
            }
            // the previous round's x_prev stores (not waited for at its end) land first
            tc::tmem_wait_st();
#pragma unroll
            for (int c = 0; c < TPT / 8; ++c) {   // 8 tokens at a time
                const int t0 = tcol + c * 8;
                float z1[8], xp[8];
                tc::tmem_ld8(tl + T_Z1 + t0, z1);
                tc::tmem_ld8(tl + T_XP + t0, xp);
                const uint4 qw4 = ld_shared_u4(sb + L::QS + (t0 >> 6) * 16384u + d * 128u +
                                               ((((uint32_t)(t0 & 63) >> 3) ^ d) & 7u) * 16u);
                const float4 g1[2] = {*reinterpret_cast<const float4 *>(k1 + t0),
                                      *reinterpret_cast<const float4 *>(k1 + t0 + 4)};
                tc::tmem_wait_ld();
                const uint32_t qw[4] = {qw4.x, qw4.y, qw4.z, qw4.w};
                float part[8];
#pragma unroll
                for (int p = 0; p < 4; ++p) {   // tokens 2p, 2p + 1
                    const float2 g1p = (p & 1) ? make_float2(g1[p >> 1].z, g1[p >> 1].w)
                                               : make_float2(g1[p >> 1].x, g1[p >> 1].y);
                    // q^T holds bf16 pairs: the low half is token 2p, the high half 2p + 1
                    const float2 qv = make_float2(__uint_as_float(qw[p] << 16),
                                                  __uint_as_float(qw[p] & 0xffff0000u));
                    float2 t = __fmul2_rn(g1p, make_float2(z1[2 * p], z1[2 * p + 1]));
                    t = __ffma2_rn(kq, qv, t);
                    t = __ffma2_rn(cB, make_float2(xc[c * 8 + 2 * p], xc[c * 8 + 2 * p + 1]), t);
                    t = __ffma2_rn(cA, make_float2(xp[2 * p], xp[2 * p + 1]), t);
                    part[2 * p] = t.x;
                    part[2 * p + 1] = t.y;
                }
                tc::tmem_st8(tl + T_XP + t0, part);
            }
        }
        if (!mbar_wait_sleep(bar_z, ph, kTcSleepProbes, kTcSleepNs)) ok = false;
        tc::fence_after_sync();
        ph ^= 1u;
        if (!out_pass) {
            tc::tmem_wait_st();   // this thread's parts are in TMEM
            // x_new = part + k3_j Z3_j: k3 = -w / sc3 for the whole chunk, or -w / s_j from
            // the table (two copies of the loop, so that the common case loads nothing)
            auto update_b = [&](auto per_token) {
#pragma unroll
                for (int c = 0; c < TPT / 8; ++c) {
                    const int t0 = tcol + c * 8;
                    float z3[8], part[8];
                    tc::tmem_ld8(tl + T_Z3 + t0, z3);
                    tc::tmem_ld8(tl + T_XP + t0, part);
                    float4 g3[2];
                    if constexpr (decltype(per_token)::value) {
                        g3[0] = *reinterpret_cast<const float4 *>(k3t + t0);
                        g3[1] = *reinterpret_cast<const float4 *>(k3t + t0 + 4);
                    }
                    tc::tmem_wait_ld();
                    // x becomes the next round's x_prev (the part just read is dead), and
                    // the new iterate takes x's registers
                    tc::tmem_st8(tl + T_XP + t0, &xc[c * 8]);
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        float2 k3 = make_float2(k3s, k3s);
                        if constexpr (decltype(per_token)::value)
                            k3 = (p & 1) ? make_float2(g3[p >> 1].z, g3[p >> 1].w)
                                         : make_float2(g3[p >> 1].x, g3[p >> 1].y);
                        const float2 t = __ffma2_rn(k3, make_float2(z3[2 * p], z3[2 * p + 1]),
                                                    make_float2(part[2 * p], part[2 * p + 1]));
                        xc[c * 8 + 2 * p] = t.x;
                        xc[c * 8 + 2 * p + 1] = t.y;
                    }
                    st_row8(sb + L::XT + (t0 >> 6) * 16384u, d, t0 & 63, &xc[c * 8]);
                }
            };
            if constexpr (kPerTokenAlways) {
                update_b(std::true_type{});
            } else {
                if (s3_common)
                    update_b(std::false_type{});
                else
                    update_b(std::true_type{});
            }
            // the next round's coefficient table (the other buffer)
            if (it + 1 < P.r) {
                for (int e = tid; e < TOK; e += kSolveThreads) {
                    s_coef[((it + 1) & 1) * TOK + e] = -w_next * s_c1[e];
                    if (!s3_common) s_coef3[((it + 1) & 1) * TOK + e] = -w_next * s_t3[e];
                }
            }
            fence_proxy_async_smem();
            tc::fence_before_sync();
            ok = __syncthreads_and(ok);
        } else if (ok) {
            // o_j[d] = b_j (M_s x_j)[d] + sum_i w_{ji} (k_i . x_j) v_i[d]; Z3 carries
            // s_j c3_j, so its readout coefficient is sK / (sV sigma) / s_j
            const float o3 = sK / (sV * sigma);
            __nv_bfloat16 *orow = o + (tok0 + tcol) * kTcD + d;
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                const int t0 = tcol + c * 16;
                float z1[16], z3[16], o1[16], t3[16];
                tc::tmem_ld16(tl + T_Z1 + t0, z1);
                tc::tmem_ld16(tl + T_Z3 + t0, z3);
                ld_f32x16(s_o1 + t0, o1);
                ld_f32x16(s_t3 + t0, t3);
                tc::tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    orow[(size_t)(c * 16 + u) * kTcD] =
                        __float2bfloat16_rn(fmaf(o1[u], z1[u], (o3 * t3[u]) * z3[u]));
            }
        }
    }

    if (XOUT && ok) {
        // x_j = x~_j invd_j / sigma, invd_j = c3_j sK^2 (thread (wg, d): element d of
        // its tokens; consecutive d of a token are consecutive threads)
        const float xs = sK * sK / sigma;
        float *xrow = x_out + (tok0 + tcol) * kTcD + d;
#pragma unroll
        for (int u = 0; u < TPT; ++u) xrow[(size_t)u * kTcD] = xc[u] * (s_c3[tcol + u] * xs);
    }
    // teardown: no MMA, copy or TMEM store of this CTA may be in flight when TMEM is freed
    tc::tmem_wait_st();
    ok = __syncthreads_and(ok);
    if (!ok) {
        if (tid == kZ3Issuer) tc::commit(bar_fin);   // bar_fin counts two arrivals
        if (tid == 0) {
            atomicExch(timeout_flag, 1);
            tc::commit(bar_fin);
            mbar_wait_bounded(bar_fin, 0, kTcWaitProbes);
            mbar_wait_bounded(bar_load, 0, kTcWaitProbes);
            if (!XOUT) mbar_wait_bounded(bar_v, 0, kTcWaitProbes);
            if (m_requested) mbar_wait_bounded(bar_m, 0, kTcWaitProbes);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace gka
