// Recurrent GKA decode step: one token per head on an fp32 state held in HBM.
//
// Method: "Gated KalmaNet" (arXiv 2511.21016), ai.info page, Key
// Contributions 2 and 4 (recurrent form for inference) and Methodology:
//   H <- beta H + k k^T;  n = ||H||_F;  lambda = a n;
//   x = r-step Chebyshev for (H + lambda I) x = q on [a n, (1+a) n];
//   M <- beta M + v k^T;  o = M x.
// With the write gate g (the paper's beta_t-augmented variant, ai.info page,
// Main Findings; nullable, NULL = 1) the writes are g k k^T and g v k^T.
//
// The step is bound by HBM traffic: each head reads and writes 2 * D * D fp32
// state words once.  One CTA of 4*D threads serves one head.  H stays in
// registers through all r - 1 matrix-vector products (warp w owns rows
// 8w..8w+7, lane l owns columns l*D/32 .. l*D/32 + D/32 - 1 of each), while a
// bulk async copy streams M into shared memory in the background.
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "tcgen05.cuh"

namespace gka {

// Sums, over the 32 lanes of a warp, each of the 8 per-row partials v[0..7].
// On return every lane holds the total of row rowsel(lane) in v[0], where
// rowsel(lane) = 4*bit4 + 2*bit3 + bit2 of the lane id (a reduce-scatter by
// halving, 9 shuffles instead of 40).
__device__ __forceinline__ float rows8_reduce(float v[8], int lane) {
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const float send = b4 ? v[s] : v[s + 4];
        const float keep = b4 ? v[s + 4] : v[s];
        v[s] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        const float send = b3 ? v[s] : v[s + 2];
        const float keep = b3 ? v[s + 2] : v[s];
        v[s] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    {
        const float send = b2 ? v[0] : v[1];
        const float keep = b2 ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 2);
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
    return v[0];
}

__device__ __forceinline__ int rows8_sel(int lane) {
    return ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
}

template <int CPL>
struct VecF;
template <>
struct VecF<1> {
    __device__ static void ld(const float *p, float *x) { x[0] = *p; }
    __device__ static void st(float *p, const float *x) { *p = x[0]; }
};
template <>
struct VecF<2> {
    __device__ static void ld(const float *p, float *x) {
        const float2 t = *reinterpret_cast<const float2 *>(p);
        x[0] = t.x; x[1] = t.y;
    }
    __device__ static void st(float *p, const float *x) {
        *reinterpret_cast<float2 *>(p) = make_float2(x[0], x[1]);
    }
};
template <>
struct VecF<4> {
    __device__ static void ld(const float *p, float *x) {
        const float4 t = *reinterpret_cast<const float4 *>(p);
        x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    }
    __device__ static void st(float *p, const float *x) {
        *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
    }
};

constexpr uint32_t kDecodeWaitProbes = 1u << 22;

template <typename Tin, int D>
__global__ void __launch_bounds__(4 * D, 2)
k_decode_step(float *__restrict__ state, const Tin *__restrict__ q, const Tin *__restrict__ k,
              const Tin *__restrict__ v, const float *__restrict__ beta,
              const float *__restrict__ gate, Tin *__restrict__ o,
              const ChebParams P, int *__restrict__ timeout_flag) {
    constexpr int NT = 4 * D, NW = NT / 32, CPL = D / 32;
    extern __shared__ __align__(128) float Msm[];   // [D][D] M tile
    __shared__ __align__(16) float xbuf[2][D];
    __shared__ float ks[D], vs[D];
    __shared__ float red[NW];
    __shared__ __align__(8) uint64_t mbar;

    const int head = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float *Hg = state + (size_t)head * 2 * D * D;
    float *Mg = Hg + D * D;

    if (tid == 0) {
        mbar_init(&mbar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        mbar_arrive_expect_tx(&mbar, D * D * 4);
        bulk_g2s(Msm, Mg, D * D * 4, &mbar);
    }
    const float bt = beta[head];
    const float gt = gate ? gate[head] : 1.f;   // write gate: g k k^T and g v k^T
    for (int i = tid; i < D; i += NT) {
        ks[i] = load_f(k + (size_t)head * D + i);
        vs[i] = load_f(v + (size_t)head * D + i) * gt;
    }
    __syncthreads();

    // H <- beta H + k k^T (registers), written back at once
    const int row0 = warp * 8, col0 = lane * CPL;
    float h[8][CPL];
    float ss = 0.f;
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
        float *rowp = Hg + (size_t)(row0 + rr) * D + col0;
        VecF<CPL>::ld(rowp, h[rr]);
        const float kr = ks[row0 + rr] * gt;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            h[rr][c] = fmaf(bt, h[rr][c], kr * ks[col0 + c]);
            ss = fmaf(h[rr][c], h[rr][c], ss);
        }
        VecF<CPL>::st(rowp, h[rr]);
    }
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    float n2 = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) n2 += red[w];
    const float nrm = sqrtf(n2);
    const float lam = P.a * nrm;
    const float invd = nrm > 0.f ? 1.f / (P.half_1p2a * nrm) : 0.f;

    // Chebyshev: the owner lane (lane % 4 == 0) of row R keeps x_prev, x_cur, q
    const int R = row0 + rows8_sel(lane);
    const bool owner = (lane & 3) == 0;
    const float qR = load_f(q + (size_t)head * D + R);
    float xprev = 0.f, xcur = qR * invd;
    if (owner) xbuf[0][R] = xcur;
    __syncthreads();
    int cur = 0;
#pragma unroll 1
    for (int it = 1; it < P.r; ++it) {
        float xv[CPL];
        VecF<CPL>::ld(&xbuf[cur][col0], xv);
        float part[8];
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
            float s = 0.f;
#pragma unroll
            for (int c = 0; c < CPL; ++c) s = fmaf(h[rr][c], xv[c], s);
            part[rr] = s;
        }
        const float y = fmaf(lam, xcur, rows8_reduce(part, lane));
        const float xn = fmaf(P.omega[it], fmaf(qR - y, invd, xcur - xprev), xprev);
        xprev = xcur;
        xcur = xn;
        if (owner) xbuf[cur ^ 1][R] = xn;
        __syncthreads();
        cur ^= 1;
    }

    // M <- beta M + v k^T and o = M x
    if (!mbar_wait_bounded(&mbar, 0, kDecodeWaitProbes)) {
        if (tid == 0) atomicExch(timeout_flag, 1);
        mbar_wait_bounded(&mbar, 0, kDecodeWaitProbes);   // let the copy land before exit
        return;
    }
    float xv[CPL];
    VecF<CPL>::ld(&xbuf[cur][col0], xv);
    float part[8];
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
        float m[CPL];
        VecF<CPL>::ld(&Msm[(row0 + rr) * D + col0], m);
        const float vr = vs[row0 + rr];
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            m[c] = fmaf(bt, m[c], vr * ks[col0 + c]);
            s = fmaf(m[c], xv[c], s);
        }
        VecF<CPL>::st(Mg + (size_t)(row0 + rr) * D + col0, m);
        part[rr] = s;
    }
    const float orow = rows8_reduce(part, lane);
    if (owner) store_f(o + (size_t)head * D + R, invd > 0.f ? orow : 0.f);
}

// ---------------------------------------------------------------------------
// Decode step for D = 128, one row per thread: a CTA of 128 threads serves one
// head and thread t owns row t of H (128 fp32 registers) for all r - 1
// matrix-vector products, so a product needs no cross-thread reduction: x is
// broadcast from shared memory and y_t = sum_c H[t][c] x[c] stays in the thread.
// H and M move between HBM and a 64 KB shared buffer as 128-byte-swizzled TMA
// tiles (bank-conflict-free row access); M is fetched into the buffer while the
// products run, and the updated M and H leave through the same buffer with TMA
// stores.  Three heads share an SM.
// ---------------------------------------------------------------------------
constexpr int kDecD = 128;
constexpr int kDecRowThreads = kDecD;
constexpr size_t kDecRowSmem = 65536 + 1024;

struct DecodeMaps {
    CUtensorMap state;   // fp32 [B*H*2*128 rows][128], box 32 x 128, 128B swizzle
};

// Byte offset of fp32 element (row, 4*chunk) in the swizzled [128][128] tile
// stored as four 32-column boxes.
__device__ __forceinline__ uint32_t dec_tile_off(int row, int chunk) {
    return (uint32_t)(chunk >> 3) * 16384u + (uint32_t)row * 128u +
           (uint32_t)(((chunk & 7) ^ row) & 7) * 16u;
}

template <typename Tin>
__global__ void __launch_bounds__(kDecRowThreads, 3)
k_decode_rows(const __grid_constant__ DecodeMaps maps, const Tin *__restrict__ q,
              const Tin *__restrict__ k, const Tin *__restrict__ v, const float *__restrict__ beta,
              const float *__restrict__ gate, Tin *__restrict__ o, const ChebParams P, int *__restrict__ timeout_flag) {
    constexpr int D = kDecD, NW = kDecRowThreads / 32;
    extern __shared__ uint8_t draw[];
    uint8_t *buf = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(draw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    __shared__ __align__(16) float xbuf[2][D];
    __shared__ __align__(16) float ks[D];
    __shared__ float vs[D];   // g v_t, parked here through the products (frees a register)
    __shared__ float red[NW];
    __shared__ __align__(8) uint64_t bar[2];

    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int head = blockIdx.x;
    const int hrow = head * 2 * D;          // first row of H in the state map; M follows

    if (t == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (t == 0) {
        mbar_arrive_expect_tx(&bar[0], D * D * 4);
        for (int b = 0; b < 4; ++b) tc::tma_load_2d(buf + b * 16384, &maps.state, b * 32, hrow, &bar[0]);
    }
    const float bt = beta[head];
    const float gt = gate ? gate[head] : 1.f;   // write gate: g k k^T and g v k^T
    ks[t] = load_f(k + (size_t)head * D + t);
    vs[t] = load_f(v + (size_t)head * D + t) * gt;
    const float qt = load_f(q + (size_t)head * D + t);
    bool ok = mbar_wait_bounded(&bar[0], 0, kDecodeWaitProbes);
    __syncthreads();   // ks complete

    // H row t -> registers, updated: h = beta h + k_t k
    float h[D];
    const float kt = ks[t] * gt;
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < D / 4; ++c) {
        const float4 hv = *reinterpret_cast<const float4 *>(buf + dec_tile_off(t, c));
        const float4 kv = *reinterpret_cast<const float4 *>(&ks[4 * c]);
        h[4 * c + 0] = fmaf(bt, hv.x, kt * kv.x);
        h[4 * c + 1] = fmaf(bt, hv.y, kt * kv.y);
        h[4 * c + 2] = fmaf(bt, hv.z, kt * kv.z);
        h[4 * c + 3] = fmaf(bt, hv.w, kt * kv.w);
        ss = fmaf(h[4 * c], h[4 * c], ss);
        ss = fmaf(h[4 * c + 1], h[4 * c + 1], ss);
        ss = fmaf(h[4 * c + 2], h[4 * c + 2], ss);
        ss = fmaf(h[4 * c + 3], h[4 * c + 3], ss);
    }
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    // buffer free: fetch M while the products run
    fence_proxy_async_smem();
    ok = __syncthreads_and(ok);
    if (t == 0 && ok) {
        mbar_arrive_expect_tx(&bar[1], D * D * 4);
        for (int b = 0; b < 4; ++b)
            tc::tma_load_2d(buf + b * 16384, &maps.state, b * 32, hrow + D, &bar[1]);
    }
    float n2 = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) n2 += red[w];
    const float nrm = sqrtf(n2);
    const float lam = P.a * nrm;
    const float invd = nrm > 0.f ? 1.f / (P.half_1p2a * nrm) : 0.f;

    // Chebyshev: thread t keeps element t of x_prev, x_cur
    float xprev = 0.f, xcur = qt * invd;
    xbuf[0][t] = xcur;
    __syncthreads();
    int cur = 0;
#pragma unroll 1
    for (int it = 1; it < P.r; ++it) {
        // packed f32x2 FMAs: half the issued instructions of scalar ones (the step runs
        // close to the power cap, where fewer issued instructions leave more clock)
        float2 y01 = make_float2(0.f, 0.f), y23 = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < D / 4; ++c) {
            const float4 xv = *reinterpret_cast<const float4 *>(&xbuf[cur][4 * c]);
            y01 = __ffma2_rn(make_float2(h[4 * c], h[4 * c + 1]), make_float2(xv.x, xv.y), y01);
            y23 = __ffma2_rn(make_float2(h[4 * c + 2], h[4 * c + 3]), make_float2(xv.z, xv.w), y23);
        }
        const float y = fmaf(lam, xcur, (y01.x + y01.y) + (y23.x + y23.y));
        const float xn = fmaf(P.omega[it], fmaf(qt - y, invd, xcur - xprev), xprev);
        xprev = xcur;
        xcur = xn;
        xbuf[cur ^ 1][t] = xn;
        __syncthreads();
        cur ^= 1;
    }

    // M row t: m = beta m + v_t k, o_t = m . x; the updated row goes back in place
    if (!mbar_wait_bounded(&bar[1], 0, kDecodeWaitProbes)) ok = false;
    const float vt = vs[t];
    const float bm = beta[head];   // reloaded (cached) rather than held through the products
    // (h stays live through this loop for the store below: a partial unroll and two
    // accumulators keep the loop's temporaries within the register budget, no spill)
    float2 o01 = make_float2(0.f, 0.f);
    const float2 bm2 = make_float2(bm, bm), vt2 = make_float2(vt, vt);
#pragma unroll 4
    for (int c = 0; c < D / 4; ++c) {
        float4 *p = reinterpret_cast<float4 *>(buf + dec_tile_off(t, c));
        const float4 mv = *p;
        const float4 kv = *reinterpret_cast<const float4 *>(&ks[4 * c]);
        const float4 xv = *reinterpret_cast<const float4 *>(&xbuf[cur][4 * c]);
        const float2 m01 = __ffma2_rn(bm2, make_float2(mv.x, mv.y),
                                      __fmul2_rn(vt2, make_float2(kv.x, kv.y)));
        const float2 m23 = __ffma2_rn(bm2, make_float2(mv.z, mv.w),
                                      __fmul2_rn(vt2, make_float2(kv.z, kv.w)));
        o01 = __ffma2_rn(m01, make_float2(xv.x, xv.y), o01);
        o01 = __ffma2_rn(m23, make_float2(xv.z, xv.w), o01);
        *p = make_float4(m01.x, m01.y, m23.x, m23.y);
    }
    store_f(o + (size_t)head * D + t, invd > 0.f ? o01.x + o01.y : 0.f);
    fence_proxy_async_smem();
    ok = __syncthreads_and(ok);
    if (t == 0 && ok) {
        for (int b = 0; b < 4; ++b) tc::tma_store_2d(&maps.state, b * 32, hrow + D, buf + b * 16384);
        tc::bulk_commit();
        tc::bulk_wait_read0();
    }
    __syncthreads();
    // updated H row t back through the buffer
#pragma unroll
    for (int c = 0; c < D / 4; ++c)
        *reinterpret_cast<float4 *>(buf + dec_tile_off(t, c)) =
            make_float4(h[4 * c], h[4 * c + 1], h[4 * c + 2], h[4 * c + 3]);
    fence_proxy_async_smem();
    __syncthreads();
    if (t == 0) {
        if (ok) {
            for (int b = 0; b < 4; ++b) tc::tma_store_2d(&maps.state, b * 32, hrow, buf + b * 16384);
            tc::bulk_commit();
            tc::bulk_wait0();
        } else {
            atomicExch(timeout_flag, 1);
            mbar_wait_bounded(&bar[0], 0, kDecodeWaitProbes);
            mbar_wait_bounded(&bar[1], 0, kDecodeWaitProbes);
        }
    }
}

}  // namespace gka
