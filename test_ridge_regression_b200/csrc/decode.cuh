// Recurrent GKA decode step: one token per head on an fp32 state held in HBM.
//
// Method: "Gated KalmaNet" (arXiv 2511.21016), ai.info page, Key
// Contributions 2 and 4 (recurrent form for inference) and Methodology:
//   H <- beta H + k k^T;  n = ||H||_F;  lambda = a n;
//   x = r-step Chebyshev for (H + lambda I) x = q on [a n, (1+a) n];
//   M <- beta M + v k^T;  o = M x.
//
// The step is bound by HBM traffic: each head reads and writes 2 * D * D fp32
// state words once.  One CTA of 4*D threads serves one head.  H stays in
// registers through all r - 1 matrix-vector products (warp w owns rows
// 8w..8w+7, lane l owns columns l*D/32 .. l*D/32 + D/32 - 1 of each), while a
// bulk async copy streams M into shared memory in the background.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

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
              const Tin *__restrict__ v, const float *__restrict__ beta, Tin *__restrict__ o,
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
    for (int i = tid; i < D; i += NT) {
        ks[i] = load_f(k + (size_t)head * D + i);
        vs[i] = load_f(v + (size_t)head * D + i);
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
        const float kr = ks[row0 + rr];
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
// Persistent, software-pipelined decode step for D = 128: one CTA of 512
// threads per SM walks its share of the heads.  While head i is updated and
// iterated (H in registers), bulk async copies already bring H, M, q, k, v of
// head i+1 into shared memory, so the HBM stream does not pause during the
// r - 1 matrix-vector products.  Shared memory: one H buffer (64 KB) and two
// M buffers (2 x 64 KB); the H buffer is refilled as soon as every thread has
// copied H_i into its registers.
// ---------------------------------------------------------------------------
constexpr int kDecD = 128;
constexpr int kDecThreads = 4 * kDecD;
constexpr size_t kDecSmem = 3 * 65536 + 2 * 3 * 512 + 1024 + 1024;

template <typename Tin>
__global__ void __launch_bounds__(kDecThreads, 1)
k_decode_pipelined(float *__restrict__ state, const Tin *__restrict__ q, const Tin *__restrict__ k,
                   const Tin *__restrict__ v, const float *__restrict__ beta, Tin *__restrict__ o,
                   int num_heads, const ChebParams P, int *__restrict__ timeout_flag) {
    constexpr int D = kDecD, NW = kDecThreads / 32, CPL = D / 32;
    constexpr uint32_t ROWB = D * sizeof(Tin);               // bytes of one q/k/v row
    extern __shared__ __align__(128) uint8_t dsm[];
    float *Hbuf = reinterpret_cast<float *>(dsm);             // [D][D]
    float *Mbuf = Hbuf + D * D;                               // [2][D][D]
    uint8_t *qkv = dsm + 3 * 65536;                           // [2][3][ROWB]
    __shared__ __align__(16) float xbuf[2][D];
    __shared__ float ks[D], vs[D];
    __shared__ float red[NW];
    __shared__ __align__(8) uint64_t barH, barM[2];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row0 = warp * 8, col0 = lane * CPL;
    const int G = gridDim.x;
    int head = blockIdx.x;
    if (head >= num_heads) return;

    auto issue = [&](int h, int buf, bool with_h) {
        // H (if requested) into Hbuf, M and q, k, v into buffer `buf`
        const float *Hg = state + (size_t)h * 2 * D * D;
        if (with_h) {
            mbar_arrive_expect_tx(&barH, D * D * 4);
            bulk_g2s(Hbuf, Hg, D * D * 4, &barH);
        }
        mbar_arrive_expect_tx(&barM[buf], D * D * 4 + 3 * ROWB);
        bulk_g2s(Mbuf + buf * D * D, Hg + D * D, D * D * 4, &barM[buf]);
        uint8_t *dst = qkv + buf * 3 * ROWB;
        bulk_g2s(dst, q + (size_t)h * D, ROWB, &barM[buf]);
        bulk_g2s(dst + ROWB, k + (size_t)h * D, ROWB, &barM[buf]);
        bulk_g2s(dst + 2 * ROWB, v + (size_t)h * D, ROWB, &barM[buf]);
    };

    if (tid == 0) {
        mbar_init(&barH, 1);
        mbar_init(&barM[0], 1);
        mbar_init(&barM[1], 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) issue(head, 0, true);

    bool ok = true;
    for (int i = 0; head < num_heads; ++i, head += G) {
        const int buf = i & 1;
        const int next = head + G;
        const float bt = beta[head];
        // H_i: shared -> registers, then the buffer goes back to the copy engine
        if (!mbar_wait_bounded(&barH, i & 1, kDecodeWaitProbes)) ok = false;
        float h[8][CPL];
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) VecF<CPL>::ld(&Hbuf[(row0 + rr) * D + col0], h[rr]);
        // q, k, v of this head (arrived with M_i on barM[buf])
        if (!mbar_wait_bounded(&barM[buf], (i >> 1) & 1, kDecodeWaitProbes)) ok = false;
        const Tin *qr = reinterpret_cast<const Tin *>(qkv + buf * 3 * ROWB);
        for (int j = tid; j < D; j += kDecThreads) {
            ks[j] = load_f(qr + D + j);
            vs[j] = load_f(qr + 2 * D + j);
        }
        fence_proxy_async_smem();
        ok = __syncthreads_and(ok);
        if (!ok) break;
        if (tid == 0 && next < num_heads) issue(next, buf ^ 1, true);

        // H <- beta H + k k^T, written back at once
        float *Hg = state + (size_t)head * 2 * D * D;
        float ss = 0.f;
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
            const float kr = ks[row0 + rr];
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                h[rr][c] = fmaf(bt, h[rr][c], kr * ks[col0 + c]);
                ss = fmaf(h[rr][c], h[rr][c], ss);
            }
            VecF<CPL>::st(Hg + (size_t)(row0 + rr) * D + col0, h[rr]);
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
        const float qR = load_f(qr + R);
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
                float s2 = 0.f;
#pragma unroll
                for (int c = 0; c < CPL; ++c) s2 = fmaf(h[rr][c], xv[c], s2);
                part[rr] = s2;
            }
            const float y = fmaf(lam, xcur, rows8_reduce(part, lane));
            const float xn = fmaf(P.omega[it], fmaf(qR - y, invd, xcur - xprev), xprev);
            xprev = xcur;
            xcur = xn;
            if (owner) xbuf[cur ^ 1][R] = xn;
            __syncthreads();
            cur ^= 1;
        }

        // M <- beta M + v k^T and o = M x (M_i is in Mbuf[buf])
        const float *Ms = Mbuf + buf * D * D;
        float *Mg = Hg + D * D;
        float xv[CPL];
        VecF<CPL>::ld(&xbuf[cur][col0], xv);
        float part[8];
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
            float m[CPL];
            VecF<CPL>::ld(&Ms[(row0 + rr) * D + col0], m);
            const float vr = vs[row0 + rr];
            float s2 = 0.f;
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                m[c] = fmaf(bt, m[c], vr * ks[col0 + c]);
                s2 = fmaf(m[c], xv[c], s2);
            }
            VecF<CPL>::st(Mg + (size_t)(row0 + rr) * D + col0, m);
            part[rr] = s2;
        }
        const float orow = rows8_reduce(part, lane);
        if (owner) store_f(o + (size_t)head * D + R, invd > 0.f ? orow : 0.f);
        // every thread is done with Mbuf[buf], ks, vs, xbuf before they are reused
        fence_proxy_async_smem();
        __syncthreads();
    }
    if (!ok && tid == 0) {
        atomicExch(timeout_flag, 1);
        // let copies still in flight land before the CTA exits
        mbar_wait_bounded(&barH, 0, kDecodeWaitProbes);
        mbar_wait_bounded(&barM[0], 0, kDecodeWaitProbes);
        mbar_wait_bounded(&barM[1], 0, kDecodeWaitProbes);
    }
}

}  // namespace gka
