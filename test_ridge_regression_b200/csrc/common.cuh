// Shared device helpers of the GKA CUDA library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gka {

constexpr int kMaxSteps = 256;   // upper bound on the Chebyshev step count r

// Chebyshev parameters shared by every token of a call.  rho = 1/(1+2a) does
// not depend on the token, so the weight schedule omega_i is one table.
struct ChebParams {
    float a;                 // ridge factor: lambda = a * ||H||_F
    float half_1p2a;         // (1 + 2a) / 2: d = half_1p2a * ||H||_F is the interval centre
    int r;                   // Chebyshev steps (r - 1 matrix-vector products)
    float omega[kMaxSteps];  // omega[i], i = 1..r-1, weight of update i
};

// Lower clamp of log(beta): beta = 0 becomes exp(-150), which underflows to 0
// in every fp32 product it enters, and keeps differences of cumulative logs
// finite (no inf - inf).  Cumulative logs are summed in double so that the
// difference of two of them keeps full fp32 precision even after resets.
constexpr double kLogBetaMin = -150.0;

__device__ __forceinline__ float load_f(const float *p) { return *p; }
__device__ __forceinline__ float load_f(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

__device__ __forceinline__ void store_f(float *p, float x) { *p = x; }
__device__ __forceinline__ void store_f(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Inclusive prefix sum, in double, of clamped log(beta) over one chunk of
// C <= 256 tokens, into ell[0..C-1].  Every thread of the block must call it;
// blockDim.x >= C.  wtot: shared scratch of blockDim.x / 32 doubles.
__device__ __forceinline__ void chunk_log_prefix(const float *beta, int C, double *ell,
                                                 double *wtot) {
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    double x = 0.0;
    if (t < C) x = fmax(log((double)beta[t]), kLogBetaMin);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        double y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wtot[w] = x;  // lanes past C carry the last valid prefix
    __syncthreads();
    if (t < C) {
        double add = 0.0;
        for (int i = 0; i < w; ++i) add += wtot[i];
        ell[t] = x + add;
    }
    __syncthreads();
}

// chunk_log_prefix with log(beta) in fp32 (the cumulative sum still in double), as the
// tensor-core state pass forms its decays; beta may be in shared or global memory.
__device__ __forceinline__ void chunk_log_prefix_f32log(const float *beta, int C, double *ell,
                                                        double *wtot) {
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    double x = 0.0;
    if (t < C) x = fmax((double)logf(beta[t]), kLogBetaMin);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        double y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wtot[w] = x;
    __syncthreads();
    if (t < C) {
        double add = 0.0;
        for (int i = 0; i < w; ++i) add += wtot[i];
        ell[t] = x + add;
    }
    __syncthreads();
}

// exp of a (non-positive) difference of cumulative logs, evaluated in fp32.
__device__ __forceinline__ float decay_exp(double d) { return expf((float)d); }

}  // namespace gka
