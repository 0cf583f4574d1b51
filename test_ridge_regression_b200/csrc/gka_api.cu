// C ABI of the GKA library: argument checks, workspace layout, launches.
// The declarations and the contract of every entry point are in include/gka.h.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <type_traits>
#include <map>
#include <mutex>
#include <vector>

#include "../../include/gka.h"
#include <cudaTypedefs.h>

#include "backward_simt.cuh"
#include "adjoint_tc.cuh"
#include "backward_tc.cuh"
#include "grads_tc.cuh"
#include "chunk_simt.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "seg_tc.cuh"
#include "solve_tc.cuh"
#include "state_tc.cuh"
#include "study_simt.cuh"

namespace gka {

// Set by a kernel whose bounded wait gave up; read and cleared by
// gka_device_status().  One per device (module-scope device variable).
__device__ int g_timeout_flag = 0;

static std::atomic<int> g_last_cuda_error{0};

// ---------------------------------------------------------------------------
// Launch profiler: when enabled, every kernel launch of the library is
// bracketed by a pair of CUDA events recorded on the launch stream.  Elapsed
// times are summed per kernel when gka_profiler_read() is called.
// ---------------------------------------------------------------------------
struct ProfRecord {
    int kernel;
    cudaEvent_t start, stop;
};
static bool g_prof_on = false;
static std::vector<ProfRecord> g_prof_pending;
static std::vector<cudaEvent_t> g_prof_pool;
static std::mutex g_prof_mu;

static cudaEvent_t prof_event() {
    if (!g_prof_pool.empty()) {
        cudaEvent_t e = g_prof_pool.back();
        g_prof_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

struct ProfScope {
    int kernel;
    cudaStream_t s;
    cudaEvent_t start = nullptr;
    ProfScope(int k, cudaStream_t st) : kernel(k), s(st) {
        if (!g_prof_on) return;
        std::lock_guard<std::mutex> g(g_prof_mu);
        start = prof_event();
        if (start) cudaEventRecord(start, s);
    }
    ~ProfScope() {
        if (!start) return;
        std::lock_guard<std::mutex> g(g_prof_mu);
        cudaEvent_t stop = prof_event();
        if (!stop) return;
        cudaEventRecord(stop, s);
        g_prof_pending.push_back({kernel, start, stop});
    }
};

static int cuda_fail(cudaError_t e) {
    g_last_cuda_error.store((int)e);
    return GKA_ERR_CUDA;
}

static int check_launch() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? GKA_OK : cuda_fail(e);
}

static bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

static size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

static bool supported_d(int D) { return D == 32 || D == 64 || D == 128; }
static bool supported_c(int C) { return C == 16 || C == 32 || C == 64 || C == 128; }

// bf16 inputs, head dimension 128 and chunks of 64 or 128 tokens run the
// tensor-core solve; everything else the CUDA-core one.
static bool tensor_core_path(int D, int C, gka_dtype dt) {
    return dt == GKA_BF16 && D == 128 && (C == 64 || C == 128);
}

// On the tensor-core path the chunk states come from one sequential pass per
// (head, matrix), one CTA each on an SM of its own.  With fewer than sms / 2
// heads that leaves SMs idle, so every sequence is cut into S segments of whole
// chunks (S <= N), as many as fill the SMs with 2 * B*H * S CTAs.
static int state_segments(int BH, int N, int sms) {
    int S = BH > 0 ? sms / (2 * BH) : 1;
    if (S > N) S = N;
    return S < 1 ? 1 : S;
}

// Chebyshev constants of one call (pith.science appendix, Lemma 3: omega_0 = 2,
// omega_i = 1/(1 - rho^2 omega_{i-1}/4)); computed in double, stored in float.
static ChebParams make_cheb(float a, int r) {
    ChebParams P;
    memset(&P, 0, sizeof(P));
    P.a = a;
    P.half_1p2a = (float)((1.0 + 2.0 * (double)a) * 0.5);
    P.r = r;
    const double rho = 1.0 / (1.0 + 2.0 * (double)a);
    double w = 2.0;
    P.omega[0] = (float)w;
    for (int i = 1; i < r && i < kMaxSteps; ++i) {
        w = 1.0 / (1.0 - rho * rho * w / 4.0);
        P.omega[i] = (float)w;
    }
    return P;
}

static int layout(int B, int H, int T, int D, int C, gka_dtype dt, gka_workspace_layout *L) {
    if (B < 0 || H < 0 || T < 0) return GKA_ERR_INVALID_ARG;
    if (dt != GKA_F32 && dt != GKA_BF16) return GKA_ERR_INVALID_ARG;
    if (!supported_d(D) || !supported_c(C)) return GKA_ERR_UNSUPPORTED;
    if (T % C != 0) return GKA_ERR_T_NOT_MULTIPLE_OF_CHUNK;
    const size_t BH = (size_t)B * H, N = (size_t)(T / C);
    size_t off = 0;
    L->states_offset = off;
    off = round256(off + sizeof(float) * BH * (N + 1) * 2 * D * D);
    L->decay_offset = off;
    off = round256(off + sizeof(float) * BH * N);
    L->norms_offset = off;
    off = round256(off + sizeof(float) * BH * (size_t)T);
    L->states_lp_offset = off;
    if (tensor_core_path(D, C, dt)) {
        off = round256(off + 2 * BH * N * 2 * (size_t)D * D);   // fp16 states
        off = round256(off + sizeof(float) * BH * N * 2);       // norm-bound increments
        off = round256(off + sizeof(int) * BH * N * 2);         // state exponents
        off = round256(off + 4 * sizeof(float) * BH * (size_t)T);   // per-token decays
    }
    L->total_bytes = off;
    return GKA_OK;
}

// Opts a kernel into `bytes` of dynamic shared memory (beyond the 48 KiB
// default, which also counts the kernel's static shared memory).  Remembered
// per (kernel, device) so the attribute call happens once.
static std::mutex g_smem_mu;
static std::map<std::pair<const void *, int>, size_t> g_smem_set;

template <typename K>
static cudaError_t set_smem(K kernel, size_t bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const auto key = std::make_pair(reinterpret_cast<const void *>(kernel), dev);
    std::lock_guard<std::mutex> g(g_smem_mu);
    auto it = g_smem_set.find(key);
    if (it != g_smem_set.end() && it->second >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) g_smem_set[key] = bytes;
    return e;
}

template <typename Tin, int D>
static int forward_simt(const Tin *q, const Tin *k, const Tin *v, const float *beta,
                        const float *gate, Tin *o, int B, int H, int T, int C,
                        const ChebParams &P, float *final_state,
                        char *ws, const gka_workspace_layout &L, cudaStream_t s) {
    const int BH = B * H, N = T / C;
    float *states = reinterpret_cast<float *>(ws + L.states_offset);
    float *decay = reinterpret_cast<float *>(ws + L.decay_offset);
    float *norms = reinterpret_cast<float *>(ws + L.norms_offset);
    cudaError_t e;

    const size_t sm_delta = sizeof(float) * 3 * (size_t)C * D;
    if ((e = set_smem(k_chunk_delta<Tin, D>, sm_delta)) != cudaSuccess) return cuda_fail(e);
    { ProfScope ps(GKA_KERNEL_CHUNK_DELTA, s);
    k_chunk_delta<Tin, D><<<dim3(N, BH), kSimtThreads, sm_delta, s>>>(k, v, beta, gate, states,
                                                                        decay, nullptr, T, N, C); }
    if (int rc = check_launch()) return rc;

    const int DD2 = 2 * D * D;
    { ProfScope ps(GKA_KERNEL_STATE_SCAN, s);
    k_state_scan<<<dim3((DD2 + 1023) / 1024, BH), 256, 0, s>>>(states, decay, final_state, nullptr,
                                                             nullptr, nullptr, N, DD2, true); }
    if (int rc = check_launch()) return rc;

    const size_t sm_norm = sizeof(float) * ((size_t)D * D + (size_t)C * (D + 1));
    if ((e = set_smem(k_chunk_norm<Tin, D>, sm_norm)) != cudaSuccess) return cuda_fail(e);
    { ProfScope ps(GKA_KERNEL_CHUNK_NORM, s);
    k_chunk_norm<Tin, D><<<dim3(N, BH), kSimtThreads, sm_norm, s>>>(k, beta, gate, states, norms,
                                                                    T, N, C); }
    if (int rc = check_launch()) return rc;

    const size_t sm_solve = SolveSmem<D>::bytes(C);
    if ((e = set_smem(k_chunk_solve<Tin, D>, sm_solve)) != cudaSuccess) return cuda_fail(e);
    { ProfScope ps(GKA_KERNEL_CHUNK_SOLVE, s);
    k_chunk_solve<Tin, D><<<dim3(C / kSolveTG, N, BH), kSimtThreads, sm_solve, s>>>(
        q, k, v, beta, gate, states, norms, o, nullptr, T, N, C, P); }
    return check_launch();
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

// 2-D map over a row-major [rows][128] 16-bit array: boxes of 64 columns
// (128 bytes) x 64 rows, 128-byte swizzle (the tensor-core operand layout).
static int rows128_map(CUtensorMap *m, const void *base, uint64_t rows, CUtensorMapDataType ty,
                       uint32_t box_cols = 64, uint32_t box_rows = 64) {
    auto enc = tensor_map_encoder();
    if (!enc) return cuda_fail(cudaErrorNotSupported);
    cuuint64_t dims[2] = {128, rows};
    const uint32_t esize = ty == CU_TENSOR_MAP_DATA_TYPE_FLOAT32 ? 4 : 2;
    cuuint64_t strides[1] = {128 * esize};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = enc(m, ty, 2, const_cast<void *>(base), dims,
                     strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GKA_OK : cuda_fail(cudaErrorInvalidValue);
}

static int timeout_flag_ptr(int **ptr);

// The tensor-core forward workspace's per-token decay planes (4 x B*H*T floats: l2, b,
// beta, beta^2) for chunk C.
static float *tc_tokdec(char *ws, const gka_workspace_layout &L, int BH, int T, int C) {
    constexpr int D = 128;
    const size_t BHN2 = (size_t)BH * (T / C) * 2;
    return reinterpret_cast<float *>(ws + L.states_lp_offset + round256(2 * BHN2 * (size_t)D * D) +
                                     round256(sizeof(float) * BHN2) + round256(sizeof(int) * BHN2));
}

// States written elsewhere for the solve: fp16 chunk-start copies and their exponents, one
// every `sstride` entries (copies at chunks sstride times shorter), with the per-token decays
// already in the workspace; `pdl`: the kernel before the solve writes none of its inputs.
struct TcExternalStates {
    const __half *slp;
    const int *sexp;
    int sstride;
    bool pdl;
};

static int forward_tc(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v,
                      const float *beta, const float *gate, __nv_bfloat16 *o, int B, int H, int T, int C,
                      const ChebParams &P, float *final_state, char *ws,
                      const gka_workspace_layout &L, cudaStream_t s, float *x_out = nullptr,
                      bool solve_only = false, const TcExternalStates *ext = nullptr) {
    // x_out: write the iterates instead of o; solve_only: the chunk states in the
    // workspace are current (an earlier call on the same keys, values and decays);
    // ext (with solve_only): the states come from ext instead
    constexpr int D = 128;
    const int BH = B * H, N = T / C;
    float *states = reinterpret_cast<float *>(ws + L.states_offset);
    float *decay = reinterpret_cast<float *>(ws + L.decay_offset);
    float *norms = reinterpret_cast<float *>(ws + L.norms_offset);
    const size_t BHN2 = (size_t)BH * N * 2;
    __half *slp = reinterpret_cast<__half *>(ws + L.states_lp_offset);
    float *bound_inc = reinterpret_cast<float *>(ws + L.states_lp_offset +
                                                 round256(2 * BHN2 * (size_t)D * D));
    int *sexp = reinterpret_cast<int *>(reinterpret_cast<char *>(bound_inc) +
                                        round256(sizeof(float) * BHN2));
    // per-token decays, 4 planes of B*H*T floats: l2, b, beta, beta^2
    const size_t plane = (size_t)BH * T;
    float *tokdec = reinterpret_cast<float *>(reinterpret_cast<char *>(sexp) +
                                              round256(sizeof(int) * BHN2));
    int *flag = nullptr;
    if (int rc = timeout_flag_ptr(&flag)) return rc;
    TcMaps maps;
    if (int rc = rows128_map(&maps.k, k, (uint64_t)BH * T, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)) return rc;
    if (int rc = rows128_map(&maps.v, v, (uint64_t)BH * T, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)) return rc;
    const int sstride = ext ? ext->sstride : 1;
    if (int rc = rows128_map(&maps.state, ext ? ext->slp : slp, (uint64_t)BH * N * sstride * 2 * D,
                             CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
        return rc;
    const int *sexp_solve = ext ? ext->sexp : sexp;
    cudaError_t e;

    if (solve_only) {
        // chunk states already in the workspace
    } else {
        // One pass per (head, matrix) over the chunks; with few heads the sequences
        // are cut into S segments (aggregates on the tensor cores, then a scan of
        // the segment starts) so that S times more CTAs share the sequential pass.
        StateMaps smaps;
        smaps.k = maps.k;
        smaps.v = maps.v;
        if (int rc = rows128_map(&smaps.out, slp, (uint64_t)BH * N * 2 * D,
                                 CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 64, 128))
            return rc;
        int dev = 0, sms = 148;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail(e);
        const int S = state_segments(BH, N, sms);
        // the aggregates (one CTA per SM each) may cut the sequences K times finer
        const int K = S > 1 ? std::max(1, std::min(sms / (BH * S), N / S)) : 1;
        const int S1 = K * S;
        // segment buffers in the fp32 state region (unused by this path otherwise):
        // starts [BH][S1][2][D][D], then decays [BH][S1], increments and bounds [BH][S1][2]
        float *seg_start = states;
        float *seg_dec = seg_start + (size_t)BH * S1 * 2 * D * D;
        float *seg_inc = seg_dec + (size_t)BH * S1;
        float *seg_bound = seg_inc + (size_t)BH * S1 * 2;
        if (S > 1) {
            if ((e = set_smem(k_seg_delta_tc, SegSmem::bytes)) != cudaSuccess) return cuda_fail(e);
            { ProfScope ps(GKA_KERNEL_CHUNK_DELTA, s);
            k_seg_delta_tc<<<dim3(S1, BH), kSegThreads, SegSmem::bytes, s>>>(
                smaps, beta, gate, seg_start, seg_dec, seg_inc, T, N, C, S1, flag); }
            if (int rc = check_launch()) return rc;
            { ProfScope ps(GKA_KERNEL_STATE_SCAN, s);
            k_seg_scan<<<dim3(2 * D * D / 1024, BH), 256, 0, s>>>(seg_start, seg_dec, seg_inc,
                                                                 seg_bound, S1); }
            if (int rc = check_launch()) return rc;
        }
        if (C == 64) {
            if ((e = set_smem(k_state_pass_tc<64>, StateSmem<64>::bytes)) != cudaSuccess)
                return cuda_fail(e);
            ProfScope ps(GKA_KERNEL_STATE_PASS_TC, s);
            k_state_pass_tc<64><<<dim3(2, BH * S), kStateThreads, StateSmem<64>::bytes, s>>>(
                smaps, beta, gate, sexp, decay, tokdec, plane, final_state, T, N, S, K, seg_start,
                seg_bound, flag, 1);
        } else {
            if ((e = set_smem(k_state_pass_tc<128>, StateSmem<128>::bytes)) != cudaSuccess)
                return cuda_fail(e);
            ProfScope ps(GKA_KERNEL_STATE_PASS_TC, s);
            k_state_pass_tc<128><<<dim3(2, BH * S), kStateThreads, StateSmem<128>::bytes, s>>>(
                smaps, beta, gate, sexp, decay, tokdec, plane, final_state, T, N, S, K, seg_start,
                seg_bound, flag, 1);
        }
        if (int rc = check_launch()) return rc;
    }

    // The solve after the state pass is launched as its programmatic dependent: its
    // input loads, barriers and TMEM allocation overlap the pass, and it waits for the
    // pass (griddepcontrol.wait) before reading the state copies and decays.  With
    // solve_only the kernel before it may have written q, which the solve reads before
    // that wait, so it is launched in plain stream order unless ext says otherwise.
    auto launch_solve = [&](auto kern, size_t smem) -> cudaError_t {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(N, BH);
        cfg.blockDim = dim3(kSolveThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        // 128-token chunks: one CTA per SM, and the early CTAs gained nothing (A/B on one
        // box: 3.5577 against 3.5466 ms median on B1 H8 T131072), so plain order there
        cfg.numAttrs = (C == 64 && (!solve_only || (ext && ext->pdl))) ? 1 : 0;
        return cudaLaunchKernelEx(&cfg, kern, maps, q, gate, (const float *)tokdec, plane, norms,
                                  sexp_solve, o, x_out, T, N, C, P, flag, sstride);
    };
    if (C == 64) {
        // one CTA per 64-token chunk
        auto kern = x_out ? k_chunk_solve_tc<64, 64, true> : k_chunk_solve_tc<64, 64, false>;
        if ((e = set_smem(kern, TcSmem<64, 64>::bytes)) != cudaSuccess) return cuda_fail(e);
        ProfScope ps(GKA_KERNEL_CHUNK_SOLVE_TC, s);
        if ((e = launch_solve(kern, TcSmem<64, 64>::bytes)) != cudaSuccess) return cuda_fail(e);
    } else {
        // one CTA per 128-token chunk (N = 128 MMAs)
        auto kern = x_out ? k_chunk_solve_tc<128, 128, true> : k_chunk_solve_tc<128, 128, false>;
        if ((e = set_smem(kern, TcSmem<128, 128>::bytes)) != cudaSuccess) return cuda_fail(e);
        ProfScope ps(GKA_KERNEL_CHUNK_SOLVE_TC, s);
        if ((e = launch_solve(kern, TcSmem<128, 128>::bytes)) != cudaSuccess) return cuda_fail(e);
    }
    if (int rc = check_launch()) return rc;
    return GKA_OK;
}

template <typename Tin>
static int forward_dispatch(const void *q, const void *k, const void *v, const float *beta,
                            const float *gate, void *o, int B, int H, int T, int D, int C, const ChebParams &P,
                            float *final_state, char *ws, const gka_workspace_layout &L,
                            cudaStream_t s) {
    auto Q = static_cast<const Tin *>(q);
    auto K = static_cast<const Tin *>(k);
    auto V = static_cast<const Tin *>(v);
    auto O = static_cast<Tin *>(o);
    if constexpr (std::is_same<Tin, __nv_bfloat16>::value) {
        if (tensor_core_path(D, C, GKA_BF16))
            return forward_tc(Q, K, V, beta, gate, O, B, H, T, C, P, final_state, ws, L, s);
    }
    switch (D) {
        case 32: return forward_simt<Tin, 32>(Q, K, V, beta, gate, O, B, H, T, C, P, final_state, ws, L, s);
        case 64: return forward_simt<Tin, 64>(Q, K, V, beta, gate, O, B, H, T, C, P, final_state, ws, L, s);
        default: return forward_simt<Tin, 128>(Q, K, V, beta, gate, O, B, H, T, C, P, final_state, ws, L, s);
    }
}

// ---------------------------------------------------------------------------
// Backward pass (CUDA cores): workspace layout and launches.
// ---------------------------------------------------------------------------
static bool supported_bwd_c(int C) { return C == 16 || C == 32; }

struct BwdLayout {
    gka_workspace_layout fwd;   // the forward's regions (chunk states, decays, norms)
    size_t xs, ys, cvec, adj, rows, tokq, chq;
    // bf16, D = 128, T a multiple of 64: the forward iterates come from the tensor-core
    // forward with 64-token chunks, whose own workspace starts at tc
    bool tc_recompute;
    gka_workspace_layout tcl;
    size_t tc, u16, total;
};

static int bwd_layout(int B, int H, int T, int D, int C, gka_dtype dt, BwdLayout *L) {
    if (!supported_bwd_c(C) && supported_c(C)) return GKA_ERR_UNSUPPORTED;
    if (int rc = layout(B, H, T, D, C, dt, &L->fwd)) return rc;
    const size_t BH = (size_t)B * H, N = (size_t)(T / C), TD = BH * (size_t)T * D;
    size_t off = round256(L->fwd.total_bytes);
    L->xs = off;   off = round256(off + sizeof(float) * TD);
    L->ys = off;   off = round256(off + sizeof(float) * TD);
    L->cvec = off; off = round256(off + sizeof(float) * BH * T);
    L->adj = off;  off = round256(off + sizeof(float) * BH * (N + 1) * 2 * D * D);
    L->rows = off; off = round256(off + 4 * sizeof(float) * TD);
    // per-token scalars uk, yhx, gmx, qe (the tensor-core row kernel writes qe's H and M
    // parts as planes 3 and 4)
    L->tokq = off; off = round256(off + 5 * sizeof(float) * BH * T);
    L->chq = off;  off = round256(off + 2 * sizeof(float) * BH * N);
    L->tc_recompute = tensor_core_path(D, 64, dt) && T % 64 == 0;
    L->tc = off;
    if (L->tc_recompute) {
        if (int rc = layout(B, H, T, D, 64, dt, &L->tcl)) return rc;
        off = round256(off + L->tcl.total_bytes);
        L->u16 = off;   // u = M^T dL/do in bf16, the right-hand side of the adjoint solve
        off = round256(off + 2 * TD);
    }
    L->total = off;
    return GKA_OK;
}

template <typename Tin, int D>
static int backward_simt(const Tin *q, const Tin *k, const Tin *v, const float *beta,
                         const float *gate, const Tin *dout, Tin *dq, Tin *dk, Tin *dv,
                         float *dbeta, float *dgate, int B, int H, int T, int C,
                         const ChebParams &P, char *ws, const BwdLayout &L, cudaStream_t s) {
    const int BH = B * H, N = T / C;
    float *states = reinterpret_cast<float *>(ws + L.fwd.states_offset);
    float *decay = reinterpret_cast<float *>(ws + L.fwd.decay_offset);
    float *norms = reinterpret_cast<float *>(ws + L.fwd.norms_offset);
    float *xs = reinterpret_cast<float *>(ws + L.xs), *ys = reinterpret_cast<float *>(ws + L.ys);
    float *cvec = reinterpret_cast<float *>(ws + L.cvec), *adj = reinterpret_cast<float *>(ws + L.adj);
    float *rows = reinterpret_cast<float *>(ws + L.rows), *tokq = reinterpret_cast<float *>(ws + L.tokq);
    float *chq = reinterpret_cast<float *>(ws + L.chq);
    cudaError_t e;
    const int DD2 = 2 * D * D;

    // forward recompute: chunk states, norms and the iterates x_t (bf16, D = 128: the
    // iterates and norms from the tensor-core forward, the fp32 chunk states here)
    // bf16, D = 128, C = 32: the chunk states as fp16 copies (scaled by 2^e, the tensor
    // cores' operands) with their exponents, in the fp32 state region (twice their size),
    // which this path leaves unused otherwise
    __half *slp32 = reinterpret_cast<__half *>(states);
    int *sexp32 = reinterpret_cast<int *>(reinterpret_cast<char *>(states) +
                                          round256(sizeof(__half) * BH * (size_t)N * 2 * D * D));
    CUtensorMap state_map;   // the fp16 copies, boxes 64 x 64, for the consumers' TMA loads
    bool states_done = false;
    if constexpr (std::is_same<Tin, __nv_bfloat16>::value && D == 128) {
        if (L.tc_recompute && C == 32) {
            // the chunk states in one sequential pass per (head, matrix) on tcgen05 (no
            // increments through memory), the chunk decays, and the per-token decays of
            // 64-token groups in the tensor-core forward's workspace: the solves below read
            // these copies at every second chunk instead of a pass of their own
            int *flag = nullptr;
            if (int rc = timeout_flag_ptr(&flag)) return rc;
            StateMaps sm32;
            if (int rc = rows128_map(&sm32.k, k, (uint64_t)BH * T, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                                     64, 32))
                return rc;
            if (int rc = rows128_map(&sm32.v, v, (uint64_t)BH * T, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                                     64, 32))
                return rc;
            if (int rc = rows128_map(&sm32.out, slp32, (uint64_t)BH * N * 2 * D,
                                     CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 64, 128))
                return rc;
            if (int rc = rows128_map(&state_map, slp32, (uint64_t)BH * N * 2 * D,
                                     CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
                return rc;
            if ((e = set_smem(k_state_pass_tc<32>, StateSmem<32>::bytes)) != cudaSuccess)
                return cuda_fail(e);
            { ProfScope ps(GKA_KERNEL_STATE_PASS_TC, s);
            k_state_pass_tc<32><<<dim3(2, BH), kStateThreads, StateSmem<32>::bytes, s>>>(
                sm32, beta, gate, sexp32, decay, tc_tokdec(ws + L.tc, L.tcl, BH, T, 64),
                (size_t)BH * T, nullptr, T, N, 1, 1, nullptr, nullptr, flag, 2); }
            if (int rc = check_launch()) return rc;
            states_done = true;
        }
    }
    if (!states_done) {
        const size_t sm_delta = sizeof(float) * 3 * (size_t)C * D;
        if ((e = set_smem(k_chunk_delta<Tin, D>, sm_delta)) != cudaSuccess) return cuda_fail(e);
        { ProfScope ps(GKA_KERNEL_CHUNK_DELTA, s);
        k_chunk_delta<Tin, D><<<dim3(N, BH), kSimtThreads, sm_delta, s>>>(
            k, v, beta, gate, states, decay, nullptr, T, N, C); }
        if (int rc = check_launch()) return rc;
        { ProfScope ps(GKA_KERNEL_STATE_SCAN, s);
        k_state_scan<<<dim3((DD2 + 1023) / 1024, BH), 256, 0, s>>>(states, decay, nullptr, nullptr,
                                                                 nullptr, nullptr, N, DD2, true); }
        if (int rc = check_launch()) return rc;
    }
    const size_t sm_solve = SolveSmem<D>::bytes(C);
    bool tc_done = false;
    if constexpr (std::is_same<Tin, __nv_bfloat16>::value && D == 128) {
        if (L.tc_recompute) {
            char *tws = ws + L.tc;
            // the iterates; with the 32-token copies (the state pass just before writes none
            // of the solve's inputs: a programmatic dependent launch)
            const TcExternalStates ext{slp32, sexp32, 2, true};
            if (int rc = forward_tc(q, k, v, beta, gate, nullptr, B, H, T, 64, P, nullptr, tws,
                                    L.tcl, s, xs, states_done, states_done ? &ext : nullptr))
                return rc;
            norms = reinterpret_cast<float *>(tws + L.tcl.norms_offset);
            tc_done = true;
        }
    }
    if (!tc_done) {
        const size_t sm_norm = sizeof(float) * ((size_t)D * D + (size_t)C * (D + 1));
        if ((e = set_smem(k_chunk_norm<Tin, D>, sm_norm)) != cudaSuccess) return cuda_fail(e);
        { ProfScope ps(GKA_KERNEL_CHUNK_NORM, s);
        k_chunk_norm<Tin, D><<<dim3(N, BH), kSimtThreads, sm_norm, s>>>(k, beta, gate, states,
                                                                        norms, T, N, C); }
        if (int rc = check_launch()) return rc;
        if ((e = set_smem(k_chunk_solve<Tin, D>, sm_solve)) != cudaSuccess) return cuda_fail(e);
        { ProfScope ps(GKA_KERNEL_CHUNK_SOLVE, s);
        k_chunk_solve<Tin, D><<<dim3(C / kSolveTG, N, BH), kSimtThreads, sm_solve, s>>>(
            q, k, v, beta, gate, states, norms, nullptr, xs, T, N, C, P); }
        if (int rc = check_launch()) return rc;
    }

    // adjoint solve: dq = y, c (bf16, D = 128: u on CUDA cores, rounded to bf16, then the
    // tensor-core solve on it with the tensor-core forward's chunk states)
    Tin *u16 = tc_done ? reinterpret_cast<Tin *>(ws + L.u16) : nullptr;
    bool u_done = false;
    if constexpr (std::is_same<Tin, __nv_bfloat16>::value && D == 128) {
        if (u16 && C == kBrC) {
            // u alone, M_s^T G^T as fp16 MMAs
            int *flag = nullptr;
            if (int rc = timeout_flag_ptr(&flag)) return rc;
            if ((e = set_smem(k_bwd_u_tc, BwdUTcSmem::bytes)) != cudaSuccess) return cuda_fail(e);
            { ProfScope ps(GKA_KERNEL_BWD_SOLVE, s);
            k_bwd_u_tc<<<dim3(N, BH), kSimtThreads, BwdUTcSmem::bytes, s>>>(
                state_map, sexp32, k, v, beta, gate, dout, u16, T, N, flag); }
            u_done = true;
        }
    }
    if (!u_done) {
        // u (into u16 for the tensor-core solve, C = 16) or the whole adjoint solve
        if ((e = set_smem(k_bwd_solve<Tin, D>, sm_solve)) != cudaSuccess) return cuda_fail(e);
        { ProfScope ps(GKA_KERNEL_BWD_SOLVE, s);
        k_bwd_solve<Tin, D><<<dim3(C / kSolveTG, N, BH), kSimtThreads, sm_solve, s>>>(
            k, v, beta, gate, dout, states, norms, xs, dq, ys, cvec, u16, T, N, C, P); }
    }
    if (int rc = check_launch()) return rc;
    if constexpr (std::is_same<Tin, __nv_bfloat16>::value && D == 128) {
        if (tc_done) {
            // y on u (u was written by the kernel just before: plain stream order)
            const TcExternalStates ext{slp32, sexp32, 2, false};
            if (int rc = forward_tc(u16, k, v, beta, gate, nullptr, B, H, T, 64, P, nullptr,
                                    ws + L.tc, L.tcl, s, ys, true, states_done ? &ext : nullptr))
                return rc;
            { ProfScope ps(GKA_KERNEL_BWD_SOLVE, s);
            k_bwd_yfinish<Tin, D><<<(unsigned)(((size_t)BH * T + 7) / 8), kSimtThreads, 0, s>>>(
                ys, xs, norms, dq, cvec, (size_t)BH * T, P.a); }
            if (int rc = check_launch()) return rc;
        }
    }
    // the adjoint states: bf16, D = 128, C = 32: the increments and the reverse scan in
    // one tensor-core pass per (head, matrix), written as fp16 copies (scaled by 2^e)
    // with their exponents and inner products, in the adjoint region (half its size
    // holds the copies); otherwise per-chunk increments and a reverse scan in fp32
    __half *alp = reinterpret_cast<__half *>(adj);
    int *aexp = reinterpret_cast<int *>(reinterpret_cast<char *>(adj) +
                                        round256(sizeof(__half) * BH * (size_t)N * 2 * D * D));
    float *ehp = reinterpret_cast<float *>(reinterpret_cast<char *>(aexp) +
                                           round256(sizeof(int) * BH * (size_t)N * 2));
    bool rows_done = false;
    if constexpr (std::is_same<Tin, __nv_bfloat16>::value && D == 128) {
        if (tc_done && C == kBrC) {
            int *flag = nullptr;
            if (int rc = timeout_flag_ptr(&flag)) return rc;
            AdjMaps am;
            const uint64_t ntok = (uint64_t)BH * T;
            if (int rc = rows128_map(&am.y, ys, ntok, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 32, 32)) return rc;
            if (int rc = rows128_map(&am.x, xs, ntok, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 32, 32)) return rc;
            if (int rc = rows128_map(&am.k, k, ntok, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 64, 32)) return rc;
            if (int rc = rows128_map(&am.g, dout, ntok, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 64, 32))
                return rc;
            am.state = state_map;
            const uint64_t crows = (uint64_t)BH * N * 2 * D;
            if (int rc = rows128_map(&am.out, alp, crows, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 64, 128))
                return rc;
            CUtensorMap adj_map;   // the copies, boxes 64 x 64, for the row kernel's loads
            if (int rc = rows128_map(&adj_map, alp, crows, CU_TENSOR_MAP_DATA_TYPE_FLOAT16)) return rc;
            if ((e = set_smem(k_adjoint_pass_tc, AdjSmem::bytes)) != cudaSuccess) return cuda_fail(e);
            { ProfScope ps(GKA_KERNEL_ADJOINT_SCAN, s);
            k_adjoint_pass_tc<<<dim3(2, BH), kAdjThreads, AdjSmem::bytes, s>>>(
                am, beta, gate, cvec, sexp32, aexp, ehp, T, N, flag); }
            if (int rc = check_launch()) return rc;
            // the chunk rows against H_s, M_s and the adjoints, as fp16 MMAs
            if ((e = set_smem(k_bwd_rows_tc, BwdRowsTcSmem::bytes)) != cudaSuccess)
                return cuda_fail(e);
            { ProfScope ps(GKA_KERNEL_BWD_ROWS, s);
            k_bwd_rows_tc<<<dim3(N, BH, 2), kSimtThreads, BwdRowsTcSmem::bytes, s>>>(
                state_map, sexp32, adj_map, alp, aexp, ehp, k, v, dout, xs, ys, rows, tokq, chq,
                T, N, flag); }
            if (int rc = check_launch()) return rc;
            rows_done = true;
        }
    }
    if (!rows_done) {
        const size_t sm_bd = sizeof(float) * 5 * (size_t)C * D;
        if ((e = set_smem(k_bwd_delta<Tin, D>, sm_bd)) != cudaSuccess) return cuda_fail(e);
        { ProfScope ps(GKA_KERNEL_BWD_DELTA, s);
        k_bwd_delta<Tin, D><<<dim3(N, BH), kSimtThreads, sm_bd, s>>>(k, beta, gate, dout, states,
                                                                    xs, ys, cvec, adj, T, N, C); }
        if (int rc = check_launch()) return rc;
        { ProfScope ps(GKA_KERNEL_ADJOINT_SCAN, s);
        k_adjoint_scan<<<dim3((DD2 / 4 + 255) / 256, BH), 256, 0, s>>>(adj, decay, N, DD2); }
        if (int rc = check_launch()) return rc;
    }
    if (rows_done) {
        // the tensor-core row products ran
    } else if (C == 16) {
        constexpr size_t sm_rows = BwdRowsSmem<Tin, D, 16>::bytes;
        if ((e = set_smem(k_bwd_rows<Tin, D, 16>, sm_rows)) != cudaSuccess) return cuda_fail(e);
        ProfScope ps(GKA_KERNEL_BWD_ROWS, s);
        k_bwd_rows<Tin, D, 16><<<dim3(N, BH), kSimtThreads, sm_rows, s>>>(
            k, v, dout, states, adj, xs, ys, rows, tokq, chq, T, N);
    } else {
        constexpr size_t sm_rows = BwdRowsSmem<Tin, D, 32>::bytes;
        if ((e = set_smem(k_bwd_rows<Tin, D, 32>, sm_rows)) != cudaSuccess) return cuda_fail(e);
        ProfScope ps(GKA_KERNEL_BWD_ROWS, s);
        k_bwd_rows<Tin, D, 32><<<dim3(N, BH), kSimtThreads, sm_rows, s>>>(
            k, v, dout, states, adj, xs, ys, rows, tokq, chq, T, N);
    }
    if (int rc = check_launch()) return rc;
    // gradients
    if constexpr (std::is_same<Tin, __nv_bfloat16>::value && D == 128) {
        if (rows_done) {
            // bf16, D = 128, C = 32: the dot matrices and the row outputs as fp16 MMAs
            int *flag = nullptr;
            if (int rc = timeout_flag_ptr(&flag)) return rc;
            if ((e = set_smem(k_bwd_grads_tc, BwdGradTcSmem::bytes)) != cudaSuccess)
                return cuda_fail(e);
            { ProfScope ps(GKA_KERNEL_BWD_GRADS, s);
            k_bwd_grads_tc<<<dim3(N, BH), kSimtThreads, BwdGradTcSmem::bytes, s>>>(
                k, v, beta, gate, dout, xs, ys, cvec, rows, tokq, chq, dk, dv, dbeta, dgate, T, N,
                flag); }
            return check_launch();
        }
    }
    if (C == 16) {
        constexpr size_t sm_gr = BwdGradSmem<D, 16>::bytes;
        if ((e = set_smem(k_bwd_grads<Tin, D, 16>, sm_gr)) != cudaSuccess) return cuda_fail(e);
        ProfScope ps(GKA_KERNEL_BWD_GRADS, s);
        k_bwd_grads<Tin, D, 16><<<dim3(N, BH), kSimtThreads, sm_gr, s>>>(
            k, v, beta, gate, dout, xs, ys, cvec, rows, tokq, chq, dk, dv, dbeta, dgate, T, N);
    } else {
        constexpr size_t sm_gr = BwdGradSmem<D, 32>::bytes;
        if ((e = set_smem(k_bwd_grads<Tin, D, 32>, sm_gr)) != cudaSuccess) return cuda_fail(e);
        ProfScope ps(GKA_KERNEL_BWD_GRADS, s);
        k_bwd_grads<Tin, D, 32><<<dim3(N, BH), kSimtThreads, sm_gr, s>>>(
            k, v, beta, gate, dout, xs, ys, cvec, rows, tokq, chq, dk, dv, dbeta, dgate, T, N);
    }
    return check_launch();
}

template <typename Tin>
static int backward_dispatch(const void *q, const void *k, const void *v, const float *beta,
                             const float *gate, const void *dout, void *dq, void *dk, void *dv,
                             float *dbeta, float *dgate, int B, int H, int T, int D, int C,
                             const ChebParams &P, char *ws, const BwdLayout &L, cudaStream_t s) {
    auto in = [](const void *p) { return static_cast<const Tin *>(p); };
    auto out = [](void *p) { return static_cast<Tin *>(p); };
    switch (D) {
        case 32:
            return backward_simt<Tin, 32>(in(q), in(k), in(v), beta, gate, in(dout), out(dq), out(dk),
                                          out(dv), dbeta, dgate, B, H, T, C, P, ws, L, s);
        case 64:
            return backward_simt<Tin, 64>(in(q), in(k), in(v), beta, gate, in(dout), out(dq), out(dk),
                                          out(dv), dbeta, dgate, B, H, T, C, P, ws, L, s);
        default:
            return backward_simt<Tin, 128>(in(q), in(k), in(v), beta, gate, in(dout), out(dq),
                                           out(dk), out(dv), dbeta, dgate, B, H, T, C, P, ws, L, s);
    }
}

// ---------------------------------------------------------------------------
// Solver study: the CUDA-core chunk states and norms, then one study kernel.
// ---------------------------------------------------------------------------
template <typename Tin, int D, int SOLVER>
static int study_launch(const Tin *q, const Tin *k, const float *beta, const float *gate,
                        const float *states, const float *norms, float *resid, int BH, int T,
                        int N, int C, const ChebParams &P, cudaStream_t s) {
    const size_t smem = sizeof(float) * ((size_t)D * SolveSmem<D>::KP +
                                         (size_t)C * SolveSmem<D>::KP + (size_t)kSolveTG * D +
                                         2 * (size_t)kSolveTG * C);
    cudaError_t e = set_smem(k_solver_study<Tin, D, SOLVER>, smem);
    if (e != cudaSuccess) return cuda_fail(e);
    ProfScope ps(GKA_KERNEL_SOLVER_STUDY, s);
    k_solver_study<Tin, D, SOLVER><<<dim3(C / kSolveTG, N, BH), kSimtThreads, smem, s>>>(
        q, k, beta, gate, states, norms, resid, T, N, C, P);
    return check_launch();
}

template <typename Tin, int D>
static int study_simt(const Tin *q, const Tin *k, const float *beta, const float *gate, int B,
                      int H, int T, int C, int solver, const ChebParams &P, float *resid, char *ws,
                      const gka_workspace_layout &L, cudaStream_t s) {
    const int BH = B * H, N = T / C;
    float *states = reinterpret_cast<float *>(ws + L.states_offset);
    float *decay = reinterpret_cast<float *>(ws + L.decay_offset);
    float *norms = reinterpret_cast<float *>(ws + L.norms_offset);
    cudaError_t e;
    const size_t sm_delta = sizeof(float) * 3 * (size_t)C * D;
    if ((e = set_smem(k_chunk_delta<Tin, D>, sm_delta)) != cudaSuccess) return cuda_fail(e);
    { ProfScope ps(GKA_KERNEL_CHUNK_DELTA, s);
    k_chunk_delta<Tin, D><<<dim3(N, BH), kSimtThreads, sm_delta, s>>>(k, k, beta, gate, states,
                                                                        decay, nullptr, T, N, C); }
    if (int rc = check_launch()) return rc;
    const int DD2 = 2 * D * D;
    { ProfScope ps(GKA_KERNEL_STATE_SCAN, s);
    k_state_scan<<<dim3((DD2 + 1023) / 1024, BH), 256, 0, s>>>(states, decay, nullptr, nullptr,
                                                             nullptr, nullptr, N, DD2, true); }
    if (int rc = check_launch()) return rc;
    const size_t sm_norm = sizeof(float) * ((size_t)D * D + (size_t)C * (D + 1));
    if ((e = set_smem(k_chunk_norm<Tin, D>, sm_norm)) != cudaSuccess) return cuda_fail(e);
    { ProfScope ps(GKA_KERNEL_CHUNK_NORM, s);
    k_chunk_norm<Tin, D><<<dim3(N, BH), kSimtThreads, sm_norm, s>>>(k, beta, gate, states, norms,
                                                                    T, N, C); }
    if (int rc = check_launch()) return rc;
    switch (solver) {
        case 0: return study_launch<Tin, D, 0>(q, k, beta, gate, states, norms, resid, BH, T, N, C, P, s);
        case 1: return study_launch<Tin, D, 1>(q, k, beta, gate, states, norms, resid, BH, T, N, C, P, s);
        case 2: return study_launch<Tin, D, 2>(q, k, beta, gate, states, norms, resid, BH, T, N, C, P, s);
        default: return study_launch<Tin, D, 3>(q, k, beta, gate, states, norms, resid, BH, T, N, C, P, s);
    }
}

static int timeout_flag_ptr(int **ptr) {
    cudaError_t e = cudaGetSymbolAddress((void **)ptr, g_timeout_flag);
    return e == cudaSuccess ? GKA_OK : cuda_fail(e);
}

template <typename Tin, int D>
static int decode_launch(float *state, const void *q, const void *k, const void *v,
                         const float *beta, const float *gate, void *o, int BH, const ChebParams &P, cudaStream_t s) {
    int *flag = nullptr;
    if (int rc = timeout_flag_ptr(&flag)) return rc;
    const size_t smem = sizeof(float) * D * D;
    cudaError_t e = set_smem(k_decode_step<Tin, D>, smem);
    if (e != cudaSuccess) return cuda_fail(e);
    ProfScope ps(GKA_KERNEL_DECODE_STEP, s);
    k_decode_step<Tin, D><<<BH, 4 * D, smem, s>>>(
        state, static_cast<const Tin *>(q), static_cast<const Tin *>(k),
        static_cast<const Tin *>(v), beta, gate, static_cast<Tin *>(o), P, flag);
    return check_launch();
}


template <typename Tin>
static int decode_rows_launch(float *state, const void *q, const void *k, const void *v,
                              const float *beta, const float *gate, void *o, int BH, const ChebParams &P,
                              cudaStream_t s) {
    int *flag = nullptr;
    if (int rc = timeout_flag_ptr(&flag)) return rc;
    DecodeMaps maps;
    if (int rc = rows128_map(&maps.state, state, (uint64_t)BH * 2 * kDecD,
                             CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 32, 128))
        return rc;
    cudaError_t e = set_smem(k_decode_rows<Tin>, kDecRowSmem);
    if (e != cudaSuccess) return cuda_fail(e);
    ProfScope ps(GKA_KERNEL_DECODE_STEP, s);
    k_decode_rows<Tin><<<BH, kDecRowThreads, kDecRowSmem, s>>>(
        maps, static_cast<const Tin *>(q), static_cast<const Tin *>(k),
        static_cast<const Tin *>(v), beta, gate, static_cast<Tin *>(o), P, flag);
    return check_launch();
}

template <typename Tin>
static int decode_dispatch(float *state, const void *q, const void *k, const void *v,
                           const float *beta, const float *gate, void *o, int BH, int D, const ChebParams &P,
                           cudaStream_t s) {
    if (D == 128) return decode_rows_launch<Tin>(state, q, k, v, beta, gate, o, BH, P, s);
    switch (D) {
        case 32: return decode_launch<Tin, 32>(state, q, k, v, beta, gate, o, BH, P, s);
        case 64: return decode_launch<Tin, 64>(state, q, k, v, beta, gate, o, BH, P, s);
        default: return decode_launch<Tin, 128>(state, q, k, v, beta, gate, o, BH, P, s);
    }
}

// ---------------------------------------------------------------------------
// Library-owned scratch for gka_forward_static_scratch().  A file-scope
// device array: every GPU that loads this library holds it until the process
// exits.  Host code must not use the symbol itself as an address (in host code
// it names a host-side stand-in); it takes the device address from
// cudaGetSymbolAddress on every call, in the caller's current context, and
// passes that to the kernels.  (The address belongs to a context, not to a
// device number, so a cached copy could outlive a cudaDeviceReset or belong to
// another context of the same device.)
// ---------------------------------------------------------------------------
constexpr size_t kStaticScratchBytes = GKA_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

static int static_scratch_address(void **out) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    *out = p;
    return GKA_OK;
}

// Failure-reporting self-test: one thread waits, with a short probe limit, on an
// mbarrier phase that nothing completes; the bounded wait gives up, raises the
// device flag and the kernel returns normally (no trap, no fault, the context
// stays usable).
__global__ void k_selftest_timeout(int *timeout_flag, uint32_t probes) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (!mbar_wait_bounded(&bar, 0, probes)) atomicExch(timeout_flag, 1);
    mbar_arrive(&bar);   // complete the phase so the barrier is quiescent at exit
}

}  // namespace gka

using namespace gka;

extern "C" {

size_t gka_forward_workspace_bytes(int B, int H, int T, int D, int chunk, gka_dtype dt) {
    gka_workspace_layout L;
    return layout(B, H, T, D, chunk, dt, &L) == GKA_OK ? L.total_bytes : 0;
}

int gka_forward_workspace_layout(int B, int H, int T, int D, int chunk, gka_dtype dt,
                                 gka_workspace_layout *out) {
    if (!out) return GKA_ERR_INVALID_ARG;
    return layout(B, H, T, D, chunk, dt, out);
}

int gka_forward(const void *q, const void *k, const void *v, const float *beta, void *o, int B,
                int H, int T, int D, gka_dtype dt, float a, int r, int chunk, float *final_state,
                void *workspace, size_t workspace_bytes, void *stream) {
    return gka_forward_gated(q, k, v, beta, nullptr, o, B, H, T, D, dt, a, r, chunk, final_state,
                             workspace, workspace_bytes, stream);
}

int gka_forward_gated(const void *q, const void *k, const void *v, const float *beta,
                      const float *gate, void *o, int B, int H, int T, int D, gka_dtype dt,
                      float a, int r, int chunk, float *final_state, void *workspace,
                      size_t workspace_bytes, void *stream) {
    gka_workspace_layout L;
    if (int rc = layout(B, H, T, D, chunk, dt, &L)) return rc;
    if (!(a > 0.f) || !isfinite(a) || r < 1) return GKA_ERR_INVALID_ARG;
    if (r > kMaxSteps) return GKA_ERR_UNSUPPORTED;
    if ((size_t)B * H > 65535) return GKA_ERR_UNSUPPORTED;
    const size_t BH = (size_t)B * H;
    if (BH == 0) return GKA_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (final_state) {
            cudaError_t e = cudaMemsetAsync(final_state, 0, sizeof(float) * BH * 2 * D * D, s);
            if (e != cudaSuccess) return cuda_fail(e);
        }
        return GKA_OK;
    }
    if (!q || !k || !v || !beta || !o || !workspace) return GKA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(beta) || !aligned16(o) ||
        (gate && !aligned16(gate)) || (final_state && !aligned16(final_state)) ||
        ((uintptr_t)workspace & 255u))
        return GKA_ERR_MISALIGNED;
    if (workspace_bytes < L.total_bytes) return GKA_ERR_WORKSPACE_TOO_SMALL;
    const ChebParams P = make_cheb(a, r);
    char *ws = static_cast<char *>(workspace);
    if (dt == GKA_BF16)
        return forward_dispatch<__nv_bfloat16>(q, k, v, beta, gate, o, B, H, T, D, chunk, P,
                                               final_state, ws, L, s);
    return forward_dispatch<float>(q, k, v, beta, gate, o, B, H, T, D, chunk, P, final_state, ws,
                                   L, s);
}

// ---------------------------------------------------------------------------
// Forward from host buffers: slices of (batch, head) pairs through two device
// slots, inputs in on one internal stream, compute on the caller's stream,
// outputs out on another internal stream.
// ---------------------------------------------------------------------------
struct HostPlan {
    size_t pairs, slice, nslices;
    size_t in_elems, st_elems;      // per slot: q/k/v/o elements, final-state floats
    size_t esize;
    size_t off_q, off_k, off_v, off_o, off_beta, off_fs, off_ws, slot_bytes, total;
};

static int host_plan(int B, int H, int T, int D, int chunk, gka_dtype dt, int slice, HostPlan *hp) {
    if (slice < 0) return GKA_ERR_INVALID_ARG;
    gka_workspace_layout L;
    if (int rc = layout(B, H, T, D, chunk, dt, &L)) return rc;
    const size_t pairs = (size_t)B * H;
    size_t sl = (size_t)slice;
    // default: 24 pairs or more (one-pass chunk states), about four slices; measured
    // fastest for the B8 H8 T2048 bf16 forward (2.32 ms vs 2.37-2.49 ms for 8-32 pairs)
    if (sl == 0) sl = std::max<size_t>(24, (pairs + 3) / 4);
    sl = std::min(sl, std::max<size_t>(pairs, 1));
    if (sl > 65535) return GKA_ERR_UNSUPPORTED;
    hp->pairs = pairs;
    hp->slice = sl;
    hp->nslices = pairs ? (pairs + sl - 1) / sl : 0;
    hp->esize = dt == GKA_BF16 ? 2 : 4;
    hp->in_elems = sl * (size_t)T * D;
    hp->st_elems = sl * 2 * (size_t)D * D;
    size_t off = 0;
    hp->off_q = off; off = round256(off + hp->in_elems * hp->esize);
    hp->off_k = off; off = round256(off + hp->in_elems * hp->esize);
    hp->off_v = off; off = round256(off + hp->in_elems * hp->esize);
    hp->off_o = off; off = round256(off + hp->in_elems * hp->esize);
    hp->off_beta = off; off = round256(off + sl * (size_t)T * sizeof(float));
    hp->off_fs = off; off = round256(off + hp->st_elems * sizeof(float));
    hp->slot_bytes = off;
    hp->off_ws = 2 * off;
    gka_workspace_layout Ls;
    if (int rc = layout(1, (int)sl, T, D, chunk, dt, &Ls)) return rc;
    hp->total = hp->off_ws + Ls.total_bytes;
    return GKA_OK;
}

// Copy streams and events of one device, made once (non-blocking streams).
constexpr int kMaxDevices = 256;
struct HostPipe {
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t entry = nullptr, in_done[2] = {}, comp_done[2] = {}, out_done[2] = {};
    std::mutex mu;
    bool ready = false;
};
static HostPipe g_pipes[kMaxDevices];

static int host_pipe(HostPipe **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return GKA_ERR_UNSUPPORTED;
    HostPipe &p = g_pipes[dev];
    std::lock_guard<std::mutex> g(p.mu);
    if (!p.ready) {
        if ((e = cudaStreamCreateWithFlags(&p.h2d, cudaStreamNonBlocking)) != cudaSuccess ||
            (e = cudaStreamCreateWithFlags(&p.d2h, cudaStreamNonBlocking)) != cudaSuccess ||
            (e = cudaEventCreateWithFlags(&p.entry, cudaEventDisableTiming)) != cudaSuccess)
            return cuda_fail(e);
        for (int i = 0; i < 2; ++i)
            if ((e = cudaEventCreateWithFlags(&p.in_done[i], cudaEventDisableTiming)) != cudaSuccess ||
                (e = cudaEventCreateWithFlags(&p.comp_done[i], cudaEventDisableTiming)) != cudaSuccess ||
                (e = cudaEventCreateWithFlags(&p.out_done[i], cudaEventDisableTiming)) != cudaSuccess)
                return cuda_fail(e);
        p.ready = true;
    }
    *out = &p;
    return GKA_OK;
}

size_t gka_forward_host_workspace_bytes(int B, int H, int T, int D, int chunk, gka_dtype dt,
                                        int slice) {
    HostPlan hp;
    return host_plan(B, H, T, D, chunk, dt, slice, &hp) == GKA_OK ? hp.total : 0;
}

int gka_forward_host(const void *q, const void *k, const void *v, const float *beta, void *o,
                     int B, int H, int T, int D, gka_dtype dt, float a, int r, int chunk,
                     float *final_state, int slice, void *workspace, size_t workspace_bytes,
                     void *stream) {
    HostPlan hp;
    if (int rc = host_plan(B, H, T, D, chunk, dt, slice, &hp)) return rc;
    if (!(a > 0.f) || !isfinite(a) || r < 1) return GKA_ERR_INVALID_ARG;
    if (r > kMaxSteps) return GKA_ERR_UNSUPPORTED;
    if (hp.pairs == 0) return GKA_OK;
    if (T > 0 && (!q || !k || !v || !beta || !o)) return GKA_ERR_INVALID_ARG;
    if (!workspace) return GKA_ERR_INVALID_ARG;
    if ((uintptr_t)workspace & 255u) return GKA_ERR_MISALIGNED;
    if (workspace_bytes < hp.total) return GKA_ERR_WORKSPACE_TOO_SMALL;
    HostPipe *pp = nullptr;
    if (int rc = host_pipe(&pp)) return rc;
    std::lock_guard<std::mutex> g(pp->mu);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);
    cudaError_t e;
    // nothing of this call starts before the work already on `stream`
    if ((e = cudaEventRecord(pp->entry, s)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaStreamWaitEvent(pp->h2d, pp->entry, 0)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaStreamWaitEvent(pp->d2h, pp->entry, 0)) != cudaSuccess) return cuda_fail(e);
    const size_t io_row = (size_t)T * D * hp.esize, st_row = 2 * (size_t)D * D * sizeof(float);
    for (size_t i = 0; i < hp.nslices; ++i) {
        const int slot = (int)(i & 1);
        const size_t p0 = i * hp.slice, np = std::min(hp.slice, hp.pairs - p0);
        char *base = ws + slot * hp.slot_bytes;
        // inputs of slice i: the slot's inputs are free once slice i - 2 is computed
        if (i >= 2 && (e = cudaStreamWaitEvent(pp->h2d, pp->comp_done[slot], 0)) != cudaSuccess)
            return cuda_fail(e);
        if (T > 0) {
            const void *src[3] = {q, k, v};
            const size_t off[3] = {hp.off_q, hp.off_k, hp.off_v};
            for (int t = 0; t < 3; ++t)
                if ((e = cudaMemcpyAsync(base + off[t], static_cast<const char *>(src[t]) + p0 * io_row,
                                         np * io_row, cudaMemcpyHostToDevice, pp->h2d)) != cudaSuccess)
                    return cuda_fail(e);
            if ((e = cudaMemcpyAsync(base + hp.off_beta, beta + p0 * T, np * T * sizeof(float),
                                     cudaMemcpyHostToDevice, pp->h2d)) != cudaSuccess)
                return cuda_fail(e);
        }
        if ((e = cudaEventRecord(pp->in_done[slot], pp->h2d)) != cudaSuccess) return cuda_fail(e);
        // compute of slice i: its outputs overwrite the slot's, copied out for slice i - 2
        if ((e = cudaStreamWaitEvent(s, pp->in_done[slot], 0)) != cudaSuccess) return cuda_fail(e);
        if (i >= 2 && (e = cudaStreamWaitEvent(s, pp->out_done[slot], 0)) != cudaSuccess)
            return cuda_fail(e);
        if (int rc = gka_forward(base + hp.off_q, base + hp.off_k, base + hp.off_v,
                                 reinterpret_cast<const float *>(base + hp.off_beta),
                                 base + hp.off_o, 1, (int)np, T, D, dt, a, r, chunk,
                                 final_state ? reinterpret_cast<float *>(base + hp.off_fs) : nullptr,
                                 ws + hp.off_ws, workspace_bytes - hp.off_ws, stream))
            return rc;
        if ((e = cudaEventRecord(pp->comp_done[slot], s)) != cudaSuccess) return cuda_fail(e);
        // outputs of slice i
        if ((e = cudaStreamWaitEvent(pp->d2h, pp->comp_done[slot], 0)) != cudaSuccess)
            return cuda_fail(e);
        if (T > 0 && (e = cudaMemcpyAsync(static_cast<char *>(o) + p0 * io_row, base + hp.off_o,
                                          np * io_row, cudaMemcpyDeviceToHost, pp->d2h)) != cudaSuccess)
            return cuda_fail(e);
        if (final_state &&
            (e = cudaMemcpyAsync(reinterpret_cast<char *>(final_state) + p0 * st_row,
                                 base + hp.off_fs, np * st_row, cudaMemcpyDeviceToHost, pp->d2h)) !=
                cudaSuccess)
            return cuda_fail(e);
        if ((e = cudaEventRecord(pp->out_done[slot], pp->d2h)) != cudaSuccess) return cuda_fail(e);
    }
    // the caller's stream completes once every output is on the host
    for (int slot = 0; slot < 2 && (size_t)slot < hp.nslices; ++slot)
        if ((e = cudaStreamWaitEvent(s, pp->out_done[slot], 0)) != cudaSuccess) return cuda_fail(e);
    return GKA_OK;
}

int gka_forward_static_scratch(const void *q, const void *k, const void *v, const float *beta,
                               void *o, int B, int H, int T, int D, gka_dtype dt, float a, int r,
                               int chunk, float *final_state, void *stream) {
    gka_workspace_layout L;
    if (int rc = layout(B, H, T, D, chunk, dt, &L)) return rc;
    if (L.total_bytes > kStaticScratchBytes) return GKA_ERR_EXCEEDS_STATIC_SCRATCH;
    void *scratch = nullptr;
    if (int rc = static_scratch_address(&scratch)) return rc;
    return gka_forward(q, k, v, beta, o, B, H, T, D, dt, a, r, chunk, final_state, scratch,
                       kStaticScratchBytes, stream);
}

int gka_decode_step(float *state, const void *q, const void *k, const void *v, const float *beta,
                    void *o, int B, int H, int D, gka_dtype dt, float a, int r, void *stream) {
    return gka_decode_step_gated(state, q, k, v, beta, nullptr, o, B, H, D, dt, a, r, stream);
}

int gka_decode_step_gated(float *state, const void *q, const void *k, const void *v,
                          const float *beta, const float *gate, void *o, int B, int H, int D,
                          gka_dtype dt, float a, int r, void *stream) {
    if (B < 0 || H < 0) return GKA_ERR_INVALID_ARG;
    if (dt != GKA_F32 && dt != GKA_BF16) return GKA_ERR_INVALID_ARG;
    if (!supported_d(D)) return GKA_ERR_UNSUPPORTED;
    if (!(a > 0.f) || !isfinite(a) || r < 1) return GKA_ERR_INVALID_ARG;
    if (r > kMaxSteps) return GKA_ERR_UNSUPPORTED;
    const size_t BH = (size_t)B * H;
    if (BH == 0) return GKA_OK;
    if (BH > 0x7fffffffu) return GKA_ERR_UNSUPPORTED;
    if (!state || !q || !k || !v || !beta || !o) return GKA_ERR_INVALID_ARG;
    if (!aligned16(state) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(beta) ||
        !aligned16(o) || (gate && !aligned16(gate)))
        return GKA_ERR_MISALIGNED;
    const ChebParams P = make_cheb(a, r);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dt == GKA_BF16)
        return decode_dispatch<__nv_bfloat16>(state, q, k, v, beta, gate, o, (int)BH, D, P, s);
    return decode_dispatch<float>(state, q, k, v, beta, gate, o, (int)BH, D, P, s);
}

size_t gka_backward_workspace_bytes(int B, int H, int T, int D, int chunk, gka_dtype dt) {
    BwdLayout L;
    return bwd_layout(B, H, T, D, chunk, dt, &L) == GKA_OK ? L.total : 0;
}

int gka_backward(const void *q, const void *k, const void *v, const float *beta, const float *gate,
                 const void *dout, void *dq, void *dk, void *dv, float *dbeta, float *dgate, int B,
                 int H, int T, int D, gka_dtype dt, float a, int r, int chunk, void *workspace,
                 size_t workspace_bytes, void *stream) {
    BwdLayout L;
    if (int rc = bwd_layout(B, H, T, D, chunk, dt, &L)) return rc;
    if (!(a > 0.f) || !isfinite(a) || r < 1) return GKA_ERR_INVALID_ARG;
    if (r > kMaxSteps) return GKA_ERR_UNSUPPORTED;
    if ((size_t)B * H > 65535) return GKA_ERR_UNSUPPORTED;
    if ((dgate != nullptr) != (gate != nullptr)) return GKA_ERR_INVALID_ARG;
    if ((size_t)B * H == 0 || T == 0) return GKA_OK;
    if (!q || !k || !v || !beta || !dout || !dq || !dk || !dv || !dbeta || !workspace)
        return GKA_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, beta, gate, dout, dq, dk, dv, dbeta, dgate};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GKA_ERR_MISALIGNED;
    if ((uintptr_t)workspace & 255u) return GKA_ERR_MISALIGNED;
    if (workspace_bytes < L.total) return GKA_ERR_WORKSPACE_TOO_SMALL;
    const ChebParams P = make_cheb(a, r);
    char *ws = static_cast<char *>(workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dt == GKA_BF16)
        return backward_dispatch<__nv_bfloat16>(q, k, v, beta, gate, dout, dq, dk, dv, dbeta, dgate,
                                                B, H, T, D, chunk, P, ws, L, s);
    return backward_dispatch<float>(q, k, v, beta, gate, dout, dq, dk, dv, dbeta, dgate, B, H, T, D,
                                    chunk, P, ws, L, s);
}

size_t gka_solver_study_workspace_bytes(int B, int H, int T, int D, int chunk, gka_dtype dt) {
    if (chunk == 128) return 0;
    gka_workspace_layout L;
    return layout(B, H, T, D, chunk, dt, &L) == GKA_OK ? L.total_bytes : 0;
}

int gka_solver_study(const void *q, const void *k, const float *beta, const float *gate, int B,
                     int H, int T, int D, gka_dtype dt, float a, int r, int chunk, int solver,
                     float *resid, void *workspace, size_t workspace_bytes, void *stream) {
    gka_workspace_layout L;
    if (int rc = layout(B, H, T, D, chunk, dt, &L)) return rc;
    if (chunk == 128) return GKA_ERR_UNSUPPORTED;   // the study's C x D tiles stop at 64
    if (!(a > 0.f) || !isfinite(a) || r < 1 || solver < 0 || solver > 3) return GKA_ERR_INVALID_ARG;
    if (r > kMaxSteps) return GKA_ERR_UNSUPPORTED;
    if ((size_t)B * H > 65535) return GKA_ERR_UNSUPPORTED;
    if ((size_t)B * H == 0 || T == 0) return GKA_OK;
    if (!q || !k || !beta || !resid || !workspace) return GKA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(beta) || (gate && !aligned16(gate)) ||
        !aligned16(resid) || ((uintptr_t)workspace & 255u))
        return GKA_ERR_MISALIGNED;
    if (workspace_bytes < L.total_bytes) return GKA_ERR_WORKSPACE_TOO_SMALL;
    const ChebParams P = make_cheb(a, r);
    char *ws = static_cast<char *>(workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto run = [&](auto tag) -> int {
        using Tin = decltype(tag);
        auto Q = static_cast<const Tin *>(q);
        auto K = static_cast<const Tin *>(k);
        switch (D) {
            case 32: return study_simt<Tin, 32>(Q, K, beta, gate, B, H, T, chunk, solver, P, resid, ws, L, s);
            case 64: return study_simt<Tin, 64>(Q, K, beta, gate, B, H, T, chunk, solver, P, resid, ws, L, s);
            default: return study_simt<Tin, 128>(Q, K, beta, gate, B, H, T, chunk, solver, P, resid, ws, L, s);
        }
    };
    return dt == GKA_BF16 ? run(__nv_bfloat16()) : run(float());
}

int gka_selftest_timeout(void *stream) {
    int *flag = nullptr;
    if (int rc = timeout_flag_ptr(&flag)) return rc;
    k_selftest_timeout<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(flag, 1u << 12);
    return check_launch();
}

int gka_device_status(void *stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e);
    int flag = 0;
    e = cudaMemcpyFromSymbol(&flag, g_timeout_flag, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e);
    if (flag) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_timeout_flag, &zero, sizeof(int));
        if (e != cudaSuccess) return cuda_fail(e);
        return GKA_ERR_DEVICE_TIMEOUT;
    }
    return GKA_OK;
}

int gka_last_cuda_error(void) { return g_last_cuda_error.load(); }

const char *gka_status_string(int status) {
    switch (status) {
        case GKA_OK: return "ok";
        case GKA_ERR_INVALID_ARG: return "invalid argument";
        case GKA_ERR_UNSUPPORTED: return "unsupported size or parameter";
        case GKA_ERR_T_NOT_MULTIPLE_OF_CHUNK: return "T is not a multiple of chunk";
        case GKA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case GKA_ERR_CUDA: return "CUDA error";
        case GKA_ERR_DEVICE_TIMEOUT: return "a bounded device wait timed out";
        case GKA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case GKA_ERR_EXCEEDS_STATIC_SCRATCH:
            return "problem needs more scratch than the library's static array holds";
        default: return "unknown status";
    }
}

int gka_version(void) { return 110; }

int gka_profiler_enable(int on) {
    std::lock_guard<std::mutex> g(g_prof_mu);
    g_prof_on = on != 0;
    return GKA_OK;
}

int gka_profiler_read(gka_kernel_times *out) {
    if (!out) return GKA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(g_prof_mu);
    memset(out, 0, sizeof(*out));
    int rc = GKA_OK;
    for (const ProfRecord &p : g_prof_pending) {
        float ms = 0.f;
        cudaError_t e = cudaEventSynchronize(p.stop);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, p.start, p.stop);
        if (e != cudaSuccess) rc = cuda_fail(e);
        if (p.kernel >= 0 && p.kernel < GKA_KERNEL_COUNT) {
            out->ms[p.kernel] += ms;
            out->launches[p.kernel] += 1;
        }
        g_prof_pool.push_back(p.start);
        g_prof_pool.push_back(p.stop);
    }
    g_prof_pending.clear();
    return rc;
}

}  // extern "C"
