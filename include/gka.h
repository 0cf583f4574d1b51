/*
 * gka.h - C ABI of the Gated KalmaNet (GKA) layer library for NVIDIA B200
 * (sm_100a).
 *
 * The layer ("Gated KalmaNet: A Fading Memory Layer Through Test-Time Ridge
 * Regression", arXiv 2511.21016; ai.info page, Key Contributions 2-3 and
 * Methodology in Plain English) keeps, per (batch, head) and per token t,
 *     H_t = beta_t H_{t-1} + k_t k_t^T         (gated fading Gram state)
 *     M_t = beta_t M_{t-1} + v_t k_t^T         (value state, the paper's U_t)
 * sets the adaptive ridge lambda_t = a ||H_t||_F (condition number at most
 * (a+1)/a), approximately solves (H_t + lambda_t I) x_t = q_t with r steps of
 * the Chebyshev iteration on the interval [a ||H_t||_F, (1+a) ||H_t||_F]
 * started from x = 0, and emits o_t = M_t x_t.  The Chebyshev weights follow
 * the schedule of the pith.science appendix (Lemma 3): omega_0 = 2,
 * omega_i = 1/(1 - rho^2 omega_{i-1}/4), rho = 1/(1+2a).
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library allocates no device memory and frees nothing.  Every call is
 *     asynchronous on `stream` (a cudaStream_t passed as void*; NULL = the
 *     legacy default stream).  Buffers must stay alive until the stream has
 *     run the call.
 *   - Layouts are dense row-major: q, k, v, o are [B, H, T, D] with D
 *     fastest; beta is [B, H, T] fp32.  States are fp32 [B, H, 2, D, D]:
 *     H then M, each row-major (M maps keys to values: o = M x).
 *   - Every tensor pointer must be 16-byte aligned.
 *   - Return value: GKA_OK (0) or a negative gka_status.  On an error no
 *     kernel has been launched and no output has been written, except for
 *     GKA_ERR_CUDA, which reports a failed launch (the CUDA error code is
 *     kept for gka_last_cuda_error()).
 *   - Supported: D in {32, 64, 128}; chunk in {16, 32, 64, 128}; 1 <= r <= 256;
 *     a > 0 and finite.  bf16 with D = 128 and chunk 64 or 128 runs the
 *     Chebyshev solve and readout on the tensor cores (tcgen05, TMEM
 *     accumulators, TMA-fed fp16 operands with per-tile or per-token scales, fp32
 *     accumulation and fp32 Chebyshev updates); every other case runs them on
 *     CUDA cores in fp32.
 */
#ifndef GKA_H
#define GKA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { GKA_F32 = 0, GKA_BF16 = 1 } gka_dtype;

typedef enum {
    GKA_OK = 0,
    GKA_ERR_INVALID_ARG = -1,            /* null pointer, negative size, a <= 0, r < 1 ... */
    GKA_ERR_UNSUPPORTED = -2,            /* D, chunk or r outside the supported set */
    GKA_ERR_T_NOT_MULTIPLE_OF_CHUNK = -3,/* the chunk-wise form needs N = T / chunk chunks */
    GKA_ERR_WORKSPACE_TOO_SMALL = -4,
    GKA_ERR_CUDA = -5,                   /* a CUDA call failed; see gka_last_cuda_error() */
    GKA_ERR_DEVICE_TIMEOUT = -6,         /* a bounded device-side wait gave up */
    GKA_ERR_MISALIGNED = -7,             /* a pointer is not 16-byte aligned */
    GKA_ERR_EXCEEDS_STATIC_SCRATCH = -8  /* gka_forward_static_scratch: problem too large */
} gka_status;

/* Byte offsets of the regions of the gka_forward workspace (diagnostics and
 * tests read the intermediate results through this).  Every offset is a
 * multiple of 256. */
typedef struct {
    size_t states_offset;   /* fp32 [B, H, N+1, 2, D, D]: H_s, M_s in force before chunk n;
                               slot N holds the state after the last token.  On the
                               tensor-core path slots 1..N keep the per-chunk increments
                               instead and the states live in the fp16 region below */
    size_t decay_offset;    /* fp32 [B, H, N]: product of beta over chunk n */
    size_t norms_offset;    /* fp32 [B, H, T]: ||H_t||_F as used by the solve */
    size_t states_lp_offset;   /* tensor-core path only (0 bytes otherwise): fp16
                                  [B, H, N, 2, D, D] copies of the chunk-start states, each
                                  scaled by a power of two, then the scales, then four fp32
                                  [B, H, T] planes of per-token decays (log2 of the
                                  chunk-relative cumulative decay, its exp, beta, beta^2);
                                  the region ends at total_bytes */
    size_t total_bytes;
} gka_workspace_layout;

/* Workspace bytes gka_forward needs for this problem (0 on invalid sizes). */
size_t gka_forward_workspace_bytes(int B, int H, int T, int D, int chunk, gka_dtype dt);

/* Fills *out with the workspace layout for this problem.  Returns a gka_status. */
int gka_forward_workspace_layout(int B, int H, int T, int D, int chunk, gka_dtype dt,
                                 gka_workspace_layout *out);

/*
 * Chunk-wise GKA forward (ai.info page, Key Contributions 3 and Methodology:
 * the sequence is cut into N = T / chunk chunks; only each chunk's start
 * state is computed sequentially; ||H_t||_F comes from a closed form through
 * the Gram matrix of the keys; everything within a chunk runs in parallel).
 * Steps, each a kernel on `stream`:
 *   1. chunk-state scan: H_s, M_s before every chunk, into workspace;
 *   2. per-token ||H_t||_F, into workspace;
 *   3. r-step Chebyshev solve for every token and 4. the readout o_t = M_t x_t
 *      (on the tensor-core path 2-4 are one kernel).
 * The result does not depend on `chunk` beyond floating-point rounding.
 *
 *   q, k, v     [B, H, T, D] in `dt` (fp32 or bf16); k and q are used as given
 *               (callers l2-normalise them, as the GKA block does)
 *   beta        [B, H, T] fp32 in [0, 1]: decay of the previous state
 *   o           [B, H, T, D] in `dt` (written)
 *   a, r        ridge factor (> 0) and Chebyshev steps (r - 1 matrix-vector
 *               products per token)
 *   chunk       chunk length C; T must be a multiple of it
 *   final_state nullable fp32 [B, H, 2, D, D]: state after the last token
 *               (written), e.g. to continue with gka_decode_step
 *   workspace   device scratch of at least gka_forward_workspace_bytes()
 *               bytes, 256-byte aligned; contents on entry are ignored
 */
int gka_forward(const void *q, const void *k, const void *v, const float *beta, void *o,
                int B, int H, int T, int D, gka_dtype dt, float a, int r, int chunk,
                float *final_state, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Write-gated forward: the paper's beta_t-augmented variant (ai.info page,
 * Main Findings, "The beta_t-augmented variant", and Future Directions: a
 * learned per-token input-selectivity gate in [0, 1] scales the token's write
 * into both states).  With the gate named g_t (beta_t names the decay here):
 *     H_t = beta_t H_{t-1} + g_t k_t k_t^T,   M_t = beta_t M_{t-1} + g_t v_t k_t^T,
 * and everything else as in gka_forward (lambda_t = a ||H_t||_F, the same
 * Chebyshev solve, o_t = M_t x_t).
 *   gate   nullable fp32 [B, H, T], values in [0, 1], 16-byte aligned; NULL
 *          means g_t = 1 for every token, and the call is then exactly
 *          gka_forward (same kernels, same results bit for bit)
 * Every other argument, the workspace size and the error behaviour are those
 * of gka_forward.  The kernels fold g_i into the weight of token i's write
 * (the chunk increments, the decode update) or scale token i's key and value
 * rows by sqrt(g_i) where both sides of a product read the same row (the
 * per-token norm, the solve and the readout); the two are equal in exact
 * arithmetic.
 */
int gka_forward_gated(const void *q, const void *k, const void *v, const float *beta,
                      const float *gate, void *o, int B, int H, int T, int D, gka_dtype dt,
                      float a, int r, int chunk, float *final_state, void *workspace,
                      size_t workspace_bytes, void *stream);

/*
 * gka_forward from HOST buffers, with the copies overlapped with the compute
 * (no counterpart in the paper: a transfer pipeline around the forward).
 * The B*H independent sequences, flattened to pairs p = b*H + h, are cut into
 * slices of `slice` pairs (the last may be shorter); slice i's inputs are
 * copied in on one internal stream while slice i-1 is computed on `stream`
 * and slice i-2's output is copied out on another, through two device slots.
 *
 *   q, k, v, beta, o, final_state   HOST pointers, layouts as for gka_forward
 *               (final_state nullable).  Page-locked (pinned) memory is needed
 *               for the copies to overlap; pageable memory works but serialises.
 *   slice       pairs per slice; 0 picks one (about a quarter of B*H, at
 *               least 24 pairs; the first slice's copy in and the last one's
 *               compute and copy out are not overlapped)
 *   workspace   device scratch of at least gka_forward_host_workspace_bytes()
 *               bytes, 256-byte aligned: two slots of device inputs and outputs
 *               plus one gka_forward workspace of a slice
 * Asynchronous with respect to the host: o and final_state are complete when
 * `stream` has completed the work enqueued before the call returns.  Work
 * already on `stream` finishes before any slot is reused.  Calls from several
 * host threads are serialised while they enqueue; calls that overlap on the
 * GPU must not share a workspace.
 */
size_t gka_forward_host_workspace_bytes(int B, int H, int T, int D, int chunk, gka_dtype dt,
                                        int slice);
int gka_forward_host(const void *q, const void *k, const void *v, const float *beta, void *o,
                     int B, int H, int T, int D, gka_dtype dt, float a, int r, int chunk,
                     float *final_state, int slice, void *workspace, size_t workspace_bytes,
                     void *stream);

/*
 * gka_forward without a caller-provided workspace.  There is no counterpart
 * of this call in the paper: it exists for callers that cannot allocate
 * device memory themselves, for example a plugin or extension run inside a
 * host application that owns every device allocation and hands it only its
 * input and output buffers, or a latency-critical caller that cannot accept
 * the implicit device synchronisation of cudaMalloc/cudaFree.
 *
 * The scratch comes from one device array of GKA_STATIC_SCRATCH_BYTES
 * (64 MiB) inside the library; every GPU that loads the library holds it
 * until the process exits.  This call allocates nothing: no cudaMalloc, no
 * cudaFree, no allocating library routine.  Arguments, layouts and results
 * are those of gka_forward; the caller still passes q, k, v, beta, o and the
 * optional final_state.
 *   - Problems whose gka_forward_workspace_bytes() exceeds
 *     GKA_STATIC_SCRATCH_BYTES are rejected with
 *     GKA_ERR_EXCEEDS_STATIC_SCRATCH before anything is launched.
 *   - Every call looks up the array's device address in the calling
 *     thread's current context (cudaGetSymbolAddress), so a context reset or
 *     a second context on the same device gets its own copy of the array.
 *     The first call on a device also sets the kernels' shared-memory
 *     attributes for that device; make that first call before any stream
 *     capture.
 *   - All calls share the one array, and it keeps the contents of the last
 *     call.  Nothing in it has to start at zero (every region is written
 *     before it is read), so no clearing is needed.  Calls whose execution
 *     overlaps on the GPU (on different streams, or from several host
 *     threads) race on the array and corrupt each other's results: serialise
 *     them on one stream.
 */
#define GKA_STATIC_SCRATCH_BYTES ((size_t)64 << 20)

int gka_forward_static_scratch(const void *q, const void *k, const void *v, const float *beta,
                               void *o, int B, int H, int T, int D, gka_dtype dt, float a, int r,
                               int chunk, float *final_state, void *stream);

/*
 * One recurrent decode step for B*H heads (ai.info page, Key Contributions 4:
 * the recurrent form used for inference), in place on the fp32 state:
 *   H <- beta H + k k^T;  n = ||H||_F;  x = r-step Chebyshev for
 *   (H + a n I) x = q on [a n, (1+a) n];  M <- beta M + v k^T;  o = M x.
 *   state  fp32 [B, H, 2, D, D] (read and written)
 *   q, k, v, o  [B, H, D] in `dt`;  beta [B, H] fp32.
 * A head whose H is all zero after the update gets o = 0.
 */
int gka_decode_step(float *state, const void *q, const void *k, const void *v,
                    const float *beta, void *o, int B, int H, int D, gka_dtype dt,
                    float a, int r, void *stream);

/*
 * Write-gated decode step (the recurrent form of gka_forward_gated):
 *   H <- beta H + g k k^T;  M <- beta M + g v k^T;  the rest as gka_decode_step.
 *   gate   nullable fp32 [B, H] in [0, 1], 16-byte aligned (NULL: g = 1, exactly
 *          gka_decode_step).
 */
int gka_decode_step_gated(float *state, const void *q, const void *k, const void *v,
                          const float *beta, const float *gate, void *o, int B, int H, int D,
                          gka_dtype dt, float a, int r, void *stream);

/*
 * Backward pass of gka_forward / gka_forward_gated by implicit
 * differentiation (ai.info page, Key Contributions 3 and Methodology: the
 * backward differentiates through the linear system that the Chebyshev
 * iteration approximately solves and reuses the iteration on the upstream
 * gradient; Main Findings: Lemma 2, dq_t = dq^_t, and the full intra-chunk
 * interaction of the backward; pith.science appendix, Eq. 50).  With x_t the
 * forward's r-step iterate, g_t = dL/do_t and A_t = H_t + a ||H_t||_F I:
 *   y_t = r-step Chebyshev for A_t y = M_t^T g_t,   dq_t = y_t,
 *   dL/dH_t = -y_t x_t^T - a (y_t . x_t) / ||H_t||_F H_t,   dL/dM_t = g_t x_t^T,
 * carried back through the decayed, write-gated recurrence to dk, dv, dbeta
 * and dgate.  It recomputes the forward quantities it needs (chunk states,
 * norms, iterates) itself.  With bf16 inputs, D = 128, chunk 32 and T a
 * multiple of 64 every product runs on the tensor cores (fp16 operands with
 * power-of-two scales, fp32 accumulation, fp32 sums and recurrences): one
 * chunk-state pass, both Chebyshev solves, u = M_t^T g_t, the adjoint states
 * (increments and reverse scan in one pass per head), the row products and
 * the gradients' intra-chunk products; otherwise every step runs on CUDA
 * cores in fp32.
 *   q, k, v, beta, gate  the forward's inputs (gate nullable)
 *   dout        [B, H, T, D] in `dt`: dL/do
 *   dq, dk, dv  [B, H, T, D] in `dt` (written)
 *   dbeta       [B, H, T] fp32 (written)
 *   dgate       [B, H, T] fp32 (written); non-NULL exactly when gate is
 *   chunk       16 or 32 (the backward's own chunking; the result does not
 *               depend on it beyond rounding); T must be a multiple of it
 *   workspace   at least gka_backward_workspace_bytes(), 256-byte aligned
 * A token whose H_t is zero (zero keys) has x_t = 0 and passes no gradient.
 * Errors as for gka_forward; GKA_ERR_UNSUPPORTED for chunk 64 or 128,
 * GKA_ERR_INVALID_ARG when exactly one of gate and dgate is NULL.
 */
size_t gka_backward_workspace_bytes(int B, int H, int T, int D, int chunk, gka_dtype dt);
int gka_backward(const void *q, const void *k, const void *v, const float *beta,
                 const float *gate, const void *dout, void *dq, void *dk, void *dv,
                 float *dbeta, float *dgate, int B, int H, int T, int D, gka_dtype dt,
                 float a, int r, int chunk, void *workspace, size_t workspace_bytes,
                 void *stream);

/*
 * Solver study (ai.info page, Key Contributions 2 and Main Findings: the
 * layer's Chebyshev iteration compared with gradient descent, accelerated
 * gradient descent and conjugate gradient; pith.science page, Fig. 1a and
 * Fig. 8: residual norms per iteration, for several regularisation
 * strengths).  For every token t, the system A_t x = q_t of the layer
 * (A_t = H_t + a ||H_t||_F I, spectrum in [mu, L] = [a, 1 + a] ||H_t||_F) is
 * solved from x_0 = 0 by
 *   solver 0  Chebyshev (the layer's iteration)
 *   solver 1  gradient descent, step 2 / (L + mu)
 *   solver 2  Nesterov's method for strongly convex quadratics, step 1 / L,
 *             momentum (sqrt(kappa) - 1) / (sqrt(kappa) + 1), kappa = L / mu
 *   solver 3  conjugate gradient (Hestenes-Stiefel)
 * and resid[t][i] = ||q_t - A_t x_i|| / ||q_t|| is written for i = 0..r (the
 * true residual of each iterate, fp32 arithmetic on CUDA cores); zero for a
 * token with H_t = 0 or q_t = 0.
 *   q, k, beta, gate  as for gka_forward_gated (gate nullable); v is not needed
 *   chunk       16, 32 or 64 (the chunk form of the products A x)
 *   resid       fp32 [B, H, T, r + 1] (written)
 *   workspace   at least gka_solver_study_workspace_bytes() bytes, 256-byte aligned
 * Errors as for gka_forward; GKA_ERR_INVALID_ARG for a solver outside 0..3,
 * GKA_ERR_UNSUPPORTED for chunk 128.
 */
size_t gka_solver_study_workspace_bytes(int B, int H, int T, int D, int chunk, gka_dtype dt);
int gka_solver_study(const void *q, const void *k, const float *beta, const float *gate, int B,
                     int H, int T, int D, gka_dtype dt, float a, int r, int chunk, int solver,
                     float *resid, void *workspace, size_t workspace_bytes, void *stream);

/* Synchronises `stream`, then returns GKA_ERR_DEVICE_TIMEOUT if any kernel of
 * this library on the current device gave up a bounded wait since the last
 * call (and clears the flag), GKA_ERR_CUDA if the stream reports an error,
 * else GKA_OK. */
int gka_device_status(void *stream);

/* Failure-reporting self-test (no counterpart in the paper): launches one
 * thread that waits, with a short bound, on a barrier nothing completes, so
 * the bounded wait gives up and raises the device flag exactly as a stuck
 * kernel of this library would.  The following gka_device_status() then
 * returns GKA_ERR_DEVICE_TIMEOUT (and clears the flag); the context stays
 * usable.  Returns a gka_status for the launch. */
int gka_selftest_timeout(void *stream);

/* CUDA error code (cudaError_t) behind the last GKA_ERR_CUDA, 0 if none. */
int gka_last_cuda_error(void);

/* Static text for a gka_status value. */
const char *gka_status_string(int status);

/* Library ABI version: 100 * major + minor. */
int gka_version(void);

/* Launch profiler.  Kernels of the library, by index into gka_kernel_times. */
enum {
    GKA_KERNEL_CHUNK_DELTA = 0,   /* chunk-state increments (scan step 1a); with few heads on the
                                     tensor-core path, the segment aggregates */
    GKA_KERNEL_STATE_SCAN = 1,    /* sequential state scan over chunks (step 1b); with few heads
                                     on the tensor-core path, the scan of the segment starts */
    GKA_KERNEL_CHUNK_NORM = 2,    /* per-token ||H_t||_F */
    GKA_KERNEL_CHUNK_SOLVE = 3,   /* Chebyshev solve + readout */
    GKA_KERNEL_DECODE_STEP = 4,   /* recurrent decode step */
    GKA_KERNEL_CHUNK_SOLVE_TC = 5,/* Chebyshev solve + readout on tensor cores (tcgen05) */
    GKA_KERNEL_STATE_PASS_TC = 6, /* chunk-state increments and scan in one pass (tcgen05) */
    GKA_KERNEL_BWD_SOLVE = 7,     /* backward: u = M^T dL/do and the Chebyshev solve for dq
                                     (tensor-core path: u and dq's finish; the solve itself
                                     counts as GKA_KERNEL_CHUNK_SOLVE_TC) */
    GKA_KERNEL_BWD_DELTA = 8,     /* backward, CUDA-core path: per-chunk increments of the
                                     adjoint state */
    GKA_KERNEL_ADJOINT_SCAN = 9,  /* backward: adjoint states, last chunk first (tensor-core
                                     path: increments and scan in one pass per head) */
    GKA_KERNEL_BWD_ROWS = 10,     /* backward: chunk rows against H_s, M_s and the adjoints */
    GKA_KERNEL_BWD_GRADS = 11,    /* backward: dk, dv, dbeta, dgate of each chunk */
    GKA_KERNEL_SOLVER_STUDY = 12, /* solver study: residual histories */
    GKA_KERNEL_COUNT = 16
};

typedef struct {
    double ms[GKA_KERNEL_COUNT];  /* summed device time per kernel */
    int launches[GKA_KERNEL_COUNT];
} gka_kernel_times;

/* While enabled (on != 0), every kernel launch is bracketed by two CUDA
 * events recorded on its stream (host-side bookkeeping; no device memory).
 * Not thread-safe against concurrent launches from several host threads
 * beyond a mutex around the bookkeeping. */
int gka_profiler_enable(int on);

/* Waits for the recorded events, fills *out with the per-kernel sums since
 * the last read, and forgets them. */
int gka_profiler_read(gka_kernel_times *out);

#ifdef __cplusplus
}
#endif

#endif /* GKA_H */
