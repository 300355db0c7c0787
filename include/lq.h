/*
 * lq.h -- C ABI of the B200 (sm_100a) LoopQ-style quantized looped linear.
 *
 * One quantized shared linear is applied at every loop t of a depth-recurrent
 * transformer.  At each call a token row x (length K) is
 *   1. rotated by a Kronecker transform, x~ = x (P1 kron P2), P1 a x a,
 *      P2 b x b, K = a*b ("paper_specification.yaml" of the LoopQ
 *      reproduction: loopq_components.shared_transformed_backbone, Section 2
 *      Eqs. (2)-(3); implementation_status.lq3, shared Kronecker transform);
 *   2. split into groups of 32 consecutive elements along K, each with the
 *      step s = fl32(fl32(c * absmax) / q_max), where c = c_{t,l} is the
 *      per-module, per-loop LAS clip (loopq_components.las, Section 4.1;
 *      implementation_status.lq2, clip scalars on dynamic token/group absmax
 *      scales; lq1_quantization.granularity, group size 32);
 *   3. quantized by symmetric round-to-nearest (ties to even):
 *      q = clip(rne(fl32(x~ / s)), -q_max, q_max), q_max = 7 (4-bit) or 127
 *      (8-bit), q = 0 where s = 0 (lq1_quantization.equation, Section 2
 *      Eq. (4): Q_a(x; c) = c clip(round(x / c), q_min, q_max); Section 5.1
 *      RTN; the bounds, tie rule and scale estimator are the paper's
 *      underspecified items, read as stated here);
 *   4. multiplied with group-32 4-bit weight codes:
 *      y[m,n] = sum_g s_a[m,g] s_w[n,g] sum_{k in g} q_a[m,k] q_w[n,k].
 * Weights are folded offline, W~ = W (P1^-T kron P2^-T) (inverse-transpose
 * folding, implementation_status.lq3), and quantized with s_w = fl32(absmax/7).
 *
 * Conventions for every entry point:
 *   - Pointers named d_* are CUDA device pointers of the current device;
 *     h_* are host pointers.  `stream` is a cudaStream_t (NULL = legacy
 *     default stream).  Work is enqueued on `stream` and the call returns
 *     without synchronising, unless stated otherwise.
 *   - Matrices are dense row-major with no padding between rows.
 *   - Inputs are never modified.  The caller owns every buffer it passes.
 *   - Every call returns an lq_status; no call aborts or throws.  On error
 *     nothing has been enqueued and lq_last_error() (thread-local) holds a
 *     one-line message.
 *   - Inputs must be finite; results for NaN/Inf inputs are unspecified.
 */
#ifndef LQ_H_
#define LQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t lq_status;

#define LQ_OK                  0
#define LQ_ERR_ARG             1  /* null pointer, non-positive size, c <= 0   */
#define LQ_ERR_SHAPE           2  /* K % 32 != 0, K != a*b, N/K mismatch, t >= T */
#define LQ_ERR_UNSUPPORTED     3  /* bits not in {4,8}, group != 32, dtype      */
#define LQ_ERR_ALIGN           4  /* pointer not 16-byte aligned                */
#define LQ_ERR_CUDA            5  /* CUDA launch or runtime error               */
#define LQ_ERR_DEVICE_TIMEOUT  6  /* a bounded device-side wait expired         */
#define LQ_ERR_NOMEM           7  /* device allocation failed                   */
#define LQ_ERR_WORKSPACE       8  /* workspace too small                        */
#define LQ_ERR_DEVICE_BOUNDS   9  /* bounds-check build: a kernel index out of range */

/* element types of activation inputs */
#define LQ_F32   0
#define LQ_BF16  1

/* lq_loop_stack modes */
#define LQ_OPEN  0  /* every (t, l) reads its own input                       */
#define LQ_CHAIN 1  /* y of step (t, l) is the input of the next step          */

typedef struct lq_wq lq_wq;        /* resident quantized weights (library-owned) */
typedef struct lq_layer lq_layer;  /* weights + P factors + LAS clips of one module */
typedef struct lq_cta lq_cta;      /* loop-transition adapter (CTA), library-owned */

/* Thread-local text of the last error (empty string if none). */
const char* lq_last_error(void);

/* ABI version: 100 * major + minor. */
int32_t lq_version(void);

/* Bytes of the scale array for an M x K activation: M * (K/32) * 4. */
int64_t lq_act_scale_bytes(int64_t M, int64_t K);

/*
 * lq_quantize_act -- rotate (optional) and group-quantize an activation.
 *
 * Steps 1-3 above for every row of d_x.
 *   d_x      M x K, element type x_dtype (LQ_F32 or LQ_BF16), 16-byte aligned.
 *   d_P1     a x a float32 (row-major) and d_P2 b x b float32, with a*b == K,
 *            a a multiple of 16, b of 8, both <= 128.  Pass d_P1 = d_P2 = NULL,
 *            a = b = 0 to skip the rotation (d_x is then the transformed
 *            input x~ itself).  The rotation accumulates in float64 and rounds
 *            once to float32.
 *   las_t    the LAS clip c_{t,l} > 0 of this module and loop.
 *   bits     4 or 8 (q_max 7 or 127).  group must be 32.
 *   d_codes8 out: M x K int8 codes (may be NULL if d_codes4 is given).
 *   d_codes4 out: M x K/2 bytes of packed 4-bit codes, element 2j in bits 3..0
 *            and element 2j+1 in bits 7..4, two's complement; bits must be 4
 *            (may be NULL).
 *   d_scales out: M x (K/32) float32 steps s_a, row-major.
 * Errors: LQ_ERR_ARG, LQ_ERR_SHAPE (K % 32, a*b != K), LQ_ERR_UNSUPPORTED,
 *         LQ_ERR_ALIGN (outputs must be 16-byte aligned), LQ_ERR_CUDA.
 */
lq_status lq_quantize_act(const void* d_x, int32_t x_dtype, int64_t M, int64_t K,
                          const float* d_P1, int32_t a, const float* d_P2, int32_t b,
                          float las_t, int32_t bits, int32_t group,
                          int8_t* d_codes8, uint8_t* d_codes4, float* d_scales,
                          void* stream);

/*
 * lq_fold_weights -- W_out = W (Q1 kron Q2), float64 accumulation, one
 * rounding to float32.  For the inverse-transpose fold pass Q = P^-T (for an
 * orthogonal P that is P itself; lq_inverse_transpose computes it).
 *   d_W, d_W_out  N x K float32 (may not alias);  d_Q1 a x a, d_Q2 b x b float32.
 */
lq_status lq_fold_weights(const float* d_W, int64_t N, int64_t K,
                          const float* d_Q1, int32_t a, const float* d_Q2, int32_t b,
                          float* d_W_out, void* stream);

/*
 * lq_inverse_transpose -- host helper: h_out = (h_P^-1)^T for an n x n float32
 * matrix, Gauss-Jordan elimination with partial pivoting in float64, rounded
 * to float32.  Synchronous, host memory only.  LQ_ERR_ARG if P is singular.
 */
lq_status lq_inverse_transpose(const float* h_P, int32_t n, float* h_out);

/*
 * lq_quantize_weights -- group-32 4-bit RTN of folded weights into caller
 * buffers: s_w[n,g] = fl32(absmax / 7), q_w = clip(rne(fl32(w / s_w)), -7, 7).
 *   d_W        N x K float32 (already folded).  bits must be 4, group 32.
 *   d_codes8   out N x K int8 (may be NULL);  d_codes4 out N x K/2 packed (may be NULL).
 *   d_scales   out N x (K/32) float32, row-major.
 */
lq_status lq_quantize_weights(const float* d_W, int64_t N, int64_t K, int32_t bits,
                              int32_t group, int8_t* d_codes8, uint8_t* d_codes4,
                              float* d_scales, void* stream);

/*
 * lq_pack_weights -- quantize folded weights into a library-owned resident
 * object used by every loop.  Allocates device memory (cudaMalloc); the call
 * synchronises `stream` before returning.  Release with lq_wq_free.
 * Resident layout: packed 4-bit codes N x K/2 and their steps N x G
 * (float32): 0.625 bytes per weight.  Calls that run the tensor-core GEMM
 * expand, per launch, an 8-bit operand copy (N x K bytes) and the steps
 * transposed (G x N) into their workspace; nothing else is kept resident.
 */
lq_status lq_pack_weights(const float* d_W_folded, int64_t N, int64_t K, int32_t bits,
                          int32_t group, lq_wq** out, void* stream);

/*
 * lq_wq_info -- shapes and device pointers of a resident weight object.
 *   d_codes4 packed codes N x K/2;  d_scales N x (K/32) float32 row-major;
 *   device_bytes: total device memory the object holds.  Any out pointer may be NULL.
 */
lq_status lq_wq_info(const lq_wq* wq, int64_t* N, int64_t* K, const uint8_t** d_codes4,
                     const float** d_scales, int64_t* device_bytes);
void lq_wq_free(lq_wq* wq);

/*
 * lq_layer_create -- bind resident weights to a module's Kronecker factors
 * and LAS clips.  Copies P1 (a x a), P2 (b x b) (device pointers) and
 * h_las[T] (host, every entry > 0) into library-owned device memory;
 * a_bits (4 or 8) selects the activation precision.
 * Synchronous.  `wq` must outlive the layer.  a*b must equal wq's K.
 */
lq_status lq_layer_create(const lq_wq* wq, const float* d_P1, int32_t a, const float* d_P2,
                          int32_t b, const float* h_las, int32_t T, int32_t a_bits,
                          lq_layer** out);
void lq_layer_free(lq_layer* layer);

/*
 * Device workspace needed by lq_loop_linear / lq_loop_stack for M tokens
 * through the given layers: the activation codes and steps of one step, and
 * for the tensor-core path (M > 16) the weight operand of the largest layer
 * (N x K code bytes + G x N steps), expanded from the resident 4-bit codes by
 * each call; for the GEMV path (M <= 16) the codes' group sums and 256 bytes
 * for the step counters of the persistent chain-mode decode kernel.
 */
int64_t lq_workspace_bytes(const lq_layer* const* layers, int32_t L, int64_t M);

/*
 * Workspace with which lq_loop_stack in LQ_OPEN mode runs up to min(T, 8)
 * loops of each layer in one quantize and one GEMM launch (the loops of a
 * layer are independent in open mode and share the resident weights).  For
 * decode-sized M (the GEMV path, M <= 16) the loops of a layer form one unit
 * while their rows fit the GEMV (16 rows), and it is the size that gives
 * every unit of a round (up to 96 units) its own region, so that each round
 * runs as one grouped quantize and one grouped GEMV launch; smaller
 * workspaces run the units as up to 16 concurrent quantize->GEMV chains on
 * internal streams, or as one chain.
 * Returns -1 on a null pointer or a non-positive L or T.
 */
int64_t lq_stack_workspace_bytes(const lq_layer* const* layers, int32_t L, int64_t M,
                                 int32_t T);

/*
 * lq_loop_linear -- one application of a shared quantized linear at loop t:
 * y = Q(x (P1 kron P2); c_t) (*) Wq, steps 1-4 above.
 *   d_x   M x K (x_dtype LQ_F32 or LQ_BF16);  d_y out M x N float32.
 *   d_ws  workspace of at least lq_workspace_bytes(&layer, 1, M) bytes,
 *         256-byte aligned; its contents are scratch.
 * Errors: LQ_ERR_SHAPE if t is not in [0, T), LQ_ERR_WORKSPACE, ...
 */
lq_status lq_loop_linear(const void* d_x, int32_t x_dtype, int64_t M, const lq_layer* layer,
                         int32_t t, float* d_y, void* d_ws, int64_t ws_bytes, void* stream);

/*
 * lq_loop_stack -- the whole T x L loop schedule with resident weights:
 * for t = 0..T-1, for l = 0..L-1: y_{t,l} = lq_loop_linear(x_{t,l}, layer l, t).
 *   mode LQ_OPEN : d_x holds T*L inputs, ordered (t, l), each M x K_l of x_dtype.
 *   mode LQ_CHAIN: d_x holds one M x K_0 input; x_{t,l} is the previous
 *                  step's y (float32).  Needs N_l == K_{l+1} and N_{L-1} == K_0.
 *   d_y   out: T*L outputs ordered (t, l), each M x N_l float32.
 *   d_ws  at least lq_workspace_bytes(layers, L, M) bytes, 256-byte aligned.
 *         In LQ_OPEN mode a larger workspace lets one launch cover several
 *         loops of a layer (as many as fit, at most 8;
 *         lq_stack_workspace_bytes gives the size for min(T, 8)), or, for
 *         decode-sized M, lets all units run in grouped launches or up to 16
 *         of them concurrently on internal streams forked from and joined
 *         back into `stream`; every schedule meets the same tolerances.
 * In LQ_CHAIN mode a decode-sized stack (M <= 4, factors whose b is a
 * multiple of 32, a <= 64, b <= 128, K a multiple of 128) runs all its steps
 * in one persistent cooperative kernel per 128 steps, its waits bounded (an
 * expired wait is reported by lq_check_device as LQ_ERR_DEVICE_TIMEOUT).
 * Consecutive kernels of the schedule use programmatic dependent launch: a
 * kernel starts its prologue (weight loads, rotation of inputs that exist
 * before the call) while its predecessor finishes, and waits for it before
 * reading its output or writing any buffer.
 * The schedule is recorded once into a CUDA graph per distinct argument set
 * and replayed (when `stream` is itself capturing, kernels are launched
 * directly into the caller's capture instead).
 */
lq_status lq_loop_stack(const void* d_x, int32_t x_dtype, int64_t M,
                        const lq_layer* const* layers, int32_t L, int32_t T, int32_t mode,
                        float* d_y, void* d_ws, int64_t ws_bytes, void* stream);

/*
 * lq_loop_stack_slt -- the loop schedule with loop-dependent transforms and
 * weights for the modules that selective loop-specific transforms (SLT)
 * picked ("paper_specification.yaml" of the LoopQ reproduction: slt, Section
 * 4.2 and Eqs. (5)-(6): selected transform-weight groups receive
 * loop-dependent transforms and weights; Appendix B.1 Table 4 and the
 * slt_budget, 4 groups on Ouro-1.4B).  The selection itself is calibration
 * and not part of this library; this call serves a selection.
 *   layers_tl  T*L handles ordered (t, l): step (t, l) applies
 *              layers_tl[t*L + l] with that handle's LAS clip c_t.  A module
 *              that SLT did not select repeats its shared handle in every
 *              loop; a selected module has one handle per loop (its own P_t,
 *              folded W_t and clips).  Every handle of module l must have the
 *              K and N of layers_tl[l], and at least t + 1 clips.
 * Everything else (modes, input and output layout, workspace, graph reuse,
 * programmatic launch, errors) as lq_loop_stack, which is this call with
 * layers_tl[t*L + l] = layers[l].  In open mode, consecutive loops of a module
 * share launches only where they share a handle.
 */
lq_status lq_loop_stack_slt(const void* d_x, int32_t x_dtype, int64_t M,
                            const lq_layer* const* layers_tl, int32_t L, int32_t T, int32_t mode,
                            float* d_y, void* d_ws, int64_t ws_bytes, void* stream);

/*
 * Cross-loop transition alignment (CTA): an affine plus gated low-rank adapter
 * applied to the recurrent state only at loop transitions
 * ("paper_specification.yaml" of the LoopQ reproduction: cta, Section 4.3,
 * Eq. (7); implementation_status lq5: U and V shared, a_t, b_t and the gate
 * eta_t loop-dependent, rank 8, identity at initialization).  Eq. (7) is not
 * printed on the pages; this library takes the plainest reading,
 *     h' = a_t * h + b_t + eta_t * (h V) U^T,
 * computed in float64 and rounded once to float32.
 *
 * lq_cta_create -- copy the adapter to library-owned device memory.
 *   d_U, d_V  d x rank float32 row-major (device), 1 <= rank <= 8;
 *   d_a, d_b  n_trans x d float32 row-major (device): a_t, b_t of transition t
 *             (t -> t + 1);  h_eta[n_trans] (host, finite): the gates.
 * d must be a multiple of 32 and at most 6144 (LQ_ERR_SHAPE).  Synchronous.  LQ_ERR_ARG on null
 * pointers or bad sizes, LQ_ERR_CUDA on a failed copy or allocation.  Release
 * with lq_cta_free.
 */
lq_status lq_cta_create(const float* d_U, const float* d_V, int64_t d, int32_t rank,
                        const float* d_a, const float* d_b, const float* h_eta, int32_t n_trans,
                        lq_cta** out);
void lq_cta_free(lq_cta* cta);

/*
 * lq_cta_apply -- d_out = CTA_t(d_h) for M rows of width d (float32, row-major,
 * 16-byte aligned; d_out may equal d_h).  LQ_ERR_SHAPE if t is not a
 * transition of the adapter.  Asynchronous on `stream`.
 */
lq_status lq_cta_apply(const float* d_h, int64_t M, const lq_cta* cta, int32_t t, float* d_out,
                       void* stream);

/*
 * lq_loop_stack_cta -- chain-mode lq_loop_stack with CTA at every loop
 * transition: after loop t < T-1 the state passed to loop t + 1 is
 * CTA_t(y_{t, L-1}).  d_y receives the unadapted outputs y_{t,l}, ordered
 * (t, l) as in lq_loop_stack.  The adapter width must be N_{L-1} (= K_0) and
 * it must have at least T - 1 transitions (LQ_ERR_SHAPE).  The workspace must
 * hold lq_cta_stack_workspace_bytes(layers, L, M) bytes: the codes and steps
 * plus the adapted state.  Graph reuse, programmatic launch and errors as
 * lq_loop_stack.
 */
int64_t lq_cta_stack_workspace_bytes(const lq_layer* const* layers, int32_t L, int64_t M);
lq_status lq_loop_stack_cta(const void* d_x, int32_t x_dtype, int64_t M,
                            const lq_layer* const* layers, int32_t L, int32_t T,
                            const lq_cta* cta, float* d_y, void* d_ws, int64_t ws_bytes,
                            void* stream);

/*
 * lq_trajectory_hessian -- calibration statistic of one module over its loop
 * inputs: H = sum_t X_t^T X_t (or H += that sum when `accumulate` is set),
 * the Hessian accumulated across recurrence steps ("Quantizing Looped
 * Transformers: Feedback Exposure and Calibration Blindness", Appendix Table
 * 19, H_t = X_t^T X_t; abstract and Section 5, accumulating the GPTQ Hessian
 * across recurrence steps).  Unnormalised.
 *   d_X   T inputs back to back, each M x K bf16 row-major (x_dtype LQ_BF16;
 *         others LQ_ERR_UNSUPPORTED), 16-byte aligned;
 *   d_H   K x K float32 row-major (read when accumulating);
 *   d_ws  lq_hessian_workspace_bytes(M, K, T) bytes, 256-byte aligned
 *         (the transposed inputs).
 * K must be a multiple of 128 (LQ_ERR_SHAPE).  bf16 products are exact in
 * float32; the sums are the tensor cores' float32 accumulation over M*T terms.
 * Asynchronous on `stream`.
 */
int64_t lq_hessian_workspace_bytes(int64_t M, int64_t K, int32_t T);
lq_status lq_trajectory_hessian(const void* d_X, int32_t x_dtype, int64_t M, int64_t K,
                                int32_t T, float* d_H, int32_t accumulate, void* d_ws,
                                int64_t ws_bytes, void* stream);

/*
 * lq_loop_linear_noalloc -- lq_loop_linear for callers that cannot allocate
 * device memory, so cannot provide its workspace: for instance the enqueue
 * hook of another runtime that hands over only input and output buffers, a
 * serving loop that forbids allocation once it has started, or code running
 * while another framework's caching allocator owns all free device memory.
 * (The paper has no counterpart; this is a deployment convenience.)
 *
 * Same arguments, checks, kernels and results as lq_loop_linear, minus the
 * workspace.  The scratch is a fixed device array of LQ_NOALLOC_SCRATCH_BYTES
 * built into the library; every GPU that loads the library holds it until the
 * process exits.  The call allocates nothing (no cudaMalloc, no cudaFree).
 *   - Calls needing more scratch than that, lq_workspace_bytes(&layer, 1, M)
 *     > LQ_NOALLOC_SCRATCH_BYTES (about M*K*(1 + 1/8) bytes, plus
 *     N*K*(1 + 1/8) for the weight operand when M > 16), fail with
 *     LQ_ERR_WORKSPACE and enqueue nothing.
 *   - All calls share the one array, which keeps the last call's contents.
 *     Each call writes every scratch byte it reads before reading it, so
 *     nothing has to start at zero; but calls whose work overlaps on the GPU
 *     (for instance on two streams without ordering between them) race on the
 *     array and give wrong results.
 *   - The first call on a device looks the array's device address up (once
 *     per device and context, with that device current); make that first
 *     call before any stream capture.  After a device reset the next call
 *     looks the address up again, so make it outside a capture too.
 */
#define LQ_NOALLOC_SCRATCH_BYTES (16ll << 20)
lq_status lq_loop_linear_noalloc(const void* d_x, int32_t x_dtype, int64_t M,
                                 const lq_layer* layer, int32_t t, float* d_y, void* stream);

/*
 * Kernel timing probe.  While enabled (on != 0), lq_loop_linear and
 * lq_loop_stack launch their kernels directly (no graph) and bracket each one
 * with CUDA events recorded on the launching stream.  lq_probe_read waits for
 * those events and returns, per kernel kind, the summed device time in
 * milliseconds and the number of launches, then clears them.  Kinds (index):
 * 0 fused rotate+quantize, 1 quantize-only, 2 tensor-core GEMM, 3 GEMV,
 * 4 weight-operand expansion (the GEMM's 8-bit weight bytes and transposed
 * steps, one per GEMM launch), 5 persistent chain-mode decode (one launch
 * covers up to 128 quantize -> GEMV steps of a decode-sized chain-mode stack).
 * h_ms and h_count point to arrays of LQ_PROBE_KINDS entries (host memory).
 */
#define LQ_PROBE_KINDS 6
lq_status lq_probe_enable(int32_t on);
lq_status lq_probe_read(double* h_ms, int64_t* h_count);

/*
 * lq_check_device -- synchronise `stream`, then read and clear the device
 * status word that kernels set when a bounded wait expires.  Returns LQ_OK or
 * LQ_ERR_DEVICE_TIMEOUT (or LQ_ERR_CUDA for an asynchronous CUDA error).  In
 * the bounds-check build (compiled with -DLQ_BOUNDS_CHECK) kernels also test
 * their store indices against the extents they write, skip and record an
 * index out of range, and this call returns LQ_ERR_DEVICE_BOUNDS with the
 * source line and index in lq_last_error(); the normal build never does.
 */
lq_status lq_check_device(void* stream);

/*
 * lq_selftest_bounded_wait -- diagnostic of the failure path: enqueue a tiny
 * kernel that waits, through the same bounded mbarrier wait the GEMM uses, on
 * a barrier phase that nothing completes.  The wait gives up after limit_us
 * microseconds (0 < limit_us <= 10 s) and records LQ_ERR_DEVICE_TIMEOUT in the
 * device status word; the kernel then returns normally and the context stays
 * usable.  A following lq_check_device(stream) reports (and clears) it.
 */
lq_status lq_selftest_bounded_wait(int64_t limit_us, void* stream);

/*
 * lq_selftest_grid_wait -- the same diagnostic for the grid barrier of the
 * persistent chain-mode decode kernel: one block waits at a grid barrier that
 * expects one block more than the launch has.  The wait gives up after
 * limit_us microseconds (0 < limit_us <= 10 s) and records
 * LQ_ERR_DEVICE_TIMEOUT; a following lq_check_device(stream) reports (and
 * clears) it.  d_scratch: 8 bytes of device memory the barrier uses.
 */
lq_status lq_selftest_grid_wait(int64_t limit_us, void* d_scratch, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LQ_H_ */
