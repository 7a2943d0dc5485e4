/*
 * muon.h - C ABI of the B200 (sm_100a) Muon optimizer step.
 *
 * The Muon step for one 2-D hidden-layer weight W (rows x cols) with gradient g:
 *
 *   g <- g - 1 mean_dim0(g)^T                  optional zero-centring, before momentum
 *                                              ("Muon meets Mamba", sections 2.1 and 4.2)
 *   m <- mu m + (1 - mu) g                     momentum buffer (EMA form)
 *   u <- nesterov ? mu m + (1 - mu) g : m      Nesterov look-ahead
 *                                              ("Muon optimizer: matrix-aware LLM training",
 *                                               `Muon.step` listing)
 *   X <- u / (||u||_F + eps), transposed when rows > cols
 *   repeat steps times:                        ("Muon optimizer ..." `newtonschulz5` listing;
 *     A <- X X^T                                "AdamW vs Muon" part 3, the quintic update
 *     B <- b_k A + c_k A A                      M_k = a M + b (M M^T) M + c (M M^T)^2 M)
 *     X <- a_k X + B X
 *   O <- X, transposed back
 *   W <- W (1 - lr wd) - lr s O               decoupled decay and update; s is the RMS factor
 *                                              ("AdamW vs Muon" part 3 "scaling and update";
 *                                               "Muon meets Mamba" section 4.2)
 *
 * All arithmetic runs in hand-written sm_100a kernels: a fused elementwise prologue, the
 * Newton-Schulz matrix products on the tcgen05 tensor cores (bf16 operands with fp32
 * accumulation in tensor memory, or fp32 accuracy through 3xTF32 products), with the parameter
 * update fused into the last product. There is no CPU fallback: on a machine without an sm_100
 * device every compute call fails with MUON_ERR_UNSUPPORTED.
 *
 * Conventions shared by every call:
 *   - Matrices are dense, row-major, contiguous (leading dimension = cols).
 *   - Pointers named "device" must be device memory (or managed memory) of the current device.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy default stream) and
 *     never synchronise the host, except a call with a list of shapes (or precision, or wave
 *     budget) that is not among the 16 most recently used on the device: it builds a plan (a
 *     small table allocation with cudaMalloc, uploaded once) and, when its buffers need more
 *     than the workspace holds, grows the workspace (cudaFree and cudaMalloc, which synchronise
 *     the device). Per-call tables (the caller's pointers) travel to the device inside kernel
 *     launch parameters, so they never wait behind the caller's own copies on a copy engine.
 *   - muon_step processes its matrices in waves of consecutive matrices (see
 *     muon_set_wave_elements); the workspace holds one wave's buffers, about 4 bytes per element
 *     of the largest wave seen so far in bf16 working precision and 16 in fp32. Plans of
 *     different shape lists share it.
 *   - The workspace is owned by the library, per process, and shared by all calls: calls must be
 *     ordered (same stream, or synchronised by the caller). Concurrent calls race.
 *   - Argument errors are detected before any device work is enqueued; the call then returns a
 *     negative code and muon_last_error() describes the first problem found.
 *   - Device-side faults of the library's own making (a wait that timed out inside a kernel, a
 *     non-finite value in an update matrix) are recorded in a device status word that
 *     muon_check_status() reads.
 */
#ifndef MUON_H_
#define MUON_H_

#include <stdint.h>

#if defined(__GNUC__)
#define MUON_API __attribute__((visibility("default")))
#else
#define MUON_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so that this header needs no CUDA headers. */
typedef struct CUstream_st* muon_stream_t;

typedef enum { MUON_BF16 = 0, MUON_FP32 = 1 } muon_dtype_t;

/* Working precision of the Newton-Schulz iterate.
 *   MUON_PREC_BF16: X, A, B stored in bf16, products on tcgen05 tensor cores with fp32
 *                   accumulation (the pages' bf16 working copy).
 *   MUON_PREC_FP32: X, A, B held in fp32, each as two planes (the value rounded toward zero to
 *                   tf32, and the remainder); products on tcgen05 tensor cores as three tf32
 *                   products (lo*hi + hi*lo + hi*hi, "3xTF32"), accumulated in fp32 in chunks of
 *                   512 along K and summed in fp32 with round-to-nearest. Relative error of one
 *                   product about 1e-6 at any K. The workspace takes 16 bytes per element of
 *                   the iterate (bf16 mode: 4). */
typedef enum { MUON_PREC_BF16 = 0, MUON_PREC_FP32 = 1 } muon_prec_t;

/* RMS factor s of the update ("AdamW vs Muon" part 3 rescales by matrix shape without giving a
 * formula): MUON_RMS_ONE gives s = 1; MUON_RMS_SQRT_MAX1_ROWS_OVER_COLS gives
 * s = sqrt(max(1, rows / cols)). */
typedef enum { MUON_RMS_ONE = 0, MUON_RMS_SQRT_MAX1_ROWS_OVER_COLS = 1 } muon_rms_t;

/* One Newton-Schulz iteration's coefficients: X <- a X + b (X X^T) X + c (X X^T)^2 X.
 * Quintic ("Muon optimizer ..." `newtonschulz5`): {3.4445, -4.7750, 2.0315}.
 * Cubic ("Muon meets Mamba" 2.2):                 {1.5, -0.5, 0}.
 * When c == 0 the A A product is skipped. */
typedef struct {
  float a, b, c;
} muon_coeffs_t;

/* Return codes. */
enum {
  MUON_OK = 0,
  MUON_WARN_NONFINITE = 1,    /* muon_check_status only: a NaN/Inf reached an update matrix   */
  MUON_ERR_INVALID_ARG = -1,  /* bad pointer, size, count, step count or aliasing             */
  MUON_ERR_UNSUPPORTED = -2,  /* no sm_100 device, or a dtype/precision combination not built  */
  MUON_ERR_WORKSPACE = -3,    /* workspace allocation failed (device out of memory)           */
  MUON_ERR_CUDA = -4,         /* a CUDA runtime/driver call failed                            */
  MUON_ERR_TIMEOUT = -5       /* muon_check_status only: a kernel wait hit its time limit and  */
                              /* the kernel returned early; results of that call are invalid  */
};

/* Largest number of Newton-Schulz iterations accepted by one call. */
#define MUON_MAX_NS_STEPS 64

/*
 * Newton-Schulz orthogonalisation of one matrix ("Muon optimizer ..." `newtonschulz5`).
 *
 *   G      device, m x n (m rows, n cols), element type g_dtype. Read only.
 *   X      device, m x n, element type x_dtype. Written: X = NS(G). May not overlap G.
 *   steps  number of iterations, 0..MUON_MAX_NS_STEPS; 0 returns G / (||G||_F + eps).
 *   coeffs host array of `steps` triples, or NULL for `steps` quintic triples.
 *   zero_center  nonzero: subtract the mean over dim 0 (column means) from G first.
 *   eps    added to the Frobenius norm before dividing (pages: 1e-7). Must be >= 0.
 *   prec   working precision (see muon_prec_t).
 * Rows > cols runs the iteration on G^T and transposes back, as the pages do.
 * Returns MUON_OK or a negative error code.
 */
MUON_API int muon_ns_orthogonalize(const void* G, muon_dtype_t g_dtype, void* X, muon_dtype_t x_dtype,
                          int64_t m, int64_t n, int steps, const muon_coeffs_t* coeffs,
                          int zero_center, float eps, muon_prec_t prec, muon_stream_t stream);

/*
 * One Muon step over `count` independent matrices ("Muon optimizer ..." `Muon.step`;
 * "Muon meets Mamba" section 4.2 `_step_muon`).
 *
 *   params[i]   device fp32, rows[i] x cols[i]; updated in place.
 *   grads[i]    device, element type grad_dtype; read only. NULL skips matrix i entirely
 *               (its params and momentum are left untouched), like a parameter with no grad.
 *   momentum[i] device fp32, same shape; updated in place. Start from zeros.
 *               (The pages keep the buffer in the gradient's dtype; fp32 is used here so that
 *               the parameter update stays accurate.)
 *   lr, mu, nesterov, weight_decay   as in the step above; 0 <= mu < 1, lr and wd finite.
 *   rms_scale   the RMS factor s (muon_rms_t).
 *   steps, coeffs, zero_center, eps, prec   as for muon_ns_orthogonalize.
 * params[i] and momentum[i] must not overlap each other or any other matrix's buffers.
 * The matrices of one wave (consecutive matrices of at most 2^29 elements in total, see
 * muon_set_wave_elements) share the same kernel launches (one prologue, one norm, one grouped
 * tensor-core launch per Newton-Schulz phase, the last of which also updates the parameters),
 * so small matrices are not launch-bound. Returns MUON_OK or a negative error code.
 */
MUON_API int muon_step(int count, float* const* params, const void* const* grads, muon_dtype_t grad_dtype,
              float* const* momentum, const int64_t* rows, const int64_t* cols, float lr, float mu,
              int nesterov, float weight_decay, muon_rms_t rms_scale, int steps,
              const muon_coeffs_t* coeffs, int zero_center, float eps, muon_prec_t prec,
              muon_stream_t stream);

/*
 * Newton-Schulz orthogonalisation of one matrix that allocates nothing.
 * (No counterpart in the pages: this is an interface concern, not part of the method.)
 *
 * For callers that cannot allocate device memory while they run: for example a plugin or
 * custom-call hook whose host framework owns all allocations and forbids cudaMalloc inside its
 * execution callback, or a service that reserves its memory at start-up and allocates nothing
 * afterwards. muon_ns_orthogonalize allocates its workspace with cudaMalloc on first use; this
 * call instead works in a fixed scratch area compiled into the library (a __device__ array of
 * about 12.1 MiB, reserved on every device that loads the library and held until the process
 * exits), and calls no cudaMalloc, cudaFree or other allocating routine.
 *
 *   G, g_dtype, X, x_dtype, m, n, steps, coeffs, eps   as for muon_ns_orthogonalize
 *           (bf16 working precision; no zero-centring).
 *   status  optional device pointer to 2 ints owned by the caller, or NULL. Kernels set
 *           bit 0 of status[0] when a wait hits its time limit (the result is then invalid)
 *           and add to status[1] the number of 8192-element chunks that held NaN or Inf; the
 *           caller clears it. With NULL these go to a word in the scratch area, cleared by
 *           every call, that the caller cannot read.
 * Limits: min(m, n) <= 1024 and m * round_up(n, 8) <= 2097152 elements; larger matrices are
 * rejected with MUON_ERR_INVALID_ARG (use muon_ns_orthogonalize).
 * The first call on a device sets that device up (it looks up the scratch address); make that
 * first call before any stream capture. All calls share the one scratch area and overwrite it:
 * calls must be ordered on the GPU (one stream, or synchronised by the caller); calls that
 * overlap on the GPU race. Returns MUON_OK or a negative error code.
 */
MUON_API int muon_ns_orthogonalize_noalloc(const void* G, muon_dtype_t g_dtype, void* X,
                                           muon_dtype_t x_dtype, int64_t m, int64_t n, int steps,
                                           const muon_coeffs_t* coeffs, float eps, int* status,
                                           muon_stream_t stream);

/*
 * One AdamW step over `count` tensors, for the parameters that do not go to Muon (embeddings,
 * prediction head, norm scales, biases: "Muon meets Mamba" sections 2.1 and 4.3; "AdamW vs Muon"
 * on which modules keep AdamW). Follows `_step_adamw` ("Muon meets Mamba" section 4.2):
 *
 *   p <- p (1 - lr wd)                                           decoupled decay, first
 *   m <- beta1 m + (1 - beta1) g,   v <- beta2 v + (1 - beta2) g^2
 *   p <- p - (lr / (1 - beta1^t)) m / (sqrt(v) / sqrt(1 - beta2^t) + eps)
 *
 *   params[i], exp_avg[i], exp_avg_sq[i]   device fp32, numel[i] elements each (any shape,
 *                  contiguous); updated in place. Start the moments from zeros.
 *   grads[i]       device, element type grad_dtype; NULL skips tensor i.
 *   step           t, the step count after this step (1 for the first step); shared by all tensors.
 *   lr, beta1, beta2, eps, weight_decay   0 <= beta < 1, eps >= 0, lr and wd finite
 *                  (the pages' defaults: lr 1e-3, betas (0.9, 0.95), eps 1e-8).
 * Arithmetic is fp32. One launch covers every tensor. Buffers of different tensors must not
 * overlap. Returns MUON_OK or a negative error code.
 */
MUON_API int muon_adamw_step(int count, float* const* params, const void* const* grads,
                             muon_dtype_t grad_dtype, float* const* exp_avg, float* const* exp_avg_sq,
                             const int64_t* numel, int64_t step, float lr, float beta1, float beta2,
                             float eps, float weight_decay, muon_stream_t stream);

/* Message describing the last error returned on the calling thread ("" if none). The pointer
 * stays valid until the next call on that thread. */
MUON_API const char* muon_last_error(void);

/* Synchronises `stream`, then reads and clears the device status word of the current device.
 * Returns MUON_ERR_TIMEOUT if a kernel gave up waiting since the last check,
 * MUON_WARN_NONFINITE if a NaN or Inf reached an update matrix, MUON_OK otherwise
 * (or MUON_ERR_CUDA if synchronising failed). */
MUON_API int muon_check_status(muon_stream_t stream);

/* Frees the workspace and cached plans of the current device (synchronises the device). */
MUON_API int muon_release_workspace(void);

/* Tuning: the largest number of elements (summed over consecutive matrices) that muon_step
 * processes in one wave of launches (prologue, norm and Newton-Schulz products); a larger matrix
 * is a wave of its own. Waves only split the launch sequence: the results do not depend on the
 * setting. Smaller launches keep more of one phase's output in L2 for the next phase and, under
 * the power cap, run at higher clocks (one Llama-8B step: about 460 ms in waves of two layers
 * against 520-580 ms in one wave), at the cost of more launches. elements = 0 restores the
 * default, 2^29; negative values are rejected with MUON_ERR_INVALID_ARG. Applies to calls made
 * after it (a cached plan built with another setting is rebuilt). */
MUON_API int muon_set_wave_elements(int64_t elements);

/* Diagnostics: the time limit, in nanoseconds, of every wait inside the Newton-Schulz product
 * kernels launched by later muon_step and muon_ns_orthogonalize calls (operand stages,
 * accumulators, epilogue loads). A wait that runs out makes the kernel stop early, set the
 * timeout bit of the device status word (muon_check_status then returns MUON_ERR_TIMEOUT; that
 * call's results are invalid) and return, leaving the device usable. ns = 0 restores the default
 * of 2 s. A limit of a few nanoseconds makes a call give up at its first wait that is not
 * already complete: a way to exercise that failure path. (The no-allocation call keeps the
 * default.) Returns MUON_OK. */
MUON_API int muon_set_wait_limit_ns(uint64_t ns);

/* Tuning and diagnostics: chained launches. A wave whose matrices all use 256 x 256 tiles (bf16
 * working precision; waves dominated by matrices with min(rows, cols) >= 2048 use 256 x 512 tiles
 * and are never chained) can run its whole Newton-Schulz iteration as one launch: tiles are
 * claimed in order, and each phase waits per matrix for the phase whose results it reads, so the
 * fixed cost of fifteen launches and their tails disappears.
 *   mode 0: never chain; one grouped kernel per phase.
 *   mode 1 (default): chain a wave when one iteration has at most 8 tiles per CTA pair of the
 *           device (small sets of small matrices, where launch costs dominate).
 *   mode 2: chain every wave of small matrices.
 * The results are bit-identical in every mode. With chaining, muon_profile_read counts the whole
 * iteration under MUON_KC_GEMM (no per-phase breakdown). Applies to calls made after it (a cached
 * plan built in another mode is rebuilt). Returns MUON_OK, or MUON_ERR_INVALID_ARG for another
 * mode. */
MUON_API int muon_set_chained_launch(int mode);

/* Kernel classes counted and timed by the library, indices into muon_profile_read's arrays. */
enum {
  MUON_KC_CENTER = 0,   /* column sums and means for zero-centring                    */
  MUON_KC_PROLOGUE = 1, /* momentum, Nesterov, norm partials, bf16 cast                 */
  MUON_KC_NORM = 2,     /* per-matrix 1 / (||u|| + eps)                                 */
  MUON_KC_GEMM = 3,     /* Newton-Schulz matrix products (all three phases)             */
  MUON_KC_EPILOGUE = 4, /* decay and parameter update, or the output conversion         */
  MUON_KC_ADAMW = 5,    /* AdamW step (muon_adamw_step)                                 */
  /* breakdown of MUON_KC_GEMM by phase: every Newton-Schulz launch is counted both in
   * MUON_KC_GEMM and in the class of its phase */
  MUON_KC_GEMM_GRAM = 6,   /* A = X X^T                                                 */
  MUON_KC_GEMM_POLY = 7,   /* B = c A A + b A (+ a I)                                   */
  MUON_KC_GEMM_UPDATE = 8, /* X' = B X (last one may carry the fused parameter update)  */
  MUON_KC_COUNT = 9
};

/* Turns per-launch timing on (nonzero) or off. While on, every kernel launch is bracketed by
 * CUDA events recorded on the launching stream. */
MUON_API int muon_profile_enable(int on);

/* Synchronises the recorded events and returns, per kernel class, the number of launches and
 * their summed device time in milliseconds since the last read (arrays of MUON_KC_COUNT).
 * Also returns, in flops (may be NULL), the nominal Newton-Schulz FLOPs of those GEMM launches
 * (4 m^2 n + 2 m^3 per quintic iteration, m = min dim) and, in exec_flops (may be NULL), the
 * FLOPs the tensor cores actually executed (triangle tiles only). Clears the records. */
MUON_API int muon_profile_read(int64_t* launches, double* ms, double* flops, double* exec_flops);

/* Total number of kernels this library has launched in this process. */
MUON_API int64_t muon_launch_count(void);

/* Library version, major * 10000 + minor * 100 + patch. */
MUON_API int muon_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MUON_H_ */
