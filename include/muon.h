/*
 * muon.h -- C ABI of the B200 (sm_100a) Muon optimizer step.
 *
 * The operation (autoresearch train.py review, web3.cnoyu.systems post
 * 71151920174080, paragraph on the MuonAdamW optimizer): for every 2-D weight W
 * with gradient G and momentum buffer M,
 *
 *   M  <- mu*M + G                      (float32 buffer, product and sum rounded
 *                                        separately)
 *   U  <- G + mu*M   (Nesterov)  or  U <- M
 *   X0 <- U / (||U||_F + eps)
 *   k = 1..K, tall (rows > cols):  A = X^T X,  X <- a_k X + X (b_k A + c_k A^2)
 *             otherwise (wide):    A = X X^T,  X <- a_k X + (b_k A + c_k A^2) X
 *   W  <- W - fl32(lr*sqrt(max(1, rows/cols))) * X_K
 *
 * The page fixes the momentum, the five Newton-Schulz steps, the tall/wide rules
 * and per-step coefficient triples ("Polar Express", values not printed); the
 * Frobenius normalisation with eps and the update scale come from the method's
 * task statement.  Newton-Schulz runs on tcgen05 tensor cores with bf16 operands and
 * fp32 accumulation in MUON_MODE_BF16, on tcgen05 tensor cores with fp32 storage and
 * 3xTF32 products in MUON_MODE_FP32_VALIDATE, and on fp32 CUDA-core FMAs in
 * MUON_MODE_FP32_SIMT.
 *
 * Conventions for every entry point
 *  - All matrix pointers are DEVICE pointers on the handle's device, row-major and
 *    contiguous (element (i, j) at i*cols + j), 16-byte aligned.  They stay owned
 *    by the caller.  No two matrices' pointers may overlap.  A pointer that is not
 *    device memory of the handle's device (host memory, another GPU's memory) is
 *    an argument error (checked when a call's pointers differ from the last call's).
 *  - Work is enqueued on `cuda_stream` (a cudaStream_t; NULL = legacy default
 *    stream) and the call returns without waiting for it.
 *  - Argument errors are detected on the host and returned before anything is
 *    enqueued (MUON_ERR_INVALID_ARG / MUON_ERR_UNSUPPORTED); the detail is
 *    available from muon_last_error().  A CUDA error while enqueueing returns
 *    MUON_ERR_CUDA.  A device-side time-out of one of the library's bounded waits
 *    is reported as MUON_ERR_TIMEOUT by the next call on the handle, or by
 *    muon_sync / muon_destroy.
 *  - The library owns a workspace on the device (two bf16 or fp32 copies of every
 *    matrix, one s x s Gram and one s x s polynomial buffer per matrix with
 *    s = min(rows, cols), per-matrix norm partials).  It is allocated, with
 *    cudaMalloc, on the first call with a new list of shapes and mode, and reused
 *    by later calls with the same list; such calls allocate nothing.  Calls that
 *    share a handle must not overlap on the GPU (use one stream per handle, or
 *    one handle per stream).  A handle is not thread-safe; distinct handles may be
 *    used from distinct host threads.
 *  - With the environment variable MUON_LOG set (and not "0") when a handle is
 *    created, that handle writes its plans (shape groups, tile counts, workspace
 *    bytes) and the detail of every error to stderr.
 *  - With MUON_DEBUG set (and not "0") when a handle is created, that handle puts a
 *    256-byte guard band filled with a fixed pattern after every workspace region, and
 *    at the end of every call (outside stream capture) waits for the call's work and
 *    checks the bands on the device: a changed band is returned as MUON_ERR_CORRUPT,
 *    naming the region it follows, and the bands are filled again.  Results are the
 *    same as without it; calls then synchronize the stream.
 *  - With MUON_NVTX set (and not "0") when a handle is created, that handle wraps every
 *    call and every kernel launch in an NVTX range named after the call or the kernel
 *    kind, for timeline profilers (no effect on results).
 */
#ifndef MUON_B200_MUON_H
#define MUON_B200_MUON_H

#include <stdint.h>

#if defined(__GNUC__)
#define MUON_API __attribute__((visibility("default")))
#else
#define MUON_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct muon_handle* muon_handle_t;

typedef enum {
  MUON_OK = 0,
  MUON_ERR_INVALID_ARG = 1,  /* null / misaligned / overlapping pointers, bad sizes or values */
  MUON_ERR_UNSUPPORTED = 2,  /* a combination the library does not implement (e.g. no sm_100 device) */
  MUON_ERR_OOM = 3,          /* workspace allocation failed */
  MUON_ERR_CUDA = 4,         /* a CUDA runtime / driver call failed */
  MUON_ERR_TIMEOUT = 5,      /* a bounded device-side wait expired (kernel gave up and returned) */
  MUON_ERR_TOO_LARGE = 6,    /* the matrix does not fit the fixed scratch of muon_newton_schulz_noalloc */
  MUON_ERR_CORRUPT = 7       /* debug mode: a guard band around a workspace region was overwritten */
} muon_status;

typedef enum { MUON_F32 = 0, MUON_BF16 = 1 } muon_dtype;

typedef enum {
  MUON_MODE_BF16 = 0,           /* Newton-Schulz on tcgen05 tensor cores, bf16 operands, fp32 accumulate */
  MUON_MODE_FP32_VALIDATE = 1,  /* fp32 storage; products on tcgen05 tensor cores as 3xTF32: each fp32
                                   value is split into hi = tf32(x) and lo = tf32(x - hi) and a
                                   product accumulates hi*hi and hi*lo + lo*hi in fp32 (validation).
                                   The tensor cores' accumulation error grows with the contraction
                                   length, so a call with a matrix side above 8192 runs on CUDA
                                   cores as in MUON_MODE_FP32_SIMT */
  MUON_MODE_FP32_SIMT = 2       /* fp32 storage and fp32 FMA on CUDA cores (validation, slowest) */
} muon_mode;

/* One weight matrix.  param: rows*cols of param_dtype, updated in place.  grad:
 * rows*cols of grad_dtype, read only.  momentum: rows*cols float32, updated in
 * place.  rows, cols >= 1. */
typedef struct {
  void* param;
  const void* grad;
  float* momentum;
  int64_t rows;
  int64_t cols;
  muon_dtype param_dtype;
  muon_dtype grad_dtype;
} muon_matrix;

/* Creates a handle bound to CUDA device `device`.  Allocates host memory only and
 * launches no GPU work.  Returns MUON_ERR_INVALID_ARG for a NULL `out` or a device
 * index out of range, MUON_ERR_UNSUPPORTED if the device is not compute
 * capability 10.0 (the kernels are built for sm_100a only). */
MUON_API muon_status muon_init(muon_handle_t* out, int device);

/* One Muon step over `n` matrices (see the operation above).
 *  lr            learning rate (finite, >= 0)
 *  momentum      mu in [0, 1)
 *  nesterov      nonzero: U = G + mu*M_new; zero: U = M_new
 *  coeffs        HOST pointer to ns_steps rows of (a, b, c) float32, row k used in
 *                Newton-Schulz step k; NULL = (3.4445, -4.7750, 2.0315) every step
 *  ns_steps      1..16
 *  eps           added to the Frobenius norm (finite, >= 0)
 *  mode          MUON_MODE_BF16, MUON_MODE_FP32_VALIDATE or MUON_MODE_FP32_SIMT
 *  cuda_stream   cudaStream_t the work is enqueued on
 * Every matrix is processed independently; their order does not matter.  The
 * applied factor per matrix is the float32 rounding of lr*sqrt(max(1,rows/cols))
 * computed in double, and the new weight is fl32(W - fl32(factor*O)) rounded to
 * nearest-even into param_dtype. */
MUON_API muon_status muon_step(muon_handle_t h, const muon_matrix* mats, int n,
                      float lr, float momentum, int nesterov,
                      const float* coeffs, int ns_steps, float eps,
                      muon_mode mode, void* cuda_stream);

/* Form of the momentum buffer update. */
typedef enum {
  MUON_MOMENTUM_SGD = 0,  /* M <- fl32(fl32(mu*M) + G);  Nesterov U = fl32(G + fl32(mu*M)) */
  MUON_MOMENTUM_LERP = 1  /* M <- fl32(fl32(mu*M) + fl32((1-mu)*G));
                             Nesterov U = fl32(fl32((1-mu)*G) + fl32(mu*M)); 1-mu in float32 */
} muon_momentum_form;

/* All options of one step (muon_step_ex).  Fields as in muon_step, plus:
 *  momentum_form   MUON_MOMENTUM_SGD (muon_step's form) or MUON_MOMENTUM_LERP
 *  weight_decay    >= 0; 0 disables.  W <- fl32(W' - fl32(fl32(lr*wd)*W)) after the
 *                  update W' = fl32(W - fl32(lr*scale)*O), with W the weight before the
 *                  step
 *  cautious        nonzero: decay only entries where O*W >= 0 (update and weight agree
 *                  in sign; zeros count as agreeing) -- the cautious weight decay of the
 *                  autoresearch train.py review's MuonAdamW paragraph */
typedef struct {
  float lr;
  float momentum;
  int nesterov;
  muon_momentum_form momentum_form;
  const float* coeffs;
  int ns_steps;
  float eps;
  muon_mode mode;
  float weight_decay;
  int cautious;
  /* NorMuon (autoresearch train.py review, MuonAdamW paragraph: a per-row -- or, by
   * aspect ratio, per-column -- second moment of the orthogonalised update, kept as an
   * EMA, scales the update per output dimension).  With s = min(rows, cols),
   * L = max(rows, cols) and i running over the shorter dimension:
   *   q_i = sum over the longer dimension of O_i^2 / L          (fp32 sums)
   *   v_i <- fl32(fl32(beta2*v_i) + fl32((1-beta2)*q_i))
   *   f_i = 1/(sqrt(v_i) + eps),  r = sqrt(sum_i q_i / sum_i q_i f_i^2)
   *   O  <- fl32(fl32(f_i*r) * O)                               (same Frobenius norm)
   * before the update (and the cautious mask) use O.  normuon_state is a HOST array of
   * n DEVICE pointers, each to s float32 values (16-byte aligned, zero before the
   * first step), updated in place.  The weight update then runs as a separate pass. */
  int normuon;
  float normuon_beta2;          /* [0, 1) */
  float normuon_eps;            /* > 0 */
  float* const* normuon_state;
} muon_options;

/* muon_step with every option; `opt` is a HOST pointer.  muon_step(h, mats, n, lr, mu,
 * nesterov, coeffs, ns_steps, eps, mode, stream) equals muon_step_ex with
 * momentum_form = MUON_MOMENTUM_SGD, weight_decay = 0, cautious = 0. */
MUON_API muon_status muon_step_ex(muon_handle_t h, const muon_matrix* mats, int n,
                                  const muon_options* opt, void* cuda_stream);

/* Newton-Schulz part alone: o_out[i] = X_K of X0 = x_in[i] / (||x_in[i]||_F + eps)
 * for n matrices of shape rows[i] x cols[i].  x_in and o_out are DEVICE pointers
 * of `dtype`; o_out must not overlap any input.  rows, cols, x_in and o_out are
 * HOST arrays of length n.  Other arguments as in muon_step. */
MUON_API muon_status muon_newton_schulz(muon_handle_t h, const void* const* x_in, void* const* o_out,
                               const int64_t* rows, const int64_t* cols, int n,
                               muon_dtype dtype, const float* coeffs, int ns_steps,
                               float eps, muon_mode mode, void* cuda_stream);

/* Allocation-free Newton-Schulz of ONE matrix.  The paper has no counterpart: this
 * entry point exists for callers that may not allocate device memory when they need
 * the update -- runtimes that reserve all device memory for their own pool at
 * start-up, engines that forbid allocation after initialisation, or latency-bound
 * loops where a cudaMalloc (which can synchronise the device) is not acceptable.
 * muon_newton_schulz allocates a workspace on first use; this function instead uses a
 * fixed 32 MiB scratch array compiled into the library and calls no cudaMalloc,
 * cudaFree or other allocating routine.
 *
 * Computes what muon_newton_schulz computes in MUON_MODE_BF16 for a single matrix,
 * with the same kernels in the same order (norm pass, tensor-core steps, export), so
 * the two give the same bits: o_out = Newton-Schulz of x_in / (||x_in||_F + eps).
 * A call enqueues kernels and a 4-byte memset only; it makes no host-to-device copy.
 *  x_in, o_out   DEVICE pointers on the CURRENT device, rows x cols of `dtype`,
 *                row-major, 16-byte aligned, not overlapping; caller-owned.  A
 *                pointer that is not device memory of the current device (host
 *                memory, another GPU's memory) returns MUON_ERR_INVALID_ARG
 *  status        optional DEVICE int (4-byte aligned, current device); if not NULL, a bounded wait
 *                that expires inside a kernel stores 1 there (the caller clears it);
 *                if NULL, such a time-out goes unreported
 *  coeffs, ns_steps, eps, cuda_stream   as in muon_newton_schulz
 * Limit: the matrix must fit the scratch: with s = min(rows, cols), L = max(rows, cols)
 * and r8(v) = v rounded up to a multiple of 8, about 4*s*r8(L) + 4*s*r8(s) bytes plus
 * small tables must stay within 32 MiB (1024x3072 and 1536x1536 fit, 2048x2048 does
 * not).  Larger matrices return MUON_ERR_TOO_LARGE with nothing enqueued.  Argument
 * errors return MUON_ERR_INVALID_ARG, a device that is not compute capability 10.0
 * MUON_ERR_UNSUPPORTED.
 * The first call on a device, with that device current, looks up the array's device
 * address (cudaGetSymbolAddress) and caches it; make that first call before any stream
 * capture.  Every call uses the same array and overwrites it: calls that overlap on the
 * GPU (other streams, other host threads) race and corrupt each other's results, and
 * the host side is not thread-safe.  Every GPU that loads the library's kernels holds
 * the 32 MiB until the process exits. */
MUON_API muon_status muon_newton_schulz_noalloc(const void* x_in, void* o_out, int64_t rows,
                                                int64_t cols, muon_dtype dtype,
                                                const float* coeffs, int ns_steps, float eps,
                                                int* status, void* cuda_stream);

/* Waits for the handle's last enqueued work and returns its device-side status
 * (MUON_OK or MUON_ERR_TIMEOUT), clearing it. */
MUON_API muon_status muon_sync(muon_handle_t h);

/* Diagnostic for the time-out path: enqueues on `cuda_stream` one kernel thread that
 * waits, with the library's bounded wait, on a barrier that nothing ever completes.
 * After limit_ns nanoseconds (0 .. 10e9) it gives up and records a time-out in the
 * handle's device status, which muon_sync or the next call then returns as
 * MUON_ERR_TIMEOUT (and clears).  The GPU context stays usable.  Returns
 * MUON_ERR_INVALID_ARG for a NULL handle or a limit out of range. */
MUON_API muon_status muon_selftest_wait_timeout(muon_handle_t h, int64_t limit_ns, void* cuda_stream);

/* How the Newton-Schulz steps of a bf16-mode call are launched.  Both forms compute
 * every tile with the same products in the same order and the same epilogue
 * arithmetic, so they give the same bits.
 *  MUON_LAUNCH_PER_PHASE   one grouped launch per phase and step (Gram, polynomial,
 *                          update; 3 * ns_steps launches per call)
 *  MUON_LAUNCH_PERSISTENT  one persistent launch for all steps: clusters take work
 *                          items in order from a global counter, and each item waits
 *                          (bounded) until its matrix has finished the previous phase, so
 *                          matrices move through the steps independently and no launch
 *                          boundary separates the phases.  Used when the call's
 *                          matrices fall into at most 8 shape groups (otherwise the
 *                          per-phase form runs)
 *  MUON_LAUNCH_AUTO        (default) the persistent launch when one Newton-Schulz step
 *                          over the call's matrices is less than 1e12 algorithmic flops
 *                          (the small sets, where launch boundaries and phase tails weigh
 *                          most), the per-phase launches otherwise */
typedef enum {
  MUON_LAUNCH_AUTO = 0,
  MUON_LAUNCH_PER_PHASE = 1,
  MUON_LAUNCH_PERSISTENT = 2
} muon_launch_mode;

/* Sets the handle's launch form for later calls (no device work).  Returns
 * MUON_ERR_INVALID_ARG for a NULL handle or an unknown mode. */
MUON_API muon_status muon_set_launch_mode(muon_handle_t h, muon_launch_mode mode);

/* Diagnostic for the abort path of the persistent launch: in the handle's next
 * persistent launch, the first polynomial item of the call's first matrix (in the
 * library's group order) waits for a count that is never reached, with a limit of
 * limit_ns nanoseconds (1 .. 10e9).  When it runs out, the kernel records a time-out in
 * the handle's device status; every other item that waits sees the status and gives up,
 * and the launch returns with its copies and tensor-core work drained.  muon_sync or
 * the next call then returns MUON_ERR_TIMEOUT (and clears it); the handle keeps
 * working.  No device work by itself.  Returns MUON_ERR_INVALID_ARG for a NULL handle
 * or a limit out of range. */
MUON_API muon_status muon_selftest_stall_persistent(muon_handle_t h, int64_t limit_ns);

/* Diagnostic for the debug mode's guard check: overwrites one byte of the last guard
 * band of the handle's workspace (synchronously, with cudaMemset), so that the next
 * call returns MUON_ERR_CORRUPT.  Returns MUON_ERR_INVALID_ARG for a NULL handle, a
 * handle not in debug mode or one without a workspace yet. */
MUON_API muon_status muon_selftest_corrupt_guard(muon_handle_t h);

/* Diagnostic for the allocation-failure path: the next time the handle must allocate
 * its workspace (a call with a new list of shapes or mode that needs more than the
 * handle holds), the allocation reports failure as if cudaMalloc had failed, once.
 * That call returns MUON_ERR_OOM with nothing enqueued, the handle then holds no
 * workspace, and the next call allocates normally.  No device work.  Returns
 * MUON_ERR_INVALID_ARG for a NULL handle. */
MUON_API muon_status muon_selftest_fail_next_alloc(muon_handle_t h);

/* Bytes of device workspace the handle currently holds. */
MUON_API int64_t muon_workspace_bytes(muon_handle_t h);

/* Number of kernel launches the last muon_step / muon_newton_schulz enqueued. */
MUON_API int muon_last_launch_count(muon_handle_t h);

/* Kernel kinds reported by muon_profile_read. */
typedef enum {
  MUON_KIND_MOMENTUM_NORM = 0,  /* momentum + Nesterov + Frobenius norm pass */
  MUON_KIND_GRAM = 1,           /* A = X X^T (scaled) */
  MUON_KIND_POLY = 2,           /* B = b A + c A^2 */
  MUON_KIND_UPDATE = 3,         /* X' = a X + B X */
  MUON_KIND_APPLY = 4,          /* separate W -= lr*scale*O pass, or the export of O */
  MUON_KIND_UPDATE_APPLY = 5,   /* last update with W -= lr*scale*O fused into its epilogue */
  MUON_KIND_NS_PERSISTENT = 6,  /* every Newton-Schulz step in one persistent launch */
  MUON_KIND_COUNT = 7
} muon_kernel_kind;

/* Per-launch timing: while enabled, every launch of the handle is bracketed by two
 * CUDA events recorded on the launch stream.  Adds two event records per launch; no
 * effect on results. */
MUON_API muon_status muon_profile_enable(muon_handle_t h, int enable);

/* Waits for the recorded events and writes, per kernel kind (indexed by
 * muon_kernel_kind, arrays of length MUON_KIND_COUNT), the summed device time in
 * milliseconds and the number of launches since the last read; then resets the
 * totals.  ms and launches are HOST arrays. */
MUON_API muon_status muon_profile_read(muon_handle_t h, double* ms, int64_t* launches);

/* Waits for outstanding work, frees the workspace and the handle.  Returns the
 * pending device-side status.  NULL is accepted and returns MUON_OK. */
MUON_API muon_status muon_destroy(muon_handle_t h);

/* Static description of a status code. */
MUON_API const char* muon_status_string(muon_status s);

/* Detail of the last error on this handle (empty string if none).  The pointer
 * stays valid until the next call on the handle. */
MUON_API const char* muon_last_error(muon_handle_t h);

#ifdef __cplusplus
}
#endif

#endif /* MUON_B200_MUON_H */
