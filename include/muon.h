/*
 * muon.h -- C ABI of the B200 (sm_100a) Muon update library.
 *
 * The Muon optimizer step of the NanoGPT speedrun: each hidden weight
 * matrix's Nesterov-momentum update is orthogonalised by Newton-Schulz
 * iteration and then applied ("NanoGPT Speedrun: The Ultimate Guide to
 * Pushing LLM Training Efficiency to Its Limits", section "Optimizer and
 * Training Strategy Tuning"); the update is replaced by its nearest
 * semi-orthogonal matrix through five Newton-Schulz steps ("The NanoGPT
 * speedrun", paragraph "Six records account for most of the speedup",
 * record #3).  The iteration is X <- aX + (bA + cA^2)X with A = X X^T, on the
 * Frobenius-normalised update, transposed so that rows <= cols.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Pointer arrays (X_ptrs, params, grads, ...) are HOST arrays of DEVICE
 *   pointers.  Each matrix is one contiguous row-major buffer owned by the
 *   caller; every device pointer must be 16-byte aligned.
 * - `stream` is a cudaStream_t (NULL = legacy default stream).  All calls are
 *   asynchronous on it: they validate, enqueue kernels and return.
 * - Argument and shape errors return a negative muon_status synchronously,
 *   before anything is enqueued; nothing is modified.  muon_last_error()
 *   then holds a message (thread-local).
 * - Errors found on the device (a bounded wait that ran out) are recorded in
 *   a per-(device, stream) status word and reported by muon_get_status().
 * - The library owns a workspace per (device, stream), grown on demand with
 *   stream-ordered allocation and freed by muon_release().  Calls that share a
 *   stream share the workspace; calls on different streams do not.
 * - Results are deterministic: no floating-point atomics anywhere, fixed
 *   reduction orders, so a rerun on the same inputs is bit-identical.
 */
#ifndef MUON_B200_H
#define MUON_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Storage / arithmetic type of muon_ns_orthogonalize's matrices. */
typedef enum {
  MUON_BF16 = 0, /* bf16 storage; bf16 tensor-core operands, fp32 accumulate,
                    X kept between steps as the pair bf16 hi + int8 residual
                    (see muon_bx_bf16), about 16 significant bits */
  MUON_FP32 = 1  /* fp32 storage; fp32 SIMT FMA verification path */
} muon_dtype;

typedef enum {
  MUON_OK = 0,
  MUON_ERR_ARG = -1,            /* null pointer, bad count/steps/dtype, misaligned */
  MUON_ERR_SHAPE = -2,          /* non-positive or too large dimensions */
  MUON_ERR_CUDA = -3,           /* a CUDA runtime call failed (message has the name) */
  MUON_ERR_ALLOC = -4,          /* workspace allocation failed */
  MUON_ERR_DEVICE_TIMEOUT = -5, /* a bounded device-side wait ran out */
  MUON_ERR_UNSUPPORTED = -6     /* device is not sm_100 or feature not built */
} muon_status;

/*
 * muon_ns_orthogonalize -- Newton-Schulz orthogonalisation of a batch, in place.
 *
 * Source: "The NanoGPT speedrun", paragraph "Six records account for most of
 * the speedup" (nearest semi-orthogonal matrix through five Newton-Schulz
 * steps); the form X <- aX + (bA + cA^2)X is the library's specification.
 *
 * batch   number of matrices (>= 0; 0 is a no-op).
 * m, n    rows and columns of EVERY matrix (1 <= m, n <= 32768).  When m > n
 *         the matrix is processed as its transpose (a view; no copy is made
 *         in the caller's memory) and written back in its own layout.
 * X_ptrs  host array of `batch` device pointers, each to an m x n row-major
 *         matrix of bf16 (dtype MUON_BF16) or fp32 (MUON_FP32).  On return
 *         (stream order) each holds NS(X / (||X||_F + 1e-7)) after `steps`
 *         iterations, rounded to the storage type.  (MUON_BF16, steps >= 1:
 *         with m <= n and n % 8 == 0 the last GEMM stores the fp32 result
 *         rounded to bf16 straight into the first 160 buffers of each launch;
 *         the others are written from the bf16 + int8 pair by a separate
 *         pass, which can differ from that rounding by one bf16 unit.)
 * a, b, c coefficients of the quintic; the speedrun's are 3.4445, -4.7750, 2.0315.
 * steps   number of iterations T (0 <= steps <= 100; 0 = normalise only).
 * dtype   a muon_dtype.
 * Returns MUON_OK or a negative muon_status.
 */
int muon_ns_orthogonalize(int batch, int m, int n, void* const* X_ptrs, float a, float b,
                          float c, int steps, int dtype, void* stream);

/*
 * muon_ns_orthogonalize_schedule -- muon_ns_orthogonalize with its own
 * coefficient triple for every step.
 *
 * Source: "The NanoGPT speedrun", paragraph "Reading guide", names Polar
 * Express polynomials among the later refinements of the same update: the
 * iteration keeps its form, X <- a_t X + (b_t A + c_t A^2) X, but the
 * polynomial changes from step to step.  The pages give no coefficients;
 * the caller supplies them.
 *
 * coeffs  HOST array of 3 * steps floats, read during the call: step t
 *         (t = 0 .. steps-1, in that order) uses a_t = coeffs[3t],
 *         b_t = coeffs[3t+1], c_t = coeffs[3t+2].  May be NULL only when
 *         steps == 0.  Every value must be finite.
 * All other arguments, the layout, the in-place result and the errors are
 * those of muon_ns_orthogonalize (a NULL table with steps > 0 or a
 * non-finite value returns MUON_ERR_ARG before any work).  A table that
 * repeats one triple gives exactly muon_ns_orthogonalize's result.
 */
int muon_ns_orthogonalize_schedule(int batch, int m, int n, void* const* X_ptrs,
                                   const float* coeffs, int steps, int dtype, void* stream);

/*
 * muon_ns_orthogonalize_static -- muon_ns_orthogonalize (bf16 storage, the
 * tensor-core path) for callers that cannot allocate device memory.
 *
 * The source pages have no counterpart for this call; it exists for library
 * users.  Some callers cannot call cudaMalloc (or any allocator) where they
 * call us: plug-ins whose host engine hands out all device memory up front and
 * forbids allocation inside its execution callback, processes that run under a
 * fixed, pre-planned memory budget, and latency-critical loops that must never
 * wait on, or fail in, an allocator.  This call allocates nothing: its
 * workspace is a static device array of 24 MiB that the library defines, so
 * every GPU that loads the library holds those 24 MiB until the process exits.
 *
 * Arguments and result are those of muon_ns_orthogonalize with dtype
 * MUON_BF16 (X_ptrs: host array of device pointers to bf16 m x n matrices,
 * overwritten in place), plus:
 * status_dev  DEVICE pointer to an int owned by the caller, or NULL.  If a
 *             bounded device-side wait runs out during this call, the kernels
 *             store MUON_ERR_DEVICE_TIMEOUT there (only if it holds 0; the
 *             library never clears it).  With NULL the code goes to a slot of
 *             the static array, which each call clears first, and is not
 *             reported.
 * Limits: the workspace of the batch -- 5*batch*m*n + 4*batch*min(m,n)^2
 * bytes with the row strides of the m x n buffers rounded up to 16 elements
 * and those of the square ones to 8, plus a few KiB -- must fit in the
 * 24 MiB; larger requests return MUON_ERR_SHAPE with the byte counts and do
 * nothing.  One 768 x 3072 matrix (about 13.5 MiB) fits; so do four 768 x 768
 * matrices.
 * Sharing: every call on every stream of a device uses the same array and
 * leaves its last contents there.  No byte of it needs to start at zero (each
 * call writes everything it later reads).  Calls whose work overlaps on the
 * GPU -- on different streams, or from different host threads -- race on the
 * array and corrupt each other's results: order them on one stream or with
 * events.
 * Set-up: the first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current, and caches it; make that
 * first call before any stream capture begins.  muon_release() forgets the
 * cached address (the next call looks it up again), which is what a context
 * re-created after cudaDeviceReset needs.
 * If kernel timing (muon_profile_begin) is on, this call's launches are not
 * timed, so no CUDA event objects are created on its behalf.
 */
int muon_ns_orthogonalize_static(int batch, int m, int n, void* const* X_ptrs, float a, float b,
                                 float c, int steps, int* status_dev, void* stream);

/*
 * muon_step -- one full Muon optimizer step over `count` hidden matrices.
 *
 * Source: "NanoGPT Speedrun: The Ultimate Guide...", section "Optimizer and
 * Training Strategy Tuning" (orthogonalise after a Nesterov-momentum update;
 * hidden matrices only) and "The NanoGPT speedrun", record #3 (T = 5).
 *
 * Per matrix i with shape (r, s) = (shapes[2i], shapes[2i+1]):
 *   buf' = beta*buf + (1-beta)*g                       (fp32, written in place)
 *   u    = (1-beta)*g + beta*buf'   if nesterov, else buf'
 *   X0   = u / (||u||_F + 1e-7), transposed when r > s
 *   X    = NS(X0) with (a,b,c) = (3.4445, -4.7750, 2.0315), `steps` iterations
 *   W'   = (W - fl(lr*wd)*W) - fl(lr*scale)*O,   O = X in (r, s) layout,
 *          scale = sqrt(max(1, r/s)) in fp32      (fp32, written in place)
 * params         host array of device pointers to fp32 W (r x s, row-major).
 * grads          host array of device pointers to bf16 g (r x s).
 * momentum_bufs  host array of device pointers to fp32 buf (r x s).
 * shapes         host array of 2*count int64: rows, cols of each matrix.
 * Matrices of equal (min, max) dimensions are batched into one group; any mix
 * of shapes is accepted.  With steps >= 1 the update of a weight whose column
 * count is a multiple of 4 (among the first 160 matrices of each launch of the
 * last step) is applied inside the last Newton-Schulz GEMM, with O its fp32
 * value; the others are applied by a separate pass from O carried as the
 * bf16 + int8 pair.  Both stay within the same tolerance of the definition.
 * Returns MUON_OK or a negative muon_status.
 */
int muon_step(int count, float* const* params, const void* const* grads,
              float* const* momentum_bufs, const int64_t* shapes, float beta, int nesterov,
              float lr, float wd, int steps, void* stream);

/* Option bits of muon_step_ex, muon_apply_ex and muon_bx_apply_bf16. */
#define MUON_CAUTIOUS_WD 1 /* cautious weight decay (below) */

/*
 * muon_step_ex -- muon_step with the later refinements of the same update.
 *
 * Source: "The NanoGPT speedrun", paragraph "Reading guide", names Polar
 * Express polynomials, NorMuon's per-neuron rescale and cautious weight decay
 * among the refinements that tune the Muon update; the pages give no
 * formulas, so the library reads them as follows.
 *
 * schedule: NULL for the default triple (3.4445, -4.7750, 2.0315) at every
 *   step, else a HOST array of 3 * steps floats, (a_t, b_t, c_t) for step
 *   t = 1 .. steps, as in muon_ns_orthogonalize_schedule (Polar Express
 *   reading: the same iteration with per-step coefficients).  Every value
 *   must be finite (else MUON_ERR_ARG).
 *
 * flags & MUON_CAUTIOUS_WD: the decay term fl(lr*wd)*W is applied only to the
 *   elements where W and the update O have the same sign (W*O > 0); elsewhere
 *   W' = fl(W - fl(lr*scale)*O).  Same fp32 operation order otherwise.
 * neuron_state != NULL: NorMuon's per-neuron rescale.  neuron_state is a HOST
 *   array of `count` DEVICE pointers, each to `rows` fp32 values (one per row
 *   of W, the caller's layout; zeros before the first step), updated in place.
 *   After the iteration, with O the update in W's layout:
 *     r_i   = mean over row i of O^2
 *     v_i'  = fl(fl(beta2*v_i) + fl(fl(1-beta2) * fl32(r_i)))      (the state)
 *     f_i   = 1 / sqrt(v_i' + 1e-10)
 *     O_i  <- O_i * f_i * g,   g = ||O||_F / ||diag(f) O||_F
 *   so the update keeps its Frobenius norm and only its split over the rows
 *   (neurons) changes; then the apply as in muon_step.  The row sums of O^2
 *   are taken over O rounded to bf16 (each within a relative 2^-7 + 2^-14 of
 *   the exact sum), in a fixed order (fp32 within a thread, fp64 across
 *   threads); the factor f_i g is rounded to fp32 and multiplies O in fp32.
 *   This path applies every update in the separate pass.  beta2 in [0, 1].
 * schedule == NULL, neuron_state == NULL and flags == 0 is exactly muon_step.
 * Returns MUON_OK or a negative muon_status (unknown flag bits: MUON_ERR_ARG).
 */
int muon_step_ex(int count, float* const* params, const void* const* grads,
                 float* const* momentum_bufs, const int64_t* shapes, float beta, int nesterov,
                 float lr, float wd, int steps, const float* schedule, int flags,
                 float* const* neuron_state, float beta2, void* stream);

/*
 * muon_momentum -- the momentum stage of muon_step on its own.
 *
 * Source: "Nesterov momentum" in "NanoGPT Speedrun: The Ultimate Guide...",
 * section "Optimizer and Training Strategy Tuning" (lerp reading, as in
 * muon_step).  Writes buf' in place, bit-exact with the fp32 order
 *   buf' = fl(fl(beta*buf) + fl(fl(1-beta)*g)),
 * and, if `sumsq_out` is not NULL, sumsq_out[i] = sum of u^2 over matrix i
 * (fp32, fixed two-stage order; u as in muon_step).  sumsq_out is a DEVICE
 * pointer to `count` floats.
 */
int muon_momentum(int count, const void* const* grads, float* const* momentum_bufs,
                  const int64_t* shapes, float beta, int nesterov, float* sumsq_out,
                  void* stream);

/*
 * muon_apply -- the apply stage of muon_step on its own.
 *
 * W' = fl(fl(W - fl(fl(lr*wd)*W)) - fl(fl(lr*scale)*O)), scale as in
 * muon_step, all fp32 with no fused multiply-add.  updates[i] is a device
 * pointer to the fp32 update O (r x s, same layout as W).
 */
int muon_apply(int count, float* const* params, const float* const* updates,
               const int64_t* shapes, float lr, float wd, void* stream);

/*
 * muon_apply_ex -- muon_apply with the options of muon_step_ex.
 *
 * flags & MUON_CAUTIOUS_WD: decay only where W*O > 0 (as in muon_step_ex).
 * row_scale: NULL, or a HOST array of `count` DEVICE pointers, each to `rows`
 *   fp32 factors; row r of matrix i's update is first multiplied by
 *   row_scale[i][r] in fp32 (the per-neuron factors of muon_step_ex).
 * Otherwise exactly muon_apply.
 */
int muon_apply_ex(int count, float* const* params, const float* const* updates,
                  const int64_t* shapes, float lr, float wd, int flags,
                  const float* const* row_scale, void* stream);

/*
 * Stage calls on contiguous bf16 batches (the tensor-core kernels of the
 * iteration, exposed for testing and for callers that run their own loop).
 * Every pointer is a DEVICE pointer to `batch` contiguous row-major matrices;
 * m and k (or n) must be multiples of 8 (16-byte row strides for the bulk
 * tensor copies).
 *
 * muon_gram_bf16:  A = X X^T          X: batch x m x k bf16, A: batch x m x m bf16.
 *                  Only the 256x256 tiles on or above the diagonal are
 *                  computed; A is exactly symmetric.
 * muon_poly_bf16:  B = b*A + c*(A A)   A, B: batch x m x m bf16, A symmetric.
 * muon_bx_bf16:    X' = a*X + B X, with X carried as the pair the iteration
 *                  keeps between steps (about 16 significant bits):
 *                    X = hi + q * 2^(E - 15),  hi = bf16(X) (nearest even),
 *                    E the exponent of hi (hi = 1.f * 2^E), q an int8 with
 *                    q = round-to-nearest-even((X - hi) / 2^(E-15)) clamped
 *                    to [-128, 127]; where hi is 0, subnormal or below
 *                    2^-111, q is ignored (X = hi).  |X - value| <= 2^(E-16)
 *                    (2^(E-15) when X lies exactly halfway above hi).
 *                  B: m x m bf16; Xhi: hi of X (bf16), the operand; Xlo: q of
 *                  X (int8, batch x m x n, n a multiple of 16), read then
 *                  overwritten by q of X'; Xhi_out: hi of X' (must not alias
 *                  Xhi).  m <= n.
 */
int muon_gram_bf16(int batch, int m, int k, const void* X, void* A, void* stream);
int muon_poly_bf16(int batch, int m, const void* A, void* B, float b, float c, void* stream);
int muon_bx_bf16(int batch, int m, int n, const void* B, const void* Xhi, void* Xlo,
                 void* Xhi_out, float a, void* stream);

/*
 * muon_bx_apply_bf16 -- the last Newton-Schulz GEMM of muon_step with the
 * update applied to the weights in its epilogue, on its own.
 *
 * Source: "The NanoGPT speedrun", record #3 (the orthogonalised update is
 * "then scaled and applied"); the apply's operation order is muon_apply's.
 * muon_step runs exactly this launch for its last step; the call exists so
 * that the fused epilogue can be checked bit for bit.
 *
 * Per matrix i (X_i = the pair Xhi_i, Xlo_i as in muon_bx_bf16, m x n, m <= n):
 *   O    = fl(a*X + acc),  acc = B_i * hi_i accumulated in fp32 (tensor cores),
 *          one rounding after a fused multiply-add
 *   W'   = fl(fl(W - fl(fl(lr*wd)*W)) - fl(fl(lr*scale)*O_W)),  no FMA,
 *   O_W  = O (tall == 0, W is m x n) or O^T (tall != 0, W is n x m),
 *   scale = sqrt(max(1, rows/cols)) of W's shape, in fp32;
 *   with flags & MUON_CAUTIOUS_WD the fl(lr*wd)*W term only where W*O > 0.
 * batch   number of matrices (>= 0).
 * ldx     row stride (elements) of Xhi and Xlo; >= n and a multiple of 16.
 *         Matrix i starts at element i*m*ldx.
 * B       DEVICE pointer, batch x m x ldb bf16 (row stride ldb >= m, a multiple
 *         of 8; matrix stride m*ldb).
 * Xhi     DEVICE pointer, bf16 hi of X; read only.
 * Xlo     DEVICE pointer, int8 q of X.  Read; overwritten with q of X' for the
 *         matrices that take the separate pass (below).  For those the bulk
 *         copies write whole 16-byte units, so when n is not a multiple of 16
 *         the row's padding bytes n .. (n rounded up to 16) - 1 may change
 *         too (they are inside the ldx-wide row; nothing past it is written).
 * W_ptrs  HOST array of `batch` DEVICE pointers to fp32 W (row-major,
 *         contiguous, 16-byte aligned), updated in place.
 * The first 160 matrices whose W has a column count that is a multiple of 4
 * are updated inside the GEMM epilogue with O as above.  The others (past
 * the first 160, or W columns not a multiple of 4) get X' as the pair (hi in
 * the library's workspace, q in Xlo) and are updated by the apply pass from
 * the pair's value, as muon_step does for them.
 * Returns MUON_OK or a negative muon_status.
 */
int muon_bx_apply_bf16(int batch, int m, int n, int ldx, const void* B, int ldb, const void* Xhi,
                       void* Xlo, float* const* W_ptrs, int tall, float a, float lr, float wd, int flags,
                       void* stream);

/*
 * muon_get_status -- synchronise `stream`, then return and clear the device
 * status word of (current device, stream): MUON_OK or MUON_ERR_DEVICE_TIMEOUT,
 * or MUON_ERR_CUDA if the synchronisation itself failed.
 */
int muon_get_status(void* stream);

/* Thread-local message of the last failed call on this thread ("" if none). */
const char* muon_last_error(void);

/*
 * muon_release -- synchronise the device and free every workspace and status
 * word the library holds on the current device.  Safe to call at any time
 * outside stream capture; later calls re-allocate on demand.  It also forgets
 * the cached address of muon_ns_orthogonalize_static's array on this device,
 * so call it after a device reset (cudaDeviceReset) before using the library
 * again on that device.
 */
int muon_release(void);

/*
 * muon_workspace_bytes -- device memory the library holds for (current
 * device, stream): its workspace plus the status word, or 0 if it holds
 * none.  `bytes` is a HOST pointer.  No synchronisation.  The allocation-free
 * call (muon_ns_orthogonalize_static) never adds to it.
 */
int muon_workspace_bytes(void* stream, long long* bytes);

/*
 * muon_set_wait_timeout_ms -- limit of every device-side wait (default 2000 ms).
 * A wait that runs out records MUON_ERR_DEVICE_TIMEOUT, the kernel drains
 * what it has in flight, frees its tensor memory and returns.
 */
int muon_set_wait_timeout_ms(int ms);

/*
 * muon_set_fault_injection -- host-controlled fault injection for tests.
 * mode 0: off.  mode 1: the next tensor-core GEMM launch withholds one
 * operand copy, so one device wait runs out and the timeout path is taken.
 * The mode resets to 0 after one launch.
 */
int muon_set_fault_injection(int mode);

/*
 * Kernel timing for measurement harnesses (off by default).
 *
 * muon_profile_begin: from now on every kernel this library launches is
 *   bracketed by two CUDA events recorded on the stream it is launched on
 *   (previous records are discarded).
 * muon_profile_end: stop recording, wait for the recorded events, and write,
 *   for each kernel kind k < kinds, the summed device time in milliseconds to
 *   total_ms[k] and the number of launches to launches[k] (host arrays of
 *   `kinds` entries; either may be NULL).  Returns the total launch count or a
 *   negative muon_status.
 */
typedef enum {
  MUON_KERNEL_FLAT = 0, /* momentum / sum of squares (flat, 128-bit vectors) */
  MUON_KERNEL_CAST = 1, /* normalise + transpose + cast to the iteration layout */
  MUON_KERNEL_GRAM = 2, /* tensor cores: A = X X^T */
  MUON_KERNEL_POLY = 3, /* tensor cores: B = bA + cA^2 */
  MUON_KERNEL_BX = 4,   /* tensor cores: X' = aX + BX */
  MUON_KERNEL_OUT = 5,  /* apply / write-back */
  MUON_KERNEL_SIMT = 6, /* fp32 verification GEMMs */
  MUON_KERNEL_SUMS = 7, /* per-matrix sums of partials */
  MUON_KERNEL_PREP = 8, /* momentum + Nesterov blend written as the bf16 + int8 pair (transposing) */
  MUON_KERNEL_SCALE = 9, /* per-matrix 1 / (||u||_F + eps) */
  MUON_KERNEL_BX_APPLY = 10, /* tensor cores: the last step's X' = aX + BX applied to W */
  MUON_KERNEL_NORM = 11,     /* per-neuron rescale: row norms, state, factors */
  MUON_KERNEL_KINDS = 12
} muon_kernel_kind;

int muon_profile_begin(void);
int muon_profile_end(int kinds, double* total_ms, int* launches);

/* Library version, major*10000 + minor*100 + patch. */
int muon_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MUON_B200_H */
