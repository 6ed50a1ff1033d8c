/*
 * muon_b200.h -- C ABI of the B200 (sm_100a) Muon optimizer step.
 *
 * The operation, as the pages define it:
 *
 *   momentum  m <- beta * m + g
 *             ("14 - modded-nanogpt: the Speedrun Community", section 3 "Muon",
 *              muon_step pseudocode)
 *   Nesterov  u = g + beta * m   (nesterov != 0), else u = m
 *             ("NanoGPT Speedrun" README, practices list after the Newton-Schulz
 *              listing: Nesterov momentum inside the update, orthogonalisation after
 *              the momentum; the page's full formula was lost, this is the reading)
 *   NS        X = u / (||u||_F + eps), short side on the rows, then per iteration k
 *             A = X X^T,  B = b_k A + c_k A A,  X = a_k X + B X,  transpose back
 *             ("NanoGPT Speedrun" README, zeroth_power_via_newtonschulz5 listing;
 *              a row per iteration covers the "Polar Express" schedules named in the
 *              same README's technique list)
 *   update    W <- W (1 - lr * wd) - lr * shape_scale * O
 *             (decoupled weight decay from the old W; the README's record list names
 *              "standard weight decay" and "Muon custom sizing" without formulas)
 *
 * Layout: every matrix is row-major, element (r, c) at base + r * ld + c, with
 * ld >= cols counted in elements.  Gradients and momentum are fp32; the parameter
 * is fp32 or bf16; the optional O output is dense fp32 (ld = cols).
 *
 * Ownership: the caller allocates and owns every buffer, including the workspace,
 * and keeps them alive until the work queued on `stream` has finished.  The library
 * allocates no device memory; the one exception is the fixed static array that
 * muon_newton_schulz_static works in, which the module holds on every GPU that loads
 * it (MUON_STATIC_SCRATCH_BYTES).  `param` and `momentum` are updated in place; `grad`
 * is only read.  Buffers of different roles (and of different matrices) must not
 * overlap.  All device pointers must belong to the current CUDA device.
 *
 * Execution: asynchronous on `stream` (a cudaStream_t; NULL is the legacy default
 * stream).  No call synchronises the host except muon_device_status.  The first
 * call with a new set of descriptors plans the work (host only, microseconds) and
 * caches the plan; later calls with identical descriptors reuse it.  muon_step and
 * muon_newton_schulz queue kernel launches only (arguments by value, no copies, no
 * host synchronisation), so they can be captured in a CUDA graph; every buffer and
 * the workspace must then stay in place for as long as the graph is replayed.
 *
 * Errors: every entry point returns a muon_status_t.  On a validation error
 * nothing is launched and no buffer is touched.  A failed CUDA launch returns
 * MUON_ERR_CUDA.  Device-side waits are bounded: a wait that runs out records
 * MUON_ERR_TIMEOUT in the workspace's status word (read it with
 * muon_device_status) and the kernel returns instead of hanging.
 *
 * Numerics: Newton-Schulz runs with bf16 tensor-core operands and fp32
 * accumulation; X is carried between iterations as a bf16 hi plus an 8-bit
 * fixed-point residual (15 significant bits, see muon_scratch_view_t), so that the
 * a*X term does not lose the precision a single bf16 copy would.  Momentum and the
 * update are fp32.
 * Finite inputs with ||u||_F below about 1e17 are required (the Gram of the
 * unscaled bf16 input is formed before the 1/||u||^2 factor is applied).
 */
#ifndef MUON_B200_H
#define MUON_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MUON_ABI_VERSION 4
#define MUON_MAX_NS_STEPS 16

typedef enum {
  MUON_OK = 0,
  MUON_ERR_INVALID_ARG = 1,        /* null pointer, n < 1, bad hyperparameter, overlap */
  MUON_ERR_ALIGNMENT = 2,          /* a pointer is not aligned to its element size */
  MUON_ERR_UNSUPPORTED_SHAPE = 3,  /* rows/cols < 1, ld < cols, or a side above 2^24 */
  MUON_ERR_UNSUPPORTED_DTYPE = 4,  /* param_dtype not MUON_F32 / MUON_BF16 */
  MUON_ERR_WORKSPACE_TOO_SMALL = 5,/* not even the largest single matrix fits */
  MUON_ERR_CUDA = 6,               /* a CUDA runtime call or launch failed */
  MUON_ERR_TIMEOUT = 7,            /* device status only: a bounded wait ran out */
  MUON_ERR_NO_DEVICE = 8,          /* current device is not an sm_100 GPU */
  MUON_ERR_STATIC_SCRATCH_LIMIT = 9, /* muon_newton_schulz_static: a matrix needs more
                                       scratch than MUON_STATIC_SCRATCH_BYTES */
  MUON_ERR_NONFINITE = 10          /* device status only: a Newton-Schulz input u held a NaN
                                      or an infinity (the values propagate into that
                                      matrix's results; no other matrix is affected) */
} muon_status_t;

typedef enum { MUON_F32 = 0, MUON_BF16 = 1 } muon_dtype_t;

/* One 2-D parameter.  80 bytes, no implicit padding. */
typedef struct {
  void*        param;        /* in/out: W, param_dtype, [rows x ld_param]; may be NULL
                                only in muon_newton_schulz */
  const float* grad;         /* in: g (muon_step) or G (muon_newton_schulz), fp32 [rows x ld_grad] */
  float*       momentum;     /* in/out: m, fp32 [rows x ld_mom]; ignored by muon_newton_schulz */
  float*       out_update;   /* optional out: O = NS(u), dense fp32 [rows x cols]; NULL skips it */
  int64_t      rows;
  int64_t      cols;
  int64_t      ld_param;     /* row stride of param, elements */
  int64_t      ld_grad;      /* row stride of grad, elements */
  int64_t      ld_mom;       /* row stride of momentum, elements */
  int32_t      param_dtype;  /* muon_dtype_t */
  float        shape_scale;  /* multiplier on lr; <= 0 selects sqrt(max(1, rows / cols)) */
} muon_matrix_t;

/*
 * Where one matrix's scratch lives inside the workspace (diagnostics and tests).
 * X is carried between iterations as hi + lo: hi = bf16(x) (the tensor-core operand,
 * rounded to nearest even) and lo = one byte per element holding the residual in fixed
 * point on the fp32 bit patterns.  With d = bits(x) - bits(hi) as signed 32-bit integers
 * (|d| <= 2^15, since rounding to bf16 rounds the bit pattern to a multiple of 2^16), the
 * stored byte is (d + 2^15 + 2^8) >> 9, unsigned, 0 .. 128; x is rebuilt as the float with
 * bits bits(hi) + 2^9 * (byte - 64), within 2^8 fp32 ulps (relative 2^-15) of the fp32 value.
 */
typedef struct {
  uint64_t x_hi_offset[2];   /* bf16 [rows x x_ld]: ping-pong high parts of X */
  uint64_t x_lo_offset;      /* uint8 [rows x x_lo_ld]: low part of X, see above */
  uint64_t a_offset;         /* bf16 [m x a_ld]: A = X X^T of the latest iteration */
  uint64_t b_offset;         /* bf16 [m x a_ld]: B = b A + c A A of the latest iteration */
  uint64_t scale_offset;     /* fp32: 1 / (||u||_F + eps) */
  uint64_t norm_offset;      /* fp32: ||u||_F */
  int64_t  x_ld;             /* elements */
  int64_t  x_lo_ld;          /* bytes (= elements) */
  int64_t  a_ld;             /* elements */
  int32_t  wave;             /* matrices are processed in waves that reuse the workspace */
  int32_t  transposed;       /* 1 when rows > cols (X is the transpose of the stored matrix) */
} muon_scratch_view_t;

/* Version of this ABI (MUON_ABI_VERSION of the library that was loaded). */
int muon_abi_version(void);

/* Static, human-readable text for a status code. */
const char* muon_status_str(int status);

/*
 * Bytes of workspace that lets muon_step / muon_newton_schulz process all n
 * matrices at full speed.  A smaller workspace is accepted as long as the
 * largest single matrix fits; the matrices are then processed in more waves.
 */
muon_status_t muon_workspace_size(const muon_matrix_t* mats, int n, size_t* bytes);

/*
 * Zeroes the device status word at the start of a workspace (queued on `stream`).
 * Call once after allocating a workspace; the word is sticky until cleared again.
 */
muon_status_t muon_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/*
 * One Muon step on n matrices (one grouped launch sequence).
 *   lr, beta, weight_decay : finite; beta in [0, 1]; lr >= 0; weight_decay >= 0
 *   nesterov               : 0 or 1
 *   ns_steps, coeffs       : 1 <= ns_steps <= MUON_MAX_NS_STEPS; coeffs is a HOST array of
 *                            ns_steps rows (a, b, c), row k used in iteration k
 *   eps                    : added to the Frobenius norm (the page uses 1e-7); > 0
 *   workspace              : device memory, 256-byte aligned, from muon_workspace_size
 */
muon_status_t muon_step(const muon_matrix_t* mats, int n, float lr, float beta,
                        float weight_decay, int nesterov, int ns_steps, const float* coeffs,
                        float eps, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Newton-Schulz alone (zeroth_power_via_newtonschulz5 with a coefficient table):
 * reads mats[i].grad as G and writes NS(G) to mats[i].out_update (required here).
 * param and momentum are ignored and left untouched.
 */
muon_status_t muon_newton_schulz(const muon_matrix_t* mats, int n, int ns_steps,
                                 const float* coeffs, float eps, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* Scratch placement of matrix `index` for this descriptor set and workspace size. */
muon_status_t muon_scratch_view(const muon_matrix_t* mats, int n, int index,
                                size_t workspace_bytes, muon_scratch_view_t* view);

/*
 * Waits for `stream`, then reads the workspace's device status word into *device_status
 * and *where (may be NULL):
 *   MUON_OK
 *   MUON_ERR_TIMEOUT    a bounded device-side wait ran out; *where = the wait site
 *   MUON_ERR_NONFINITE  the elementwise pass found a NaN or an infinity in u (muon_step)
 *                       or G (muon_newton_schulz); *where = the index, in that call's
 *                       descriptor array, of a matrix that held one
 * The first event recorded wins; the word is sticky until muon_workspace_init clears it.
 * The pages define no status reporting (the step is a plain function there); the
 * workspace argument replaces a per-stream query, since every call owns its workspace.
 */
muon_status_t muon_device_status(const void* workspace, void* stream, int32_t* device_status,
                                 int32_t* where);

/*
 * Waits for `stream`, then reads how many non-finite values of u (or G) the elementwise
 * passes that used this workspace have counted since muon_workspace_init cleared it.
 */
muon_status_t muon_nonfinite_count(const void* workspace, void* stream, int64_t* count);

/*
 * Budget of every device-side wait, in microseconds (default 2,000,000 = 2 s).  A
 * value <= 0 restores the default.  Takes effect for launches queued afterwards.
 * Waits on the way out of a kernel that gave up (for copies and MMAs already in
 * flight) always get at least 2 s.
 */
muon_status_t muon_set_wait_timeout_us(int64_t us);

/*
 * Per-kernel timing for diagnostics and benchmarks.  Between muon_profile_begin and
 * muon_profile_end every launch the library queues is bracketed by a pair of CUDA
 * events recorded on its own stream.  muon_profile_end waits for those events and
 * returns, per kernel kind (MUON_KIND_*), the summed device time in milliseconds and
 * the number of launches.  Timing state is per process; calls are not thread safe
 * while a profile is open.
 */
#define MUON_KIND_MOMENTUM 0   /* momentum, Nesterov input, hi/lo split, chunk sums */
#define MUON_KIND_NORM 1       /* per-matrix norm and scale */
#define MUON_KIND_GRAM 2       /* A = X X^T */
#define MUON_KIND_POLY 3       /* B = b A + c A A */
#define MUON_KIND_APPLY 4      /* X <- a X + B X */
#define MUON_KIND_APPLY_LAST 5 /* last iteration, fused parameter update */
#define MUON_NUM_KINDS 6

muon_status_t muon_profile_begin(void);
muon_status_t muon_profile_end(double* ms_by_kind, int64_t* launches_by_kind, int kinds);

/*
 * AdamW for the parameters Muon does not take: biases, norm gains and embeddings.
 * "14 - modded-nanogpt: the Speedrun Community", section 3: the canonical Muon setup is
 * hybrid, Muon on the 2-D matmul weights and AdamW on the rest.  The pages give no
 * formula; this is the textbook decoupled-decay AdamW with bias correction:
 *   m <- beta1 m + (1 - beta1) g,  v <- beta2 v + (1 - beta2) g^2
 *   p <- p (1 - lr wd) - (lr / (1 - beta1^step)) m / (sqrt(v / (1 - beta2^step)) + eps)
 * Each tensor is contiguous and flattened to `numel` elements.
 *   param       in/out, fp32 or bf16 (param_dtype), aligned to its element size
 *   grad        in, fp32
 *   exp_avg     in/out fp32 (m), exp_avg_sq in/out fp32 (v); start from zeros
 * All device pointers; 16-byte aligned buffers take the vector path.  Buffers written
 * (param, exp_avg, exp_avg_sq) may overlap no other buffer of the call.
 * Hyperparameters: finite, lr >= 0, 0 <= beta1, beta2 < 1, eps > 0, weight_decay >= 0,
 * step >= 1 (the 1-based count of updates including this one).  Asynchronous on `stream`;
 * on a validation error nothing is queued.
 */
typedef struct {
  void*        param;
  const float* grad;
  float*       exp_avg;
  float*       exp_avg_sq;
  int64_t      numel;
  int32_t      param_dtype;   /* MUON_F32 or MUON_BF16 */
  int32_t      reserved;      /* set to 0 */
} muon_adamw_tensor_t;

muon_status_t muon_adamw_step(const muon_adamw_tensor_t* tensors, int n, float lr, float beta1,
                              float beta2, float eps, float weight_decay, int64_t step,
                              void* stream);

/*
 * Newton-Schulz without a caller-supplied workspace, for callers that cannot allocate
 * device memory: code that runs inside another framework's memory pool or allocator
 * (where a cudaMalloc of its own would fragment that pool, or is forbidden), plugins
 * and embedded hosts that only receive ready-made device buffers, and callers that
 * must not allocate between steps.  The pages define no such call; this is a
 * packaging of muon_newton_schulz.
 *
 * Same arguments and results as muon_newton_schulz, except that the scratch is a
 * static device array of MUON_STATIC_SCRATCH_BYTES inside this library.  Every GPU
 * that loads the library holds that array until the process exits.  The call
 * allocates no device memory: no cudaMalloc or cudaFree, no allocating library.
 *
 *   - A matrix whose own scratch (hi/lo copies, Gram and polynomial buffers) does not
 *     fit in MUON_STATIC_SCRATCH_BYTES is rejected with MUON_ERR_STATIC_SCRATCH_LIMIT
 *     before anything is queued.  Sets that fit only together are processed in waves.
 *   - The first call on a device looks up the array's device address with the
 *     device current (cudaGetSymbolAddress), and so does the first call after that
 *     device's context has been re-created (e.g. by cudaDeviceReset).  Make those
 *     calls outside any stream capture.
 *   - All calls share the one array, which keeps the last call's contents.  Each call
 *     clears the array's status word before its kernels run.  Calls whose kernels
 *     overlap on the GPU (other streams, other host threads) race on the array and
 *     give wrong results: keep them ordered, e.g. on one stream.
 *   - device_status (may be NULL): 2 int32 in device or pinned host memory; after the
 *     call's kernels, in stream order, it receives the status word (MUON_OK,
 *     MUON_ERR_TIMEOUT or MUON_ERR_NONFINITE) and its `where`, as muon_device_status
 *     reports them.
 */
#define MUON_STATIC_SCRATCH_BYTES (64u << 20)

muon_status_t muon_newton_schulz_static(const muon_matrix_t* mats, int n, int ns_steps,
                                        const float* coeffs, float eps, int32_t* device_status,
                                        void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MUON_B200_H */
