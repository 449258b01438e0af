/*
 * muonh.h -- C ABI of the MuonH optimizer step for NVIDIA B200 (sm_100a).
 *
 * MuonH ("Muon with the Hyperball wrapper") is the optimizer the Puro-2B
 * report applies to the attention and MLP matrices of a Qwen3-architecture
 * model (arXiv HTML, Sec. 3.3 "Hyperball Optimization").  For each wrapped
 * matrix W (m x n) one step computes
 *
 *   M_t   = beta M_{t-1} + G_t                      heavy-ball momentum
 *   X     = G_t + beta M_t   (Nesterov)  or  M_t
 *   O     = NS(X)                                   quintic Newton-Schulz:
 *           Y = X/(||X||_F + eps) on the wide orientation, then ns_steps times
 *           A = Y Y^T;  B = b A + c A A;  Y = a Y + B Y
 *           (evaluated as written, or in runs of up to three iterations on
 *           r x r matrices, A <- A p(A)^2 and one Y <- Q Y per run, which is
 *           the same O in exact arithmetic; see muonh_config.ns_form)
 *   u^    = O/||O||_F                               Sec. 3.3, Eq. (1)
 *   W~    = W_t - lr R u^                           Sec. 3.3, Eq. (1)
 *   W_t+1 = R W~/||W~||_F                           Sec. 3.3, Eq. (1)
 *
 * with the radius fixed at R = ||W_0||_F (Sec. 3.3).  The effective LR of
 * Sec. 3.3.1 Eq. (4), ||lr R u^||_F/||W_t||_F, then equals lr, so `lr` is the
 * prescribed effective LR (eta^H = m eta^base of Sec. 3.3.1; the caller
 * applies the multiplier m and the schedule).  The pages name the Muon update
 * but not its internals: momentum form, Nesterov, eps and the coefficients
 * (a, b, c) are per-matrix inputs here.
 *
 * Conventions shared by every entry point
 *   - All functions are host functions; `stream` is a cudaStream_t passed as
 *     void* (NULL = the legacy default stream).  Work is enqueued
 *     asynchronously on it; argument checking is synchronous.
 *   - Device pointers are CUDA device (or managed) addresses on the current
 *     device.  The library never frees memory it did not allocate.
 *   - Argument errors (INVALID_ARG, ALIGNMENT, UNSUPPORTED) are found before
 *     any work is enqueued and leave every caller buffer untouched.  After
 *     MUONH_ERR_CUDA from a call that launches several kernels (muonh_step,
 *     muonh_init) the caller's buffers are unspecified: kernels enqueued
 *     before the failing launch still run.  The message of the last failure
 *     on the calling thread is in muonh_last_error().
 *   - Conditions found on the device (non-finite input, zero update, a
 *     bounded wait that gave up) never abort a step: they set per-matrix
 *     flags in muonh_stats and are reported by muonh_device_status().
 *   - A context is not thread-safe: calls on one context must not overlap
 *     in time.  Distinct contexts are independent.  The context-free
 *     functions (averaging, AdamW, the diagnostics) are reentrant, except
 *     muonh_momentum_norm_noalloc (one shared scratch array, see there).
 */
#ifndef MUONH_H_
#define MUONH_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MUONH_OK = 0,
  MUONH_ERR_INVALID_ARG = 1,   /* NULL pointer, bad size, bad enum value     */
  MUONH_ERR_ALIGNMENT = 2,     /* pointer or stride not 16-byte aligned      */
  MUONH_ERR_CUDA = 3,          /* a CUDA runtime call failed                 */
  MUONH_ERR_OOM = 4,           /* workspace allocation failed                */
  MUONH_ERR_TIMEOUT = 5,       /* a device-side bounded wait gave up         */
  MUONH_ERR_UNSUPPORTED = 6    /* no sm_100 device, or a size beyond limits  */
} muonh_status;

/* Arithmetic of the Newton-Schulz GEMMs (tensor cores, fp32 accumulation).
 *   FP16: operands stored as fp16 with exact power-of-two scaling (default)
 *   BF16: operands stored as bf16
 *   FP32: each operand split into an fp16 high and low part, three products
 *         per GEMM (hi*hi + hi*lo + lo*hi), about fp32 accuracy, 3x the work */
enum { MUONH_NS_FP16 = 0, MUONH_NS_BF16 = 1, MUONH_NS_FP32 = 2 };

/* Per-matrix flags reported in muonh_stats.flags. */
enum {
  MUONH_FLAG_NONFINITE_INPUT = 1u,   /* X had NaN/Inf: W kept unchanged          */
  MUONH_FLAG_ZERO_UPDATE = 2u,       /* ||X|| or ||O|| == 0: W only re-projected */
  MUONH_FLAG_NONFINITE_UPDATE = 4u,  /* X finite, O not: W kept unchanged        */
  MUONH_FLAG_DEGENERATE = 8u,        /* ||W~|| == 0: W kept unchanged            */
  MUONH_FLAG_TIMEOUT = 16u           /* a device wait gave up during this step   */
};

/* Update rule of a matrix (report Sec. 3.3 and 3.3.1).
 *   HYPERBALL     Eq. (1): MuonH, W <- R (W - lr R u^)/||.||, lr = the ELR.
 *   DECOUPLED_WD  Eq. (3): ordinary Muon, W <- (1 - wd lr) W - lr u.
 *   ELR_ALIGNED   Eq. (5): ordinary Muon with eta = lr ||W||/||u|| (lr = the
 *                 prescribed ELR), W <- (1 - wd eta) W - eta u, no projection.
 * For the ordinary rules u = update_scale * O, O the Newton-Schulz output. */
enum { MUONH_RULE_HYPERBALL = 0, MUONH_RULE_DECOUPLED_WD = 1, MUONH_RULE_ELR_ALIGNED = 2 };

/* One wrapped matrix.  w and m are caller-owned fp32 device buffers of
 * rows x cols elements, row-major with row stride ld (elements, ld >= cols),
 * 16-byte aligned base.  Rows are moved with 16-byte vector accesses when
 * cols and ld are multiples of 4, element by element otherwise (slower, any
 * ld).  The library updates them in
 * place on every step and keeps the pointers: they must stay valid until
 * muonh_destroy.  m must hold zeros before the first step (momentum starts
 * at 0).  radius <= 0 asks muonh_init to use ||W_0||_F (the Sec. 3.3 rule);
 * a positive value is used as R as given.  ns_steps in [0, 64]. */
typedef struct {
  float* w;
  float* m;
  int64_t rows;
  int64_t cols;
  int64_t ld;
  float radius;
  float beta;
  int32_t nesterov;
  int32_t ns_steps;
  float ns_a;
  float ns_b;
  float ns_c;
  int32_t update_rule;    /* MUONH_RULE_*; 0 = MuonH                        */
  float weight_decay;     /* lambda of Eq. (3)/(5); ignored by MuonH         */
  float update_scale;     /* u = update_scale * O for the ordinary rules     */
} muonh_matrix_desc;

/* Context-wide settings.
 *   groups  0: automatic.  A set of at least 16M elements on the 16-bit path
 *              then runs as two matrix groups of equal Newton-Schulz work,
 *              whose elementwise kernels overlap the other group's GEMMs on
 *              an internal stream.
 *           1: one group.  Every kernel runs on the caller's stream, one
 *              after another; the context creates no stream of its own.
 *           2, 3: that many groups on the 16-bit path, whatever the size
 *              (three groups take a quarter, a half and a quarter of the
 *              work, so the two phases no GEMM hides are short).
 *           Other values are rejected (MUONH_ERR_INVALID_ARG).  The results
 *           are the same bit for bit whatever the grouping.
 *   ns_form  how the Newton-Schulz iteration is evaluated (MUONH_NS_FORM_*).
 *           Y-space: every iteration forms A = Y Y^T, B' = a I + b A + c A A
 *           and Y <- B' Y (three products, two of them over the r x c Y).
 *           Gram-space: runs of up to three iterations are carried on r x r
 *           matrices, A_{k+1} = A_k p(A_k)^2 with p(A) = a I + b A + c A A,
 *           and each run ends with one Y <- Q Y, Q the product of the run's
 *           p(A_k) (fewer FLOPs where c >= 2r; a restart every three
 *           iterations keeps fp16 storage accurate).  In exact arithmetic
 *           both give the same O; their fp16 rounding differs.  The Gram
 *           form needs FP16 operands and ns_steps equal to the largest
 *           ns_steps of the context; other matrices use the Y-space form.
 *           Values outside MUONH_NS_FORM_* are rejected. */
enum {
  MUONH_NS_FORM_AUTO = 0,    /* Gram form for classes with r >= 1024, c >= 2r  */
  MUONH_NS_FORM_Y = 1,       /* Y-space form for every matrix                   */
  MUONH_NS_FORM_GRAM = 2     /* Gram form for every matrix that can take it     */
};
typedef struct {
  int32_t ns_precision;   /* MUONH_NS_FP16 / _BF16 / _FP32                  */
  float eps;              /* Newton-Schulz input: X/(||X||_F + eps), >= 0    */
  int32_t groups;         /* 0 = automatic, 1 = a single group, 2 or 3      */
  int32_t ns_form;        /* MUONH_NS_FORM_*                                */
} muonh_config;

/* Per-matrix result of one step (24 bytes, plain fp32 + uint32). */
typedef struct {
  float elr;          /* ||lr R u^||_F / ||W_t||_F  (Eq. (4) for Eq. (1))   */
  float pre_norm;     /* ||W_t||_F                                          */
  float post_norm;    /* ||W_t+1||_F, measured on the stored result         */
  float update_norm;  /* ||O||_F, the Newton-Schulz output                  */
  float input_norm;   /* ||X||_F, the Newton-Schulz input                   */
  uint32_t flags;     /* MUONH_FLAG_*                                       */
} muonh_stats;

typedef struct muonh_ctx muonh_ctx;

/* Build the step for n matrices: validates the descriptors, groups matrices
 * of equal Newton-Schulz shape, allocates the device workspace (owned by the
 * context, freed by muonh_destroy), computes R = ||W_0||_F where asked and
 * ||W_0||_F^2 for every matrix, and synchronises `stream` once.
 * *out receives the context; on failure *out is set to NULL. */
muonh_status muonh_init(muonh_ctx** out, const muonh_matrix_desc* mats, int32_t n,
                        const muonh_config* cfg, void* stream);

/* One MuonH step over all matrices (the hot path).
 *   lr     host array of n floats: the effective LR (eta^H) of each matrix,
 *          read before the call returns.
 *   grads  host array of n device pointers to fp32 gradients, each laid out
 *          like its matrix's w (same rows, cols, ld); read before return.
 *   stats  NULL, or device-accessible memory (device, managed or mapped
 *          pinned host) for n muonh_stats, written by the last kernel.
 * Updates every w and m in place.  Enqueued on `stream`; the caller
 * synchronises before reading w, m or stats.  A large set (>= 16M elements)
 * also runs its Newton-Schulz GEMMs on an internal stream of the context;
 * `stream` waits for that work before the step's last kernels, so the step
 * is complete in `stream`'s order like any single-stream launch sequence. */
muonh_status muonh_step(muonh_ctx* ctx, const float* lr, const float* const* grads,
                        muonh_stats* stats, void* stream);

/* Per-matrix arguments of one step, in device memory, for muonh_step_device
 * (16 bytes: the gradient pointer, the effective LR, 4 bytes of padding). */
typedef struct {
  const float* grad;   /* fp32 device gradient, laid out like the matrix's w */
  float lr;            /* the matrix's effective LR (eta^H) for this step     */
  float pad_;
} muonh_step_args;

/* muonh_step with its per-matrix arguments in device memory: `args` is a
 * device array of n muonh_step_args, read by the step's kernels when they
 * run.  The call enqueues kernel launches and, for a grouped step, event
 * records and waits between `stream` and the context's internal stream;
 * it copies nothing from the host and never synchronises.  It can
 * therefore be captured in a CUDA graph, and every replay uses whatever
 * `args` and the gradients hold when it runs.  The library cannot inspect
 * device-resident arguments: every grad must be non-NULL, 16-byte aligned
 * and laid out like its matrix's w, and every lr finite, as muonh_step
 * checks on the host.  `args` itself must be 16-byte aligned
 * (MUONH_ERR_ALIGNMENT otherwise).  Results are bit-identical to
 * muonh_step with the same arguments. */
muonh_status muonh_step_device(muonh_ctx* ctx, const muonh_step_args* args, muonh_stats* stats, void* stream);

/* Copy the last step's per-matrix stats to host memory (n entries);
 * synchronises the stream of the last step. */
muonh_status muonh_get_stats(muonh_ctx* ctx, muonh_stats* host_out);

/* Write matrix i's Newton-Schulz output O of the last step, unscaled and in
 * the orientation of w (rows x cols), as fp32 into device memory `dst` with
 * row stride ld (elements).  Enqueued on `stream`. */
muonh_status muonh_get_update(muonh_ctx* ctx, int32_t i, float* dst, int64_t ld, void* stream);

/* Host copy of the n radii R. */
muonh_status muonh_get_radius(const muonh_ctx* ctx, float* host_R);

/* Checkpointing of the library-held state (R[], ||W_t||^2[], the scale the
 * next step writes the Newton-Schulz input with, and the step count).
 * W and M are caller-owned and saved by the caller.  With buf == NULL,
 * *len receives the size needed.  Export synchronises the last stream. */
muonh_status muonh_export_state(muonh_ctx* ctx, void* buf, size_t* len);
muonh_status muonh_import_state(muonh_ctx* ctx, const void* buf, size_t len);

/* Synchronises the last stream and returns MUONH_ERR_TIMEOUT if a device
 * wait gave up since the previous call (then clears the record), else OK. */
muonh_status muonh_device_status(muonh_ctx* ctx);

/* Number of kernel launches the last muonh_step enqueued. */
int32_t muonh_last_launch_count(const muonh_ctx* ctx);

/* Kernel phases of one step, in launch order (ns_* repeat ns_steps times). */
enum {
  MUONH_PHASE_MOMENTUM_NORM = 0,   /* M update, ||X||^2 partials            */
  MUONH_PHASE_FINALIZE_INPUT = 1,  /* per-matrix 1/(||X|| + eps)            */
  MUONH_PHASE_WRITE_X = 2,         /* normalised 16-bit X, wide orientation */
  MUONH_PHASE_NS_GRAM = 3,         /* A = Y Y^T                             */
  MUONH_PHASE_NS_SQUARE = 4,       /* B = b A + c A A                       */
  MUONH_PHASE_NS_APPLY = 5,        /* Y = a Y + B Y                         */
  MUONH_PHASE_UPDATE_DOTS = 6,     /* ||O||^2, <W, O> partials              */
  MUONH_PHASE_FINALIZE_UPDATE = 7, /* Eq. (1) scalars per matrix            */
  MUONH_PHASE_PROJECT = 8,         /* W <- R (W - lr R u^)/||.||            */
  MUONH_PHASE_FINALIZE_STEP = 9,   /* ||W_t+1||, stats                      */
  MUONH_PHASE_NS_PRODUCT = 10,     /* Gram form: products of r x r factors  */
  MUONH_NUM_PHASES = 11
};

/* With enable != 0, every following muonh_step brackets each kernel with a
 * pair of CUDA events on its stream (a few microseconds per step); 0 stops
 * recording.  Recorded pairs are kept until muonh_phase_times reads them. */
muonh_status muonh_enable_timing(muonh_ctx* ctx, int32_t enable);

/* Synchronises the last stream and returns, per phase, the summed kernel
 * time in ms (ms_out[MUONH_NUM_PHASES]) and the number of launches timed
 * (launches_out[MUONH_NUM_PHASES], may be NULL) since the previous call;
 * then clears the record. */
muonh_status muonh_phase_times(muonh_ctx* ctx, float* ms_out, int64_t* launches_out);

/* Tensor-core FLOPs that the Newton-Schulz launches of the last muonh_step
 * executed, per phase (flops_out[MUONH_NUM_PHASES]; 0 for the elementwise
 * phases): for each launch, its tiles' 2 M N K on the padded buffers, three
 * products per tile in FP32 mode.  Symmetric products count only the tiles
 * they compute (those that touch the upper block triangle). */
muonh_status muonh_phase_flops(const muonh_ctx* ctx, double* flops_out);

/* Allocation-free momentum stage for one matrix (the report has no
 * counterpart; this is a deployment convenience).  Computes, like the first
 * kernel of muonh_step, M <- beta M + G in place and writes ||X||_F of the
 * Newton-Schulz input X = G + beta M (nesterov != 0) or X = M to the device
 * double *x_norm.  For callers that cannot call cudaMalloc -- code running
 * under global-mode stream capture, programs whose device memory is owned
 * entirely by a framework allocator or a fixed arena, loops that must not
 * take the driver's allocation locks -- it allocates nothing: its scratch
 * (one fp32 partial sum per 4096-element tile) is a 256 KB array compiled
 * into the library, held by every device that loads it until exit.
 *   m, g   fp32 device buffers, rows x cols, row stride ld, 16-byte aligned;
 *          m is updated in place, g is read.
 *   limit  at most 65,536 tiles (268,435,456 elements); a larger matrix
 *          returns MUONH_ERR_UNSUPPORTED and touches nothing.
 * The first call on a device looks up the scratch array's device address
 * (cudaGetSymbolAddress) and the SM count, and keeps both for that device
 * ordinal; make that first call before any stream capture.  The address is
 * the one in the device's primary context (the CUDA runtime's default, which
 * PyTorch uses): call it only with the primary context current, and not
 * after cudaDeviceReset, which invalidates the kept address.
 * All calls share the one scratch array, so calls whose kernels overlap on
 * the GPU (different streams without ordering) race; calls on one stream are
 * ordered and safe.  Enqueued on `stream`. */
muonh_status muonh_momentum_norm_noalloc(float* m, const float* g, int64_t rows, int64_t cols, int64_t ld,
                                         float beta, int32_t nesterov, double* x_norm, void* stream);

/* ---------------------------------------------------------------------------
 * Auxiliary operations of the same training recipe.  Stateless: no context,
 * no allocation; enqueued on `stream`.
 * ------------------------------------------------------------------------- */

#define MUONH_DTYPE_F32 0
#define MUONH_DTYPE_BF16 1
#define MUONH_AVERAGE_MAX_INPUTS 16
#define MUONH_ADAMW_MAX_TENSORS 32   /* per launch; longer lists take several */

/* Checkpoint parameter averaging (Puro-2B report, Sec. 3.4: the released
 * model is the equal average of six checkpoints; parameters only).
 *   out[j] = (in[0][j] + in[1][j] + ... + in[k-1][j]) / k
 * summed in fp32 in that order, rounded once to out_dtype.
 *   out     device buffer of `count` elements of out_dtype; may alias in[0]
 *           (each element is read before it is written, by the same thread).
 *   in      HOST array of k device pointers, each `count` elements of in_dtype.
 *   dtypes  MUONH_DTYPE_F32 or MUONH_DTYPE_BF16.
 *   k       1..MUONH_AVERAGE_MAX_INPUTS.
 * Every pointer must be 16-byte aligned (MUONH_ERR_ALIGNMENT otherwise).
 * count == 0 checks k and the dtypes only (the buffers may be NULL) and
 * enqueues nothing. */
muonh_status muonh_average(void* out, int32_t out_dtype, const void* const* in, int32_t in_dtype, int32_t k,
                           int64_t count, void* stream);

/* One flat fp32 tensor of the AdamW group: parameters p, first and second
 * moments m and v (updated in place), gradient g (read), `count` elements
 * each.  Pointers need 4-byte alignment; a tensor whose four pointers are
 * all 16-byte aligned takes the vector path. */
typedef struct {
  float* p;
  float* m;
  float* v;
  const float* g;
  int64_t count;
} muonh_adamw_tensor;

typedef struct {
  float lr;
  float beta1;          /* Puro-2B report App. E: 0.9  */
  float beta2;          /*                        0.95 */
  float eps;
  float weight_decay;   /* Table 8: 0.1 for the AdamW group */
} muonh_adamw_config;

/* AdamW step for the parameter group outside MuonH (Puro-2B report, Table 8:
 * embeddings, normalisation layers, LM head).  With `step` = t >= 1 (1-based,
 * the caller's count of steps taken including this one), per element:
 *   p <- p (1 - lr wd);   m <- b1 m + (1 - b1) g;   v <- b2 v + (1 - b2) g^2
 *   p <- p - lr (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps)
 * in fp32 (the bias corrections are formed in double, then rounded).
 * `tensors` is a HOST array of n descriptors; all of them are updated by
 * ceil(n / MUONH_ADAMW_MAX_TENSORS) launches.  Tensors must not overlap. */
muonh_status muonh_adamw_step(const muonh_adamw_tensor* tensors, int32_t n, const muonh_adamw_config* cfg,
                              int64_t step, void* stream);

/* Diagnostic of the failure path every pipelined kernel uses (the report has
 * no counterpart).  Launches one thread that waits on an mbarrier nothing
 * will ever complete, with the same bounded wait as the kernels but a limit
 * of `seconds` (0 < seconds <= 10) instead of 2 s.  The wait gives up,
 * records the failure in a device flag, and the kernel returns, so no GPU
 * hangs.  Returns MUONH_ERR_TIMEOUT when that happened, which is the
 * expected outcome; MUONH_ERR_CUDA if the wait did not give up or a CUDA
 * call failed.  Allocates and frees a 4-byte flag; synchronises `stream`. */
muonh_status muonh_check_wait_timeout(double seconds, void* stream);

void muonh_destroy(muonh_ctx* ctx);

const char* muonh_status_string(muonh_status s);

/* Message of the last failure on the calling thread ("" if none). */
const char* muonh_last_error(void);

#ifdef __cplusplus
}
#endif

#endif  /* MUONH_H_ */
