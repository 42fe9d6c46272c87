/*
 * muon_step.h - C ABI of the B200 (sm_100a) Muon optimizer step library.
 *
 * The method (sources cited by page title and section):
 *
 *   [V4-breakdown] "Muon 优化器完全拆解：矩阵级正交化更新如何撑起万亿 MoE 训练",
 *                  section "V4 的完整更新公式，逐行拆解", Algorithm 1
 *                  "Muon Optimizer for DeepSeek-V4" and its five steps.
 *   [V4-book]      "Ch 06 · Muon — 矩阵参数的指南针" (DeepSeek-V4-book ch. 6),
 *                  §3 (Newton-Schulz), §4 (hybrid 8 + 2 schedule),
 *                  §5 Algorithm 1 "Muon Optimizer (V4 Hybrid)".
 *
 * For every 2-D weight W (n x m) with gradient G and momentum buffer M:
 *
 *   M   <- mu M + G                                  momentum
 *   N    = mu M + G        (M itself if nesterov=0)  Nesterov look-ahead
 *   X    = N / (||N||_F + eps), transposed when n > m (rows <= cols)
 *   X   <- a_k X + b_k (X X^T) X + c_k (X X^T)^2 X   k = 1 .. steps
 *   O'   = X, transposed back                       (orthogonalised direction)
 *   W   <- W (1 - lr wd) - lr gamma sqrt(max(n, m)) O'
 *
 * The default schedule is 8 steps of (3.4445, -4.7750, 2.0315) then 2 steps
 * of (2, -1.5, 0.5), with eps = 1e-7.
 *
 * Conventions for every entry point:
 *   - Matrices are caller-owned, contiguous, row-major fp32 DEVICE arrays.
 *     Distinct matrices must not overlap. The library allocates no device
 *     memory: all scratch lives in the caller's workspace.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). All device work is asynchronous on that stream; nothing
 *     synchronises except muon_sync_status().
 *   - Argument errors are reported synchronously and leave the device
 *     untouched. Device-side failures (a bounded wait that expired) set a
 *     per-device error word that muon_sync_status() reports and clears.
 *   - NaN / Inf in the inputs are not checked; they propagate as in the
 *     plain definition.
 *   - Host threads: the library-wide setters (muon_set_wait_limit_ns,
 *     muon_set_tracing) and the one-shot calls may be used from any thread.
 *     A plan holds no lock: calls on one plan (execute, the set_* calls,
 *     destroy) must not overlap in time. Work that runs concurrently must
 *     not share a workspace. The device error word is shared by every caller
 *     on a device, so muon_sync_status() reports and clears the errors of
 *     all of them.
 */
#ifndef MUON_STEP_H
#define MUON_STEP_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MUON_API __attribute__((visibility("default")))
#else
#define MUON_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MUON_ABI_VERSION 1
#define MUON_MAX_NS_STEPS 64

typedef enum {
  MUON_OK = 0,
  MUON_ERR_INVALID_ARG = 1, /* NULL pointer, bad size, bad count, bad schedule */
  MUON_ERR_WORKSPACE = 2,   /* workspace NULL, misaligned (256 B) or too small */
  MUON_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  MUON_ERR_UNSUPPORTED = 4, /* no sm_100 device, or a size beyond the limits */
  MUON_ERR_TIMEOUT = 5      /* a device-side bounded wait expired */
} muon_status_t;

/* Newton-Schulz operand precision. BF16: bf16 tensor-core operands with fp32
 * accumulation; the iterate is kept as bf16 high + low parts (16 significant
 * bits) so that the a X term does not lose the operand's rounding. FP32: fp32 operands on
 * the CUDA cores (validation; slow). Momentum and update are fp32 in both. */
typedef enum { MUON_NS_BF16 = 0, MUON_NS_FP32 = 1 } muon_precision_t;

/* One matrix of a Muon step ([V4-breakdown] Algorithm 1 inputs). */
typedef struct {
  float* W;       /* n x m weight, updated in place */
  const float* G; /* n x m gradient, read only */
  float* M;       /* n x m momentum buffer, updated in place */
  float* O;       /* optional n x m output of O' (before the RMS rescale); NULL to skip */
  int64_t n, m;   /* 1 <= n, m <= 2^31 - 8 */
} muon_param_t;

/* Newton-Schulz schedule ([V4-book] §4). `abc` is a HOST array of steps * 3
 * floats (a, b, c per step, applied in order); 1 <= steps <= MUON_MAX_NS_STEPS;
 * eps > 0 is added to the Frobenius norm. A NULL schedule means the hybrid
 * 8 + 2 schedule with eps = 1e-7. The library copies it. */
typedef struct {
  int steps;
  const float* abc;
  float eps;
} muon_ns_schedule_t;

/* One matrix for ns_orthogonalize: O = O'(X) in X's orientation. */
typedef struct {
  const float* X; /* n x m input, read only */
  float* O;       /* n x m output, must not overlap X */
  int64_t n, m;   /* 1 <= n, m <= 2^31 - 8 */
} muon_ns_matrix_t;

/* Hyper-parameters of one step ([V4-breakdown] Algorithm 1: eta, mu, lambda,
 * gamma). nesterov != 0 selects N = mu M + G. */
typedef struct {
  float lr;
  float momentum;
  float weight_decay;
  float gamma;
  int nesterov;
} muon_hyper_t;

/* How O' is scaled into the update O (W <- W (1 - lr wd) - lr O):
 *   SHAPE     O = O' sqrt(max(n, m)) gamma   ([V4-breakdown] Algorithm 1; default)
 *   UNIT_RMS  O = O' gamma / RMS(O')         ([V4-breakdown] "另一条路：开源生态干脆不分片":
 *             the Megatron-Bridge recipe's unit_rms_norm scale mode; O' = 0 gives O = 0)
 *   NONE      O = O' gamma                   (the original Muon with gamma = 1) */
typedef enum { MUON_SCALE_SHAPE = 0, MUON_SCALE_UNIT_RMS = 1, MUON_SCALE_NONE = 2 } muon_scale_mode_t;

typedef struct muon_plan_s* muon_plan_t;

/* ---------------------------------------------------------------- plans
 * A plan holds, on the host, everything that depends only on the shapes:
 * shape groups, tile lists, the workspace layout. It is built once and
 * executed many times. Executing a plan on a workspace pointer it has not
 * seen before first copies its descriptor tables into that workspace
 * (cudaMemcpyAsync on `stream`); later executes on the same pointer launch
 * kernels only, so they can be captured in a CUDA graph. Between executes the
 * caller must not modify the workspace (or must pass another pointer). */

/* Plan a Muon step over `count` matrices. Pointers in `params` are recorded
 * and used by every execute. */
MUON_API muon_status_t muon_plan_create(const muon_param_t* params, int count, muon_precision_t prec,
                               const muon_ns_schedule_t* sched, muon_plan_t* plan);

/* Plan ns_orthogonalize over `count` matrices. */
MUON_API muon_status_t muon_plan_create_ns(const muon_ns_matrix_t* mats, int count,
                                  muon_precision_t prec, const muon_ns_schedule_t* sched,
                                  muon_plan_t* plan);

/* Select the update scale of later executes (default MUON_SCALE_SHAPE). In
 * UNIT_RMS mode the last step adds a per-matrix reduction and an elementwise
 * update pass for matrices larger than 128 x 128. */
MUON_API muon_status_t muon_plan_set_scale_mode(muon_plan_t plan, muon_scale_mode_t mode);

/* Per-matrix diagnostics of later executes ([V4-breakdown] section
 * "更新尺度：让 Muon 借用 AdamW 的超参": the update-RMS lemma says RMS(O') is
 * about sqrt(1 / max(n, m)), so the shape rule's update has RMS about gamma).
 * `out` is a caller-owned DEVICE array of 2 * count floats, in the order of
 * the plan's params; each execute writes
 *   out[2 i]     = ||N_i||_F   the Frobenius norm of the orthogonaliser's input
 *   out[2 i + 1] = RMS(O_i)    the RMS of the scaled update that lr multiplies
 * (0 for a zero gradient). NULL turns them off (the default). With the SHAPE
 * or NONE scale the last step then adds one per-matrix reduction launch for
 * matrices larger than 128 x 128. Muon-step plans only. */
MUON_API muon_status_t muon_plan_set_diagnostics(muon_plan_t plan, float* out);

/* L2 batching of the Newton-Schulz stages (off by default; 0 turns it off).
 * With `bytes` > 0, later executes run all steps of the schedule batch by
 * batch, a batch being consecutive matrices of the plan whose Newton-Schulz
 * buffers (bf16: 6 r ldc + 4 r ldr bytes per matrix) add up to at most
 * `bytes` (at least one matrix). With a budget below the L2 size (126 MB on
 * B200) a batch's buffers stay in L2 across its 3 x steps launches; the
 * price is 3 x steps launches per batch. The workspace and the results do
 * not change. Timing events must be set again afterwards. */
MUON_API muon_status_t muon_plan_set_l2_batching(muon_plan_t plan, size_t bytes);

/* How later executes launch the Newton-Schulz stages in the bf16 precision
 * (without L2 batching). on = 1 (the default): every Gram, Poly and Apply
 * stage of the schedule in one persistent launch, then the last Apply fused
 * with the update. Its CTA pairs take the tiles of a host-built list in
 * order, each pair the next unclaimed one (a counter in the workspace) as it
 * becomes free; a tile waits (bounded) until the earlier stages of its own
 * matrix have finished, signalled through per-matrix counters in the
 * workspace. The list keeps `window` matrices in flight at a time (0: chosen
 * from the tile counts), so their buffers can stay in L2 from one stage to
 * the next. on = 0: one launch per stage and step. Both give bit-identical
 * results. Pairs that other streams' work keeps from starting delay the
 * chained launch but cannot stall it. Timing events must be set again
 * afterwards. */
MUON_API muon_status_t muon_plan_set_chaining(muon_plan_t plan, int on, int window);

/* Bytes of workspace the plan needs (device memory, 256-byte aligned). */
MUON_API muon_status_t muon_plan_workspace_size(muon_plan_t plan, size_t* bytes);

/* Run the plan: one kernel for momentum / norm / cast, then three kernels per
 * Newton-Schulz step, each one persistent launch over every matrix. `hyper` is
 * ignored (may be NULL) for an ns_orthogonalize plan. The first execute on a
 * workspace (or on another device) copies the plan's descriptor tables into
 * it with cudaMemcpyAsync from host memory the plan owns: the plan must
 * outlive that copy, and anything that repeats it. */
MUON_API muon_status_t muon_plan_execute(muon_plan_t plan, const muon_hyper_t* hyper, void* workspace,
                                size_t workspace_bytes, void* stream);

/* Number of kernel launches one execute issues, and the kind of each
 * (0 momentum/norm/cast, 1 Gram, 2 polynomial, 3 apply, 4 apply + update,
 * 5 small-matrix kernel (all steps and the update of matrices up to
 * 128 x 128), 6 per-matrix RMS reduction, 7 update pass, 8 mid-size kernel
 * (all steps and the update of matrices with min(n, m) <= 128 < max(n, m)
 * <= 512), 9 tiny-matrix kernel (bf16 precision only: matrices of at most
 * 4096 elements run every step with fp32 operands, since bf16 operand
 * rounding does not average out over so few elements), 10 chained launch of
 * every Newton-Schulz stage (see muon_plan_set_chaining)). */
MUON_API muon_status_t muon_plan_launches(muon_plan_t plan, int* count, int* kinds, int max_kinds);

/* Optional timing: `events` holds 2 * launches cudaEvent_t (as void*); each
 * execute records events[2k] before and events[2k + 1] after launch k on the
 * execute's stream. count = 0 turns timing off. The caller owns the events. */
MUON_API muon_status_t muon_plan_set_events(muon_plan_t plan, void* const* events, int count);

/* Useful floating-point operations of one execute's Newton-Schulz stages, per
 * stage kind (Gram, polynomial, apply), counted over the tiles that are
 * actually computed and clipped to the matrices' bounds. */
MUON_API muon_status_t muon_plan_flops(muon_plan_t plan, double* gram, double* poly, double* apply);

MUON_API void muon_plan_destroy(muon_plan_t plan);

/* ---------------------------------------------------------------- one-shot
 * Plan, execute and destroy in one call. The plan's descriptor tables reach
 * the workspace as kernel arguments (at most 32 KB per launch; all-zero
 * chunks as memsets), so no device work left pending by the call refers to
 * the host memory it releases, and the call does not wait on the stream.
 * A persistent plan (muon_plan_execute) saves the planning and this copy on
 * every later call. */

MUON_API muon_status_t muon_workspace_size(const muon_param_t* params, int count, muon_precision_t prec,
                                  size_t* bytes);

MUON_API muon_status_t muon_step(const muon_param_t* params, int count, float lr, float momentum,
                        float weight_decay, float gamma, int nesterov,
                        const muon_ns_schedule_t* sched, muon_precision_t prec, void* workspace,
                        size_t workspace_bytes, void* stream);

MUON_API muon_status_t ns_workspace_size(const muon_ns_matrix_t* mats, int count, muon_precision_t prec,
                                size_t* bytes);

/* O' = HybridNewtonSchulz(X / (||X||_F + eps)) per matrix ([V4-book] §5
 * Algorithm 1, the normalisation and the two loops), without the rescale. */
MUON_API muon_status_t ns_orthogonalize(const muon_ns_matrix_t* mats, int count,
                               const muon_ns_schedule_t* sched, muon_precision_t prec,
                               void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------- status */

/* Synchronise `stream`, then read and clear the current device's error word.
 * Returns MUON_ERR_TIMEOUT if a bounded wait expired since the last call. */
MUON_API muon_status_t muon_sync_status(void* stream);

MUON_API const char* muon_status_string(muon_status_t status);

MUON_API int muon_abi_version(void);

/* NVTX ranges (host side) around each kernel launch of later executes,
 * named by launch kind ("muon:gram", "muon:apply", ...), for profilers that
 * collect NVTX; off (0) by default. Process-wide. */
MUON_API void muon_set_tracing(int on);

/* Bound, in nanoseconds, on every device-side spin-wait of later launches
 * (default 2e9). Values below 1000 are raised to 1000. */
MUON_API void muon_set_wait_limit_ns(uint64_t ns);

/* Test of the timeout path: launch one bounded wait on the device word `flag`
 * (device memory; the wait ends when it becomes non-zero) for at most
 * `limit_ns`. If the limit passes, the device error word gets the timeout
 * bit, which muon_sync_status() then reports. */
MUON_API muon_status_t muon_wait_probe(const int* flag, uint64_t limit_ns, void* stream);

/* Test of the chained launch's dependency wait (muon_plan_set_chaining): one
 * thread waits, as a chained tile does, until the DEVICE word `counter`
 * (acquire loads) reaches `target`, for at most `limit_ns`. If the limit
 * passes, the device error word gets the timeout bit, which
 * muon_sync_status() then reports. */
MUON_API muon_status_t muon_dep_wait_probe(const uint32_t* counter, uint32_t target,
                                           uint64_t limit_ns, void* stream);

/* ---------------------------------------------------------------- no allocation
 * The pages describe no counterpart of this entry point; it serves callers
 * that cannot allocate device memory during a step: runtimes that reserve
 * (nearly) all of HBM up front for their own pool, real-time or multi-stream
 * code that cannot afford the device-wide synchronisation cudaMalloc and
 * cudaFree may cause, plugins handed data pointers but no allocator.
 *
 * Same step and arguments as muon_step(), without a workspace: the scratch is
 * a file-scope device array of MUON_STATIC_SCRATCH_BYTES inside the library,
 * held on every device where the library is loaded until the process exits.
 * The call allocates no device memory. The first call on a device looks up
 * the array's device address (cudaGetSymbolAddress); make that first call
 * before any stream capture on that device.
 *   - Returns MUON_ERR_WORKSPACE, before any device work, when the matrices
 *     need more scratch than MUON_STATIC_SCRATCH_BYTES (see
 *     muon_workspace_size for the amount).
 *   - Each call writes its descriptor tables, including the counters that
 *     must start at zero, into the array before its kernels run, so the
 *     contents left by the previous call do not matter.
 *   - All calls on a device share the one array: calls whose GPU work
 *     overlaps (different streams, no ordering between them) race and give
 *     wrong results. Order them on one stream or with events. */
#define MUON_STATIC_SCRATCH_BYTES (64u << 20)

MUON_API muon_status_t muon_step_static_scratch(const muon_param_t* params, int count, float lr,
                                                float momentum, float weight_decay, float gamma,
                                                int nesterov, const muon_ns_schedule_t* sched,
                                                muon_precision_t prec, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MUON_STEP_H */
