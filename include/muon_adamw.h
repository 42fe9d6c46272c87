/*
 * muon_adamw.h - C ABI of the AdamW companion step (sm_100a).
 *
 * The Muon recipe keeps some parameters on AdamW: embeddings, the prediction
 * head, biases, gates and all RMSNorm weights ([V4-breakdown] "Muon
 * 优化器完全拆解：矩阵级正交化更新如何撑起万亿 MoE 训练", section
 * "为什么嵌入层、输出头、bias、RMSNorm 还在用 AdamW"). AdamW moves each element
 * by its bias-corrected first moment over the square root of its
 * bias-corrected second moment (section "AdamW 到底哪里”不协调”"), with the
 * decoupled weight decay written as a factor (1 - lr wd) (Algorithm 1, step
 * five). Per element, at step t >= 1:
 *
 *   m <- b1 m + (1 - b1) g
 *   v <- b2 v + (1 - b2) g^2
 *   p <- p (1 - lr wd) - (lr / (1 - b1^t)) m / (sqrt(v) / sqrt(1 - b2^t) + eps)
 *
 * The pages give neither b1, b2 nor eps; callers pass them (customary values
 * 0.9, 0.999 and 1e-8). Arithmetic is fp32; (1 - b1), (1 - b2) and the bias
 * corrections are formed in double on the host (or on the device from
 * `step_dev`) and rounded once.
 *
 * Conventions are those of muon_step.h: caller-owned contiguous fp32 DEVICE
 * arrays, no device allocation by the library, everything asynchronous on
 * `stream`, argument errors returned synchronously. One launch per execute;
 * HBM-bound (16 bytes read and 12 written per element).
 */
#ifndef MUON_ADAMW_H
#define MUON_ADAMW_H

#include "muon_step.h"

#ifdef __cplusplus
extern "C" {
#endif

/* One tensor of the AdamW group, flattened: p, m, v updated in place, g read.
 * 0 <= numel <= 2^40; a tensor with numel = 0 is skipped. The four arrays must
 * not overlap one another or another tensor's. Tensors whose four pointers are
 * 16-byte aligned take the vectorised path; others a scalar one. */
typedef struct {
  float* p;
  const float* g;
  float* m;
  float* v;
  int64_t numel;
} muon_adamw_param_t;

/* Hyper-parameters. 0 <= beta1, beta2 < 1, eps > 0, all finite. beta1 and
 * beta2 are doubles: 1 - beta2 for beta2 = 0.999 is 1.3e-5 off when formed
 * from the nearest float, which would show in v at fp32 accuracy. The step t
 * counts from 1: it is `step` unless `step_dev` (a DEVICE int32) is non-NULL,
 * in which case each execute reads t from it on the device (values below 1
 * count as 1), so that a captured CUDA graph can advance t itself. */
typedef struct {
  float lr;
  float eps;
  float weight_decay;
  int32_t step;
  double beta1;
  double beta2;
  const int32_t* step_dev;
} muon_adamw_hyper_t;

typedef struct muon_adamw_plan_s* muon_adamw_plan_t;

/* Plan an AdamW step over `count` tensors (count >= 1). The pointers are
 * recorded and used by every execute. Executing on a workspace pointer the
 * plan has not seen before first copies its tensor table there
 * (cudaMemcpyAsync on `stream`); later executes launch one kernel only and
 * can be captured in a CUDA graph. */
MUON_API muon_status_t muon_adamw_plan_create(const muon_adamw_param_t* params, int count,
                                              muon_adamw_plan_t* plan);

/* Workspace bytes the plan needs (device memory, 256-byte aligned). */
MUON_API muon_status_t muon_adamw_plan_workspace_size(muon_adamw_plan_t plan, size_t* bytes);

MUON_API muon_status_t muon_adamw_plan_execute(muon_adamw_plan_t plan,
                                               const muon_adamw_hyper_t* hyper, void* workspace,
                                               size_t workspace_bytes, void* stream);

/* Elements of all tensors of the plan (for bandwidth figures). */
MUON_API muon_status_t muon_adamw_plan_numel(muon_adamw_plan_t plan, int64_t* numel);

MUON_API void muon_adamw_plan_destroy(muon_adamw_plan_t plan);

/* One-shot forms (plan, execute, destroy; not for graph capture). */
MUON_API muon_status_t muon_adamw_workspace_size(const muon_adamw_param_t* params, int count,
                                                 size_t* bytes);

MUON_API muon_status_t muon_adamw_step(const muon_adamw_param_t* params, int count,
                                       const muon_adamw_hyper_t* hyper, void* workspace,
                                       size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MUON_ADAMW_H */
