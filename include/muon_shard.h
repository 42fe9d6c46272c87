/*
 * muon_shard.h - elementwise steps of the ZeRO-sharded Muon step (sm_100a).
 *
 * Distributed Muon ([V4-breakdown] "Muon 优化器完全拆解：矩阵级正交化更新如何撑起
 * 万亿 MoE 训练", section "分布式工程", Algorithm 1 "Distributed Muon") keeps
 * the momentum and the parameters sharded over the data-parallel ranks:
 *
 *   1. g  = reduce_scatter(G)            this rank's shard of the gradient
 *   2. g' = momentum update of g with the local momentum shard
 *   3. G' = gather(g')                   the whole matrix
 *   4. U  = NewtonSchulz(G')             (ns_orthogonalize in muon_step.h)
 *   5. u  = this rank's shard of U
 *   6. p' = update of the local parameter shard with u
 *   7. P  = all_gather(p')
 *
 * Steps 2 and 6 are the calls below; the collectives are the caller's
 * (NCCL through torch.distributed in muon_step_b200.distributed). A shard is
 * any contiguous range of a flattened row-major matrix. Both calls take a list
 * of shards and run one launch over all of them (HBM-bound: 20 and 12 bytes
 * per element). The arithmetic is that of muon_step(): the same fp32
 * operations in the same order, so a one-rank sharded step equals muon_step()
 * given the same orthogonalised direction.
 *
 * muon_copy_segments is the gather / permute step of a grouped exchange: it
 * moves every matrix's shards between a per-matrix layout and a rank-major
 * one in one launch, so that each of the steps 1, 3 and 7 is one collective
 * over one buffer instead of one per matrix.
 *
 * Conventions are those of muon_step.h (caller-owned fp32 DEVICE arrays, no
 * device allocation, asynchronous on `stream`, argument errors returned
 * synchronously). Each call writes its descriptor list into `workspace`
 * (muon_shard_workspace_size bytes, 256-byte aligned) through kernel
 * arguments before its kernel runs, so the workspace must not be shared by
 * calls that run concurrently, and nothing refers to host memory after the
 * call returns.
 */
#ifndef MUON_SHARD_H
#define MUON_SHARD_H

#include "muon_step.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Step 2 on one shard: M <- mu M + G; N = mu M + G (nesterov) or N = M.
 * M is updated in place; N may not overlap M or G. 0 <= numel <= 2^40. */
typedef struct {
  float* M;
  const float* G;
  float* N;
  int64_t numel;
} muon_shard_momentum_t;

/* Step 6 on one shard: W <- W (1 - lr wd) - lr gamma sqrt(max(n, m)) O, with
 * (n, m) the shape of the whole matrix the shard belongs to (the shape rule of
 * [V4-breakdown] Algorithm 1 step four). O is the shard of O' (before the
 * rescale); W may not overlap O. */
typedef struct {
  float* W;
  const float* O;
  int64_t numel;
  int64_t n, m;
} muon_shard_update_t;

/* One segment of a copy: dst[i] = src[i] for 0 <= i < numel (fp32). */
typedef struct {
  float* dst;
  const float* src;
  int64_t numel;
} muon_segment_t;

/* Workspace bytes for a list of `count` shards or segments (any kind). */
MUON_API muon_status_t muon_shard_workspace_size(int count, size_t* bytes);

MUON_API muon_status_t muon_shard_momentum(const muon_shard_momentum_t* shards, int count,
                                           float momentum, int nesterov, void* workspace,
                                           size_t workspace_bytes, void* stream);

MUON_API muon_status_t muon_shard_update(const muon_shard_update_t* shards, int count, float lr,
                                         float weight_decay, float gamma, void* workspace,
                                         size_t workspace_bytes, void* stream);

/* Copy every segment, one launch over all of them (HBM-bound: 8 bytes per
 * element). Pointers need 4-byte alignment; a segment whose two pointers are
 * 16-byte aligned moves 16 bytes per access. 0 <= numel <= 2^40. No
 * destination may overlap another segment's destination or any source. */
MUON_API muon_status_t muon_copy_segments(const muon_segment_t* segs, int count, void* workspace,
                                          size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MUON_SHARD_H */
