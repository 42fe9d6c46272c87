// Launchers of the library's kernels (host side, C++ linkage, internal).
#pragma once

#include <cuda_runtime.h>

#include "muon_internal.h"

namespace muon {

// Momentum + Nesterov (or plain input) + per-tile sums of squares + write of
// the Newton-Schulz iterate in its orientation; the last tile of each matrix
// turns the partial sums into the normalisation scale.
cudaError_t launch_elementwise(const EwArgs& args, cudaStream_t stream);

// One Newton-Schulz stage over every matrix of the plan, bf16 operands on
// the tcgen05 tensor cores (TMA -> shared memory -> MMA -> TMEM -> epilogue).
// `wide`: Gram, Poly or ApplyLast with eight epilogue warps (short main loops);
// Apply always has eight
cudaError_t launch_stage_tc(StageKind kind, const StageArgs& args, int grid, bool wide,
                            cudaStream_t stream);

// Every Gram, Poly and Apply stage listed in args.chain (tiles
// [tile_begin, total_tiles)) in one persistent launch, with per-matrix
// dependency counters args.dep (reset to zero by the elementwise kernel).
// The grid must not exceed 2 * chain_max_pairs(): every CTA pair must be
// resident at once.
cudaError_t launch_stage_chain(const StageArgs& args, int grid, cudaStream_t stream);
cudaError_t chain_max_pairs(int* pairs);

// Every Newton-Schulz step and the update for the small matrices, one CTA
// per matrix (bf16 precision).
cudaError_t launch_small(const SmallArgs& args, int grid, cudaStream_t stream);

// The same for min(n, m) <= 128 < max(n, m) <= 512, one 512-thread CTA per
// matrix (args.small_mats lists those matrices).
cudaError_t launch_mid(const SmallArgs& args, int grid, cudaStream_t stream);

// Matrices of at most kTinyMaxElems elements in the bf16 precision: every
// step and the update with fp32 operands, one CTA per matrix (args.small_mats
// lists those matrices).
cudaError_t launch_tiny(const SmallArgs& args, int grid, cudaStream_t stream);

// Unit-RMS update scale, grouped / fp32 path: per-matrix RMS of O' from the
// last Apply's sums of squares, then W <- W (1 - lr wd) - lr (gamma / RMS) O'.
cudaError_t launch_rms_reduce(const FinishArgs& args, cudaStream_t stream);
cudaError_t launch_finish(const FinishArgs& args, cudaStream_t stream);

// The same stage in fp32 on the CUDA cores (validation precision).
cudaError_t launch_stage_simt(StageKind kind, const StageArgs& args, int grid,
                              cudaStream_t stream);

// Dynamic shared memory the tcgen05 stage kernels need.
size_t stage_tc_smem_bytes();

// Copy `bytes` (a multiple of 16) of host memory to `dst` (16-byte aligned)
// through kernel arguments, 32 KB per launch (all-zero chunks as memsets):
// once the call returns, no pending device work refers to `src`.
cudaError_t launch_blob_copy(void* dst, const void* src, size_t bytes, cudaStream_t stream);

// Bounded wait on a host-visible word that nothing sets: used by the tests of
// the timeout path. Sets the timeout bit of `err` when the limit passes.
cudaError_t launch_wait_probe(const int* flag, int* err, unsigned long long limit_ns,
                              cudaStream_t stream);

// The chained launch's dependency wait on `counter` >= target, alone, for
// the tests of its timeout path.
cudaError_t launch_dep_wait_probe(const uint32_t* counter, uint32_t target, int* err,
                                  unsigned long long limit_ns, cudaStream_t stream);

}  // namespace muon
