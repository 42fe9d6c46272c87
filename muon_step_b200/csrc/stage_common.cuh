// Pieces shared by the two implementations of a Newton-Schulz stage.
//
// One Newton-Schulz step X <- a X + b (X X^T) X + c (X X^T)^2 X ("Ch 06 · Muon"
// §3 and §5 Algorithm 1) runs as three GEMM stages with fused epilogues:
//
//   Gram   A = X X^T                 (step one also folds s^2: X_0 = s N)
//   Poly   B = b A + c A A           (A symmetric: A A = A A^T)
//   Apply  X' = a X + B X            (step one folds s)
//
// which is the same polynomial regrouped: (X X^T)^2 X = A (A X) = (A A) X.
// The last step's Apply epilogue instead forms the update of "Muon 优化器完全拆解…",
// Algorithm 1 steps four and five:
//
//   O = O' sqrt(max(n, m)) gamma,   W <- W (1 - lr wd) - lr O
//
// written in the caller's orientation.
#pragma once

#include <cstdint>

#include "muon_internal.h"

namespace muon {

// Which group a stage tile belongs to (groups are few; linear scan).
template <int KIND>
__device__ __forceinline__ int stage_group(const StageArgs& a, int64_t t) {
  int g = 0;
  while (g + 1 < a.ngroups && __ldg(&a.groups[g + 1].tile_base[KIND]) <= t) ++g;
  return g;
}

// Caller-orientation element index of iterate element (row, col).
__device__ __forceinline__ int64_t caller_index(const MatDesc& md, int64_t row, int64_t col) {
  return md.transposed ? col * md.m + row : row * md.m + col;
}

// Update constants of the last step: W' = W * keep - step * O'.
struct UpdateConsts {
  float keep;  // 1 - lr wd
  float step;  // lr gamma sqrt(max(n, m))
};

// Scale modes of the update (muon_scale_mode_t).
enum : int { kScaleShape = 0, kScaleUnitRms = 1, kScaleNone = 2 };

// step = lr gamma sqrt(max(n, m)) (shape), lr gamma (none); the unit-RMS mode
// passes gamma / RMS(O') as `gamma` with the none rule.
__device__ __forceinline__ UpdateConsts update_consts_raw(float lr, float wd, float gamma, int c,
                                                          int scale_mode = kScaleShape) {
  UpdateConsts u;
  u.keep = 1.0f - lr * wd;
  u.step = (scale_mode == kScaleShape) ? lr * gamma * sqrtf(static_cast<float>(c)) : lr * gamma;
  return u;
}

__device__ __forceinline__ UpdateConsts update_consts(const StageArgs& a, int c) {
  return update_consts_raw(a.lr, a.wd, a.gamma, c, a.scale_mode);
}

__device__ __forceinline__ void write_update(const MatDesc& md, const UpdateConsts& u,
                                             int64_t row, int64_t col, float o) {
  const int64_t idx = caller_index(md, row, col);
  if (md.O) md.O[idx] = o;
  if (md.W) md.W[idx] = fmaf(md.W[idx], u.keep, -u.step * o);
}

}  // namespace muon
