// Update pass of the unit-RMS scale mode for matrices on the grouped (or
// fp32) path.
//
// "Muon 优化器完全拆解…", section "另一条路：开源生态干脆不分片": the Megatron-Bridge recipe scales
// the update to unit RMS and then by an extra factor, O = gamma O' / RMS(O').
// RMS(O') needs all of O' before any element of W can move, so here the last
// Apply stage keeps O' in the iterate buffers and records sums of squares per
// tile; then
//
//   rms_reduce_kernel   one CTA per matrix adds its tiles' sums in a fixed
//                       order (double) and stores gamma / RMS(O') (0 when
//                       O' = 0);
//   finish_kernel       W <- W (1 - lr wd) - lr factor O' (and O = O'), over
//                       64 x 128 tiles of the caller's matrix; when the
//                       iterate is the transpose, the tile is read through
//                       shared memory so every global access stays coalesced.
//
// HBM-bound: 4 B of O' read (fp32, or bf16 high + low parts), 8 B of W read
// and written per element. Where the caller's rows allow 16-byte accesses
// and the iterate is not transposed, a thread takes four consecutive columns
// (one 16-byte piece of W, two 8-byte pieces of O') of eight rows, loading
// four rows before it stores any, as the elementwise kernel does. (Transposed
// tiles keep one column per thread: four-column reads of the staged tile
// would meet four-way bank conflicts.)
//
// With diagnostics on, rms_reduce_kernel also runs after a fused last step (any
// scale mode) and writes the RMS of the applied update per matrix.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "stage_common.cuh"

namespace muon {

namespace {

__global__ void __launch_bounds__(256) rms_reduce_kernel(const __grid_constant__ FinishArgs a) {
  __shared__ double part[8];
  const int mat = blockIdx.x;
  const MatDesc& md = a.mats[mat];
  const GroupDesc& gd = a.groups[md.group];
  if (gd.small) return;  // the small-matrix kernel has already updated it
  const int64_t per = gd.tiles_per_mat[a.apply_kind];
  const int64_t first = (gd.tile_base[a.apply_kind] + md.index * per) * a.sumsq_per_tile;
  const int64_t count = per * a.sumsq_per_tile;
  double acc = 0.0;
  for (int64_t k = threadIdx.x; k < count; k += blockDim.x) acc += static_cast<double>(a.sumsq[first + k]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int w = 0; w < 8; ++w) tot += part[w];
    const double rms = sqrt(tot / (static_cast<double>(md.n) * static_cast<double>(md.m)));
    a.factor[mat] = rms > 0.0 ? static_cast<float>(static_cast<double>(a.gamma) / rms) : 0.f;
    if (a.diag) {
      // RMS of the applied update O: gamma sqrt(max(n, m)) RMS(O') (shape), gamma
      // (unit RMS; 0 when O' = 0) or gamma RMS(O') (none)
      double o_rms = static_cast<double>(a.gamma) * rms;
      if (a.scale_mode == kScaleShape) o_rms *= sqrt(static_cast<double>(gd.c));
      if (a.scale_mode == kScaleUnitRms) o_rms = rms > 0.0 ? static_cast<double>(a.gamma) : 0.0;
      a.diag[2 * md.caller + 1] = static_cast<float>(o_rms);
    }
  }
}

__global__ void __launch_bounds__(256, 4) finish_kernel(const __grid_constant__ FinishArgs a) {
  __shared__ float stage[kEwRows][kEwCols + 1];
  const int tid = threadIdx.x;
  const int64_t tile = blockIdx.x;
  const int mat = __ldg(&a.tile_mat[tile]);
  const MatDesc md = a.mats[mat];
  const GroupDesc& gd = a.groups[md.group];
  if (gd.small) return;
  const int64_t n = md.n, m = md.m;
  const int64_t col_tiles = (m + kEwCols - 1) / kEwCols;
  const int64_t local = tile - md.ew_tile_begin;
  const int64_t row0 = (local / col_tiles) * kEwRows;
  const int64_t col0 = (local % col_tiles) * kEwCols;
  const int64_t ldc = gd.ldc;
  const int64_t mo = static_cast<int64_t>(md.index) * gd.r * ldc;
  const float* of = reinterpret_cast<const float*>(a.ws + gd.xf_off[a.xf_slot]) + mo;
  const __nv_bfloat16* oh = reinterpret_cast<const __nv_bfloat16*>(a.ws + gd.xb_off[a.xf_slot]) + mo;
  const __nv_bfloat16* ol = reinterpret_cast<const __nv_bfloat16*>(a.ws + gd.xlo_off) + mo;
  // O' element at iterate offset k: fp32, or high + low parts
  auto o_at = [&](int64_t k) -> float {
    return a.split ? __bfloat162float(oh[k]) + __bfloat162float(ol[k]) : of[k];
  };
  const UpdateConsts uc = update_consts_raw(a.lr, a.wd, a.factor[mat], gd.c, kScaleNone);

  const bool vec = !md.transposed && (m & 3) == 0 &&
                   ((reinterpret_cast<uintptr_t>(md.W) | reinterpret_cast<uintptr_t>(md.O)) & 15) == 0;
  if (vec) {
    // thread -> columns c4 .. c4 + 3, rows r0 + 8 k; ldc is a multiple of 8,
    // so the four iterate elements are one 8-byte piece per bf16 part
    static_assert(kEwCols == 128 && kEwRows == 64, "32 lanes x 4 columns, 8 warps x 8 rows");
    const int c4 = (tid & 31) * 4;
    const int r0 = tid >> 5;
    const int64_t col = col0 + c4;
    const bool col_ok = col < m;  // m % 4 == 0: all four columns are in range
#pragma unroll
    for (int ph = 0; ph < 2; ++ph) {
      float4 w4[4], o4[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t row = row0 + r0 + 8 * (4 * ph + j);
        w4[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        o4[j] = w4[j];
        if (!col_ok || row >= n) continue;
        const int64_t k = row * ldc + col;
        if (a.split) {
          const uint2 hr = *reinterpret_cast<const uint2*>(oh + k);
          const uint2 lr = *reinterpret_cast<const uint2*>(ol + k);
          const float2 h0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hr.x));
          const float2 h1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hr.y));
          const float2 l0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&lr.x));
          const float2 l1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&lr.y));
          o4[j] = make_float4(h0.x + l0.x, h0.y + l0.y, h1.x + l1.x, h1.y + l1.y);
        } else {
          o4[j] = *reinterpret_cast<const float4*>(of + k);
        }
        if (md.W) w4[j] = *reinterpret_cast<const float4*>(md.W + row * m + col);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t row = row0 + r0 + 8 * (4 * ph + j);
        if (!col_ok || row >= n) continue;
        if (md.O) *reinterpret_cast<float4*>(md.O + row * m + col) = o4[j];
        if (md.W) {
          float4 w = w4[j];
          w.x = fmaf(w.x, uc.keep, -uc.step * o4[j].x);
          w.y = fmaf(w.y, uc.keep, -uc.step * o4[j].y);
          w.z = fmaf(w.z, uc.keep, -uc.step * o4[j].z);
          w.w = fmaf(w.w, uc.keep, -uc.step * o4[j].w);
          *reinterpret_cast<float4*>(md.W + row * m + col) = w;
        }
      }
    }
    return;
  }

  if (md.transposed) {
    // O'(caller i, j) is iterate element (j, i): read iterate rows j, two
    // consecutive i per lane, 64 per warp access
    static_assert(kEwRows == 64, "two caller rows per lane");
    const int w = tid >> 5, lane = tid & 31;
    const int64_t i = row0 + 2 * lane;
#pragma unroll 4
    for (int q = 0; q < kEwCols / 8; ++q) {
      const int cc = w * (kEwCols / 8) + q;
      const int64_t j = col0 + cc;
      const bool jin = j < m;
      stage[2 * lane][cc] = (i < n && jin) ? o_at(j * ldc + i) : 0.f;
      stage[2 * lane + 1][cc] = (i + 1 < n && jin) ? o_at(j * ldc + i + 1) : 0.f;
    }
    __syncthreads();
  }
  // caller element (row, col): thread -> one column, rows (tid / 128) + 2 k,
  // in two halves of the tile (loads of a half before its stores)
  constexpr int R = kEwRows / 4;
  const int cc = tid & (kEwCols - 1);
  const int64_t col = col0 + cc;
#pragma unroll 1
  for (int half = 0; half < 2; ++half) {
    const int r0 = half * (kEwRows / 2) + (tid >> 7);
    float o[R], w[R];
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const int rr = r0 + 2 * k;
      const int64_t row = row0 + rr;
      const bool in = row < n && col < m;
      o[k] = !in ? 0.f : (md.transposed ? stage[rr][cc] : o_at(row * ldc + col));
      w[k] = (in && md.W) ? md.W[row * m + col] : 0.f;
    }
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const int64_t row = row0 + r0 + 2 * k;
      if (row >= n || col >= m) continue;
      if (md.O) md.O[row * m + col] = o[k];
      if (md.W) md.W[row * m + col] = fmaf(w[k], uc.keep, -uc.step * o[k]);
    }
  }
}

}  // namespace

cudaError_t launch_rms_reduce(const FinishArgs& args, cudaStream_t stream) {
  if (args.nmats <= 0) return cudaSuccess;
  rms_reduce_kernel<<<args.nmats, 256, 0, stream>>>(args);
  return cudaGetLastError();
}

cudaError_t launch_finish(const FinishArgs& args, cudaStream_t stream) {
  if (args.total_tiles <= 0) return cudaSuccess;
  if (args.total_tiles > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  finish_kernel<<<static_cast<unsigned>(args.total_tiles), 256, 0, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace muon
