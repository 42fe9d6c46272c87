// Newton-Schulz stages in fp32 on the CUDA cores: the validation precision.
//
// Same stages and epilogues as the tensor-core path, with fp32 operands and
// fp32 A, B and iterate buffers (the iterate ping-pongs between two fp32
// buffers because the Apply stage reads the whole current iterate as its
// right operand). Tiles are dense 64 x 64 (no symmetric skipping), K steps of
// 16, 256 threads with a 4 x 4 register tile each. Not a performance path.
//
// Accumulation is fp32 in two levels: each run of kKBlock products goes into a
// fresh partial sum, which is then added to the total. A single running sum
// over K = 2048 .. 65536 products grows its rounding error with the full
// length of K; two levels grow it with about the square root of that. On
// inputs whose spectrum spans four decades, Newton-Schulz magnifies those
// errors along the small singular directions: with one running sum, O' of a
// 2048 x 2048 sweep matrix was 2.3e-4 away from the float64 result, four times
// a float32 BLAS's error on the same input.
#include "kernels.cuh"
#include "stage_common.cuh"

namespace muon {

namespace {

constexpr int kKBlock = 128;  // products per partial sum (a multiple of kSBK)
static_assert(kKBlock % kSBK == 0, "whole K steps per partial sum");

template <int KIND>
__global__ void __launch_bounds__(256) stage_simt_kernel(const __grid_constant__ StageArgs a) {
  __shared__ __align__(16) float As[kSBK][kSBM + 4];
  __shared__ __align__(16) float Bs[kSBK][kSBN + 4];
  __shared__ float red[8];
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;

  for (int64_t t = a.tile_begin + blockIdx.x; t < a.total_tiles; t += gridDim.x) {
    const int g = stage_group<KIND>(a, t);
    const GroupDesc& gd = a.groups[g];
    const int64_t local = t - gd.tile_base[KIND];
    const int64_t per = gd.tiles_per_mat[KIND];
    const int64_t b = local / per;
    const int64_t u = local % per;
    const int64_t r = gd.r, c = gd.c, ldc = gd.ldc, ldr = gd.ldr;
    const int64_t ncols = (KIND == kApply) ? c : r;
    const int64_t col_tiles = (ncols + kSBN - 1) / kSBN;
    const int64_t row0 = (u / col_tiles) * kSBM;
    const int64_t col0 = (u % col_tiles) * kSBN;
    const int64_t K = (KIND == kGram) ? c : r;
    const int mat = gd.first_mat + static_cast<int>(b);

    const float* xcur = reinterpret_cast<const float*>(a.ws + gd.xf_off[a.xsrc]) + b * r * ldc;
    const float* Am = reinterpret_cast<const float*>(a.ws + gd.a_off) + b * r * ldr;
    const float* Bm = reinterpret_cast<const float*>(a.ws + gd.b_off) + b * r * ldr;
    // left operand P (rows = output rows), right operand Q
    const float* P = (KIND == kGram) ? xcur : (KIND == kPoly ? Am : Bm);
    const int64_t ldp = (KIND == kGram) ? ldc : ldr;
    const float* Q = (KIND == kPoly) ? Am : xcur;
    const int64_t ldq = (KIND == kPoly) ? ldr : ldc;

    float acc[4][4] = {};
    float part[4][4] = {};
    for (int64_t k0 = 0; k0 < K; k0 += kSBK) {
      // P tile: As[kk][mm] = P[row0 + mm][k0 + kk]
      for (int idx = tid; idx < kSBK * kSBM; idx += 256) {
        const int mm = idx / kSBK, kk = idx % kSBK;
        const int64_t row = row0 + mm, k = k0 + kk;
        As[kk][mm] = (row < r && k < K) ? P[row * ldp + k] : 0.f;
      }
      if (KIND == kApply) {
        // Bs[kk][nn] = X[k0 + kk][col0 + nn]
        for (int idx = tid; idx < kSBK * kSBN; idx += 256) {
          const int kk = idx / kSBN, nn = idx % kSBN;
          const int64_t k = k0 + kk, col = col0 + nn;
          Bs[kk][nn] = (k < K && col < ncols) ? Q[k * ldq + col] : 0.f;
        }
      } else {
        // Bs[kk][nn] = Q[col0 + nn][k0 + kk]   (Q Q^T form)
        for (int idx = tid; idx < kSBK * kSBN; idx += 256) {
          const int nn = idx / kSBK, kk = idx % kSBK;
          const int64_t col = col0 + nn, k = k0 + kk;
          Bs[kk][nn] = (col < ncols && k < K) ? Q[col * ldq + k] : 0.f;
        }
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < kSBK; ++kk) {
        const float4 av = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
        const float4 bv = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
        const float ar[4] = {av.x, av.y, av.z, av.w};
        const float br[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
        for (int ii = 0; ii < 4; ++ii)
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) part[ii][jj] = fmaf(ar[ii], br[jj], part[ii][jj]);
      }
      if ((k0 + kSBK) % kKBlock == 0 || k0 + kSBK >= K) {
#pragma unroll
        for (int ii = 0; ii < 4; ++ii)
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            acc[ii][jj] += part[ii][jj];
            part[ii][jj] = 0.f;
          }
      }
      __syncthreads();
    }

    // epilogue
    const float s = a.first ? a.scale[mat] : 1.f;
    const MatDesc md = a.mats[mat];
    const UpdateConsts uc = update_consts(a, static_cast<int>(c));
    float* xnext = reinterpret_cast<float*>(a.ws + gd.xf_off[a.xsrc ^ 1]) + b * r * ldc;
    float* Aw = reinterpret_cast<float*>(a.ws + gd.a_off) + b * r * ldr;
    float* Bw = reinterpret_cast<float*>(a.ws + gd.b_off) + b * r * ldr;
    float ssq = 0.f;  // sum of squares of X' over this tile (unit-RMS update scale)
#pragma unroll
    for (int ii = 0; ii < 4; ++ii) {
      const int64_t row = row0 + ty * 4 + ii;
      if (row >= r) continue;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int64_t col = col0 + tx * 4 + jj;
        if (col >= ncols) continue;
        const float v = acc[ii][jj];
        if (KIND == kGram) {
          Aw[row * ldr + col] = s * s * v;
        } else if (KIND == kPoly) {
          Bw[row * ldr + col] = fmaf(a.b, Am[row * ldr + col], a.c * v);
        } else {
          const float x = s * fmaf(a.a, xcur[row * ldc + col], v);
          if (a.last) write_update(md, uc, row, col, x);
          else xnext[row * ldc + col] = x;
          ssq = fmaf(x, x, ssq);
        }
      }
    }
    if (KIND == kApply && a.sumsq_per_tile > 0) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
      if ((tid & 31) == 0) red[tid >> 5] = ssq;
      __syncthreads();
      if (tid == 0) {
        float tot = 0.f;
        for (int w = 0; w < 8; ++w) tot += red[w];
        a.sumsq[t] = tot;
      }
      __syncthreads();
    }
  }
}

}  // namespace

cudaError_t launch_stage_simt(StageKind kind, const StageArgs& args, int grid,
                              cudaStream_t stream) {
  if (args.total_tiles <= args.tile_begin) return cudaSuccess;
  switch (kind) {
    case kGram: stage_simt_kernel<kGram><<<grid, 256, 0, stream>>>(args); break;
    case kPoly: stage_simt_kernel<kPoly><<<grid, 256, 0, stream>>>(args); break;
    case kApply: stage_simt_kernel<kApply><<<grid, 256, 0, stream>>>(args); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace muon
