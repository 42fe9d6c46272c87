// Elementwise front of the Muon step, one pass over G and M:
//
//   M_t = mu M_{t-1} + G_t                  (momentum accumulation)
//   N_t = mu M_t + G_t                      (Nesterov look-ahead)
//   X_0 = N_t (or N_t^T when n > m)         (orientation rows <= cols)
//   s   = 1 / (||N_t||_F + eps)             (Frobenius normalisation scale)
//
// "Muon 优化器完全拆解…" (pinghaoyang.com.cn), section "V4 的完整更新公式，逐行拆解",
// Algorithm 1 steps one and two; "Ch 06 · Muon" §5 Algorithm 1 (momentum,
// Nesterov and the division by ||N_t||_F). The scale s is not applied here:
// the first Newton-Schulz step folds s^2 into the Gram matrix and s into the
// iterate, so the unscaled N is written once: in bf16 mode as a bf16 high part
// (the tensor-core operand) plus a bf16 low part, N = high + low to 16
// significant bits; in fp32 mode as fp32.
//
// HBM-bound: each element reads G and M (8 B) and writes M and the two bf16
// parts (8 B; fp32 mode: M and the fp32 iterate). Tiles are 64 x 128 elements; a tile's threads
// read and write whole 128-byte lines (64 x 128 elements). When the iterate is the transpose, the
// tile is staged in shared memory so that the transposed writes stay
// coalesced. Per-tile partial sums of squares go to a buffer; the last tile of
// each matrix to finish (arrival counter) adds them in a fixed order, in
// double, so the norm is deterministic.
#include <cuda_bf16.h>

#include "kernels.cuh"

namespace muon {

namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

struct alignas(8) Bf16x4 {
  __nv_bfloat162 lo, hi;
};

}  // namespace

__global__ void __launch_bounds__(256) ew_kernel(const __grid_constant__ EwArgs a) {
  __shared__ float stage[kEwRows][kEwCols + 1];
  __shared__ float warp_part[8];
  __shared__ double warp_part_d[8];
  __shared__ int is_last;

  const int tid = threadIdx.x;
  const int64_t tile = blockIdx.x;
  const int mi = __ldg(&a.tile_mat[tile]);
  const MatDesc md = a.mats[mi];
  const GroupDesc& gd = a.groups[md.group];
  const int64_t n = md.n, m = md.m;
  const int64_t col_tiles = (m + kEwCols - 1) / kEwCols;
  const int64_t local = tile - md.ew_tile_begin;
  const int64_t row0 = (local / col_tiles) * kEwRows;
  const int64_t col0 = (local % col_tiles) * kEwCols;

  const int64_t ldc = gd.ldc;
  const int64_t mat_elems = static_cast<int64_t>(gd.r) * ldc;
  // fp32 mode: the fp32 iterate; bf16 mode: its bf16 high part (the MMA
  // operand) and low part, N = high + low to 16 significant bits
  float* xf = reinterpret_cast<float*>(a.ws + gd.xf_off[0]) + md.index * mat_elems;
  __nv_bfloat16* xb = reinterpret_cast<__nv_bfloat16*>(a.ws + gd.xb_off[0]) + md.index * mat_elems;
  __nv_bfloat16* xl = reinterpret_cast<__nv_bfloat16*>(a.ws + gd.xlo_off) + md.index * mat_elems;
  const int lo_kind = gd.small;  // layout of the low part (lo_index)
  // mid-size matrices keep the low part in 8-column groups: it is written
  // from the staged tile in a second pass, one 16-byte piece per thread
  const bool lo_staged = a.split && lo_kind == 2;
  auto put = [&](int64_t irow, int64_t icol, float v) {  // iterate element (irow, icol)
    const int64_t xo = irow * ldc + icol;
    if (a.split) {
      const __nv_bfloat16 h = __float2bfloat16_rn(v);
      xb[xo] = h;
      if (!lo_staged)
        xl[lo_index(lo_kind, gd.r, ldc, irow, icol)] = __float2bfloat16_rn(v - __bfloat162float(h));
    } else {
      xf[xo] = v;
    }
  };
  const bool transposed = md.transposed != 0;
  const float mu = a.mu;
  float sumsq = 0.f;

  // N for one element: momentum update written back, look-ahead returned.
  auto step = [&](float g, float mprev, float* mdst) -> float {
    if (a.mode != 0) return g;
    const float mt = fmaf(mu, mprev, g);
    *mdst = mt;
    return a.nesterov ? fmaf(mu, mt, g) : mt;
  };

  const bool vec = ((m & 3) == 0) &&
                   (((reinterpret_cast<uintptr_t>(md.G) | reinterpret_cast<uintptr_t>(md.M)) & 15) == 0);
  if (vec) {
    // thread -> 4 consecutive columns, rows (tid / 32) + 8 k; every load is
    // issued before the first store
    constexpr int R = kEwRows / 8;
    const int c4 = (tid & 31) * 4;
    const int64_t col = col0 + c4;
    float4 g4[R], m4[R];
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const int64_t row = row0 + (tid >> 5) + 8 * k;
      g4[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      m4[k] = g4[k];
      if (row < n && col < m) {  // m % 4 == 0: the 4 columns are all in range
        const int64_t off = row * m + col;
        g4[k] = __ldcs(reinterpret_cast<const float4*>(md.G + off));
        if (a.mode == 0) m4[k] = __ldcs(reinterpret_cast<const float4*>(md.M + off));
      }
    }
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const int rr = (tid >> 5) + 8 * k;
      const int64_t row = row0 + rr;
      float nv[4] = {0.f, 0.f, 0.f, 0.f};
      if (row < n && col < m) {
        const int64_t off = row * m + col;
        float4 mo;
        nv[0] = step(g4[k].x, m4[k].x, &mo.x);
        nv[1] = step(g4[k].y, m4[k].y, &mo.y);
        nv[2] = step(g4[k].z, m4[k].z, &mo.z);
        nv[3] = step(g4[k].w, m4[k].w, &mo.w);
        if (a.mode == 0) __stcs(reinterpret_cast<float4*>(md.M + off), mo);
        sumsq += nv[0] * nv[0] + nv[1] * nv[1] + nv[2] * nv[2] + nv[3] * nv[3];
        if (!transposed) {
          const int64_t xo = row * ldc + col;
          if (a.split) {
            Bf16x4 h, l;
            h.lo = __floats2bfloat162_rn(nv[0], nv[1]);
            h.hi = __floats2bfloat162_rn(nv[2], nv[3]);
            const float2 h01 = __bfloat1622float2(h.lo), h23 = __bfloat1622float2(h.hi);
            l.lo = __floats2bfloat162_rn(nv[0] - h01.x, nv[1] - h01.y);
            l.hi = __floats2bfloat162_rn(nv[2] - h23.x, nv[3] - h23.y);
            *reinterpret_cast<Bf16x4*>(xb + xo) = h;
            if (!lo_staged) *reinterpret_cast<Bf16x4*>(xl + lo_index(lo_kind, gd.r, ldc, row, col)) = l;
          } else {
            *reinterpret_cast<float4*>(xf + xo) = make_float4(nv[0], nv[1], nv[2], nv[3]);
          }
        }
      }
      if (transposed || lo_staged) {
#pragma unroll
        for (int e = 0; e < 4; ++e) stage[rr][c4 + e] = nv[e];
      }
    }
  } else {
    // scalar path: thread -> one column, rows (tid / 128) + 2 k; loads first
    constexpr int R = kEwRows / 2;
    const int cc = tid & (kEwCols - 1);
    const int64_t col = col0 + cc;
    float gs[R], ms[R];
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const int64_t row = row0 + (tid >> 7) + 2 * k;
      gs[k] = 0.f;
      ms[k] = 0.f;
      if (row < n && col < m) {
        const int64_t off = row * m + col;
        gs[k] = __ldcs(md.G + off);
        if (a.mode == 0) ms[k] = __ldcs(md.M + off);
      }
    }
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const int rr = (tid >> 7) + 2 * k;
      const int64_t row = row0 + rr;
      float nv = 0.f;
      if (row < n && col < m) {
        const int64_t off = row * m + col;
        float mo;
        nv = step(gs[k], ms[k], &mo);
        if (a.mode == 0) __stcs(md.M + off, mo);
        sumsq += nv * nv;
        if (!transposed) {
          put(row, col, nv);
        }
      }
      if (transposed || lo_staged) stage[rr][cc] = nv;
    }
  }

  if (transposed) {
    // iterate row j = caller column, iterate columns i, i + 1 = caller rows:
    // each lane writes two consecutive elements, a warp 64 of one iterate row
    static_assert(kEwRows == 64, "two caller rows per lane");
    __syncthreads();
    const int w = tid >> 5, lane = tid & 31;
    const int64_t i = row0 + 2 * lane;
#pragma unroll 4
    for (int q = 0; q < kEwCols / 8; ++q) {
      const int cc = w * (kEwCols / 8) + q;
      const int64_t j = col0 + cc;
      if (j >= m || i >= n) continue;
      const float v0 = stage[2 * lane][cc], v1 = stage[2 * lane + 1][cc];
      const int64_t xo = j * ldc + i;  // even: 4-byte aligned pairs (8 bytes in fp32)
      if (i + 1 < n) {
        if (a.split) {
          const __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
          const float2 fh = __bfloat1622float2(h);
          *reinterpret_cast<__nv_bfloat162*>(xb + xo) = h;
          if (!lo_staged)
            *reinterpret_cast<__nv_bfloat162*>(xl + lo_index(lo_kind, gd.r, ldc, j, i)) =
                __floats2bfloat162_rn(v0 - fh.x, v1 - fh.y);
        } else {
          *reinterpret_cast<float2*>(xf + xo) = make_float2(v0, v1);
        }
      } else {
        put(j, i, v0);
      }
    }
  }

  if (lo_staged) {
    // low part of a mid-size matrix, [col / 8][row][col % 8]: 16-byte pieces,
    // consecutive threads on consecutive iterate rows (contiguous addresses)
    if (!transposed) __syncthreads();  // (the transposed pass has synchronised already)
    constexpr int kPieces = kEwRows * kEwCols / 8;
    for (int p = tid; p < kPieces; p += blockDim.x) {
      float v[8];
      int64_t irow, icol0;
      if (!transposed) {
        // iterate rows = caller rows row0 .., columns col0 + 8 g ..
        const int g = p / kEwRows, rr = p % kEwRows;
        irow = row0 + rr;
        icol0 = col0 + 8 * g;
        if (irow >= n || icol0 >= m) continue;
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = stage[rr][8 * g + e];
      } else {
        // iterate rows = caller columns col0 + cc, columns = caller rows row0 + 8 g ..
        const int g = p / kEwCols, cc = p % kEwCols;
        irow = col0 + cc;
        icol0 = row0 + 8 * g;
        if (irow >= m || icol0 >= n) continue;
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = stage[8 * g + e][cc];
      }
      Bf16x4 l0, l1;
      const __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]), h1 = __floats2bfloat162_rn(v[2], v[3]);
      const __nv_bfloat162 h2 = __floats2bfloat162_rn(v[4], v[5]), h3 = __floats2bfloat162_rn(v[6], v[7]);
      const float2 f0 = __bfloat1622float2(h0), f1 = __bfloat1622float2(h1);
      const float2 f2 = __bfloat1622float2(h2), f3 = __bfloat1622float2(h3);
      l0.lo = __floats2bfloat162_rn(v[0] - f0.x, v[1] - f0.y);
      l0.hi = __floats2bfloat162_rn(v[2] - f1.x, v[3] - f1.y);
      l1.lo = __floats2bfloat162_rn(v[4] - f2.x, v[5] - f2.y);
      l1.hi = __floats2bfloat162_rn(v[6] - f3.x, v[7] - f3.y);
      __nv_bfloat16* dst = xl + lo_index(lo_kind, gd.r, ldc, irow, icol0);  // 16-byte aligned
      reinterpret_cast<Bf16x4*>(dst)[0] = l0;
      reinterpret_cast<Bf16x4*>(dst)[1] = l1;
    }
  }

  // tile partial sum of squares
  sumsq = warp_sum(sumsq);
  if ((tid & 31) == 0) warp_part[tid >> 5] = sumsq;
  __syncthreads();
  if (tid == 0) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += warp_part[w];
    a.partial[tile] = s;
    __threadfence();
    const unsigned prev = atomicAdd(&a.counter[mi], 1u);
    is_last = (prev + 1 == static_cast<unsigned>(md.ew_tiles));
  }
  __syncthreads();
  if (!is_last) return;

  // last tile of this matrix: fixed-order double sum of the partials
  __threadfence();
  double acc = 0.0;
  for (int64_t k = tid; k < md.ew_tiles; k += blockDim.x)
    acc += static_cast<double>(__ldcg(a.partial + md.ew_tile_begin + k));
  acc = warp_sum_d(acc);
  if ((tid & 31) == 0) warp_part_d[tid >> 5] = acc;
  __syncthreads();
  if (tid == 0) {
    double s = 0.0;
    for (int w = 0; w < 8; ++w) s += warp_part_d[w];
    a.scale[mi] = static_cast<float>(1.0 / (sqrt(s) + static_cast<double>(a.eps)));
    if (a.diag) a.diag[2 * md.caller] = static_cast<float>(sqrt(s));
    a.counter[mi] = 0u;
  }
}

cudaError_t launch_elementwise(const EwArgs& args, cudaStream_t stream) {
  if (args.total_tiles <= 0) return cudaSuccess;
  if (args.total_tiles > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  ew_kernel<<<static_cast<unsigned>(args.total_tiles), 256, 0, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace muon
