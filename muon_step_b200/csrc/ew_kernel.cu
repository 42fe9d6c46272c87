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
// parts (8 B; fp32 mode: M and the fp32 iterate). Tiles are 64 x 128
// elements, and a tile's threads read and write whole 128-byte lines. When
// the iterate is the transpose, the tile is staged in shared memory so that
// the transposed writes stay coalesced. Per-tile partial sums of squares go to a buffer; the last tile of
// each matrix to finish (arrival counter) adds them in a fixed order, in
// double, so the norm is deterministic.
//
// Each CTA lives for one tile, so what keeps HBM busy is the number of loads
// in flight per SM: the kernel is built for 4 resident CTAs per SM (64
// registers a thread), and a thread loads its 8 rows in two phases of 4, which
// keeps 4 CTAs x 32 KB of reads in flight per SM without spilling. The
// per-element work is kept to the arithmetic itself: the tile position is a
// 32-bit division, each thread walks its rows with pointer increments, and
// outside the mid-size layout the low part sits at the high part's offset.
// The sums of squares are taken in the same order whatever the phases, so the
// norm does not depend on them.
#include <cuda_bf16.h>

#include "kernels.cuh"

namespace muon {

namespace {

constexpr int kEwThreads = 256;
constexpr int kEwWarps = kEwThreads / 32;
constexpr int kEwMinBlocks = 4;  // CTAs resident per SM: a budget of 64 registers
constexpr int kEwPhases = 2;     // load phases of a thread's 8 rows (4 rows in flight)

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

// high and low bf16 parts of four consecutive iterate elements
__device__ __forceinline__ void split4(const float (&v)[4], Bf16x4& h, Bf16x4& l) {
  h.lo = __floats2bfloat162_rn(v[0], v[1]);
  h.hi = __floats2bfloat162_rn(v[2], v[3]);
  const float2 h01 = __bfloat1622float2(h.lo), h23 = __bfloat1622float2(h.hi);
  l.lo = __floats2bfloat162_rn(v[0] - h01.x, v[1] - h01.y);
  l.hi = __floats2bfloat162_rn(v[2] - h23.x, v[3] - h23.y);
}

}  // namespace

__global__ void __launch_bounds__(kEwThreads, kEwMinBlocks) ew_kernel(const __grid_constant__ EwArgs a) {
  __shared__ float stage[kEwRows][kEwCols + 1];
  __shared__ float warp_part[kEwWarps];
  __shared__ double warp_part_d[kEwWarps];
  __shared__ int is_last;

  const int tid = threadIdx.x;
  const int64_t tile = blockIdx.x;
  const int mi = __ldg(&a.tile_mat[tile]);
  const MatDesc md = a.mats[mi];
  const GroupDesc& gd = a.groups[md.group];
  const int64_t n = md.n, m = md.m;
  const int64_t ldc = gd.ldc;
  if (a.next_tile && tile == 0 && tid == 0) *a.next_tile = 0u;  // the chained launch's list starts over
  const int gr = gd.r;
  const int lo_kind = gd.small;  // layout of the low part (lo_index)

  // tile position: row band and column tile within the matrix
  const int64_t col_tiles = (m + kEwCols - 1) / kEwCols;
  const int64_t local = tile - md.ew_tile_begin;
  int64_t band, ctile;
  if ((local | col_tiles) < 0x80000000LL) {
    const uint32_t l32 = static_cast<uint32_t>(local), c32 = static_cast<uint32_t>(col_tiles);
    const uint32_t b32 = l32 / c32;
    band = b32;
    ctile = l32 - b32 * c32;
  } else {
    band = local / col_tiles;
    ctile = local - band * col_tiles;
  }
  const int64_t row0 = band * kEwRows;
  const int64_t col0 = ctile * kEwCols;
  // rows and columns of the caller matrix inside this tile (1 .. 64, 1 .. 128)
  const int rows = static_cast<int>(n - row0 < kEwRows ? n - row0 : kEwRows);
  const int cols = static_cast<int>(m - col0 < kEwCols ? m - col0 : kEwCols);

  const int64_t mat_elems = static_cast<int64_t>(gr) * ldc;
  // fp32 mode: the fp32 iterate; bf16 mode: its bf16 high part (the MMA
  // operand) and low part, N = high + low to 16 significant bits
  float* xf = reinterpret_cast<float*>(a.ws + gd.xf_off[0]) + md.index * mat_elems;
  __nv_bfloat16* xb = reinterpret_cast<__nv_bfloat16*>(a.ws + gd.xb_off[0]) + md.index * mat_elems;
  __nv_bfloat16* xl = reinterpret_cast<__nv_bfloat16*>(a.ws + gd.xlo_off) + md.index * mat_elems;
  // mid-size matrices keep the low part in 8-column groups: it is written
  // from the staged tile in a second pass, one 16-byte piece per thread
  const bool lo_staged = a.split && lo_kind == 2;
  const bool split = a.split != 0;
  const bool transposed = md.transposed != 0;
  const bool stage_tile = transposed || lo_staged;
  const bool momentum = a.mode == 0;
  const bool nesterov = a.nesterov != 0;
  const float mu = a.mu;
  float sumsq = 0.f;

  // N for one element: momentum update returned in mt, look-ahead returned.
  auto step = [&](float g, float mprev, float& mt) -> float {
    if (!momentum) return g;
    mt = fmaf(mu, mprev, g);
    return nesterov ? fmaf(mu, mt, g) : mt;
  };
  // one iterate element (irow, icol) outside the vector paths
  auto put = [&](int64_t irow, int64_t icol, float v) {
    const int64_t xo = irow * ldc + icol;
    if (split) {
      const __nv_bfloat16 h = __float2bfloat16_rn(v);
      xb[xo] = h;
      if (!lo_staged)
        xl[lo_index(lo_kind, gr, ldc, irow, icol)] = __float2bfloat16_rn(v - __bfloat162float(h));
    } else {
      xf[xo] = v;
    }
  };

  const bool vec = ((m & 3) == 0) &&
                   (((reinterpret_cast<uintptr_t>(md.G) | reinterpret_cast<uintptr_t>(md.M)) & 15) == 0);
  if (vec) {
    // thread -> 4 consecutive columns, rows r0 + kEwWarps k; every load is
    // issued before the first store. Outside the mid-size layout the low part
    // of element (row, col) sits at the high part's offset row ldc + col.
    constexpr int R = kEwRows / kEwWarps;
    const int c4 = (tid & 31) * 4;
    const int r0 = tid >> 5;
    const bool col_ok = c4 < cols;  // m % 4 == 0: the 4 columns are all in range
    const float4* gp = reinterpret_cast<const float4*>(md.G + (row0 + r0) * m + col0 + c4);
    float4* mp = momentum ? reinterpret_cast<float4*>(md.M + (row0 + r0) * m + col0 + c4) : nullptr;
    const int64_t gstep = static_cast<int64_t>(kEwWarps) * m / 4;  // float4 per kEwWarps rows
    const int64_t xo0 = (row0 + r0) * ldc + col0 + c4;
    const int64_t xstep = static_cast<int64_t>(kEwWarps) * ldc;
    constexpr int RP = R / kEwPhases;
#pragma unroll
    for (int ph = 0; ph < kEwPhases; ++ph) {
      float4 g4[RP], m4[RP];
#pragma unroll
      for (int j = 0; j < RP; ++j) {
        const int k = ph * RP + j;
        g4[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        m4[j] = g4[j];
        if (col_ok && r0 + kEwWarps * k < rows) {
          g4[j] = __ldcs(gp + k * gstep);
          if (momentum) m4[j] = __ldcs(mp + k * gstep);
        }
      }
#pragma unroll
      for (int j = 0; j < RP; ++j) {
        const int k = ph * RP + j;
        const int rr = r0 + kEwWarps * k;
        float nv[4] = {0.f, 0.f, 0.f, 0.f};
        if (col_ok && rr < rows) {
          float4 mo;
          nv[0] = step(g4[j].x, m4[j].x, mo.x);
          nv[1] = step(g4[j].y, m4[j].y, mo.y);
          nv[2] = step(g4[j].z, m4[j].z, mo.z);
          nv[3] = step(g4[j].w, m4[j].w, mo.w);
          if (momentum) __stcs(mp + k * gstep, mo);
          sumsq += nv[0] * nv[0] + nv[1] * nv[1] + nv[2] * nv[2] + nv[3] * nv[3];
          if (!transposed) {
            const int64_t xo = xo0 + k * xstep;
            if (split) {
              Bf16x4 h, l;
              split4(nv, h, l);
              *reinterpret_cast<Bf16x4*>(xb + xo) = h;
              if (!lo_staged) *reinterpret_cast<Bf16x4*>(xl + xo) = l;
            } else {
              *reinterpret_cast<float4*>(xf + xo) = make_float4(nv[0], nv[1], nv[2], nv[3]);
            }
          }
        }
        if (stage_tile) {
#pragma unroll
          for (int e = 0; e < 4; ++e) stage[rr][c4 + e] = nv[e];
        }
      }
    }
  } else {
    // scalar path (m % 4 != 0 or unaligned rows): thread -> one column, rows
    // r0 + kRowStep k, loaded eight rows ahead of their use
    constexpr int kRowStep = kEwThreads / kEwCols;
    constexpr int R = kEwRows / kRowStep;
    const int cc = tid & (kEwCols - 1);
    const int r0 = tid / kEwCols;
    const bool col_ok = cc < cols;
    const float* gp = md.G + (row0 + r0) * m + col0 + cc;
    float* mp = momentum ? md.M + (row0 + r0) * m + col0 + cc : nullptr;
    const int64_t gstep = static_cast<int64_t>(kRowStep) * m;
    constexpr int kChunk = 16;  // rows loaded ahead of their use
#pragma unroll 1
    for (int k0 = 0; k0 < R; k0 += kChunk) {
      float gs[kChunk], ms[kChunk];
#pragma unroll
      for (int j = 0; j < kChunk; ++j) {
        const int k = k0 + j;
        gs[j] = 0.f;
        ms[j] = 0.f;
        if (col_ok && r0 + kRowStep * k < rows) {
          gs[j] = __ldcs(gp + k * gstep);
          if (momentum) ms[j] = __ldcs(mp + k * gstep);
        }
      }
#pragma unroll
      for (int j = 0; j < kChunk; ++j) {
        const int k = k0 + j;
        const int rr = r0 + kRowStep * k;
        float nv = 0.f;
        if (col_ok && rr < rows) {
          float mo;
          nv = step(gs[j], ms[j], mo);
          if (momentum) __stcs(mp + k * gstep, mo);
          sumsq += nv * nv;
          if (!transposed) put(row0 + rr, col0 + cc, nv);
        }
        if (stage_tile) stage[rr][cc] = nv;
      }
    }
  }

  if (transposed) {
    // iterate row j = caller column, iterate columns i, i + 1 = caller rows:
    // each lane writes two consecutive elements, a warp 64 of one iterate row
    static_assert(kEwRows == 64, "two caller rows per lane");
    constexpr int Q = kEwCols / kEwWarps;  // iterate rows per warp
    __syncthreads();
    const int w = tid >> 5, lane = tid & 31;
    const int il = 2 * lane;  // caller row within the tile
    if (il < rows) {
      const bool pair = il + 1 < rows;
      int64_t xo = (col0 + w * Q) * ldc + row0 + il;  // even: 4-byte aligned pairs (8 bytes in fp32)
#pragma unroll 4
      for (int q = 0; q < Q; ++q, xo += ldc) {
        const int cc = w * Q + q;
        if (cc >= cols) break;
        const float v0 = stage[il][cc];
        if (pair) {
          const float v1 = stage[il + 1][cc];
          if (split) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
            const float2 fh = __bfloat1622float2(h);
            *reinterpret_cast<__nv_bfloat162*>(xb + xo) = h;
            if (!lo_staged)
              *reinterpret_cast<__nv_bfloat162*>(xl + lo_index(lo_kind, gr, ldc, col0 + cc, row0 + il)) =
                  __floats2bfloat162_rn(v0 - fh.x, v1 - fh.y);
          } else {
            *reinterpret_cast<float2*>(xf + xo) = make_float2(v0, v1);
          }
        } else {
          put(col0 + cc, row0 + il, v0);
        }
      }
    }
  }

  if (lo_staged) {
    // low part of a mid-size matrix, [col / 8][row][col % 8]: 16-byte pieces,
    // consecutive threads on consecutive iterate rows (contiguous addresses)
    if (!transposed) __syncthreads();  // (the transposed pass has synchronised already)
    constexpr int kPieces = kEwRows * kEwCols / 8;
    for (int p = tid; p < kPieces; p += kEwThreads) {
      float v[8];
      int64_t irow, icol0;
      if (!transposed) {
        // iterate rows = caller rows row0 .., columns col0 + 8 g ..
        const int g = p / kEwRows, rr = p % kEwRows;
        if (rr >= rows || 8 * g >= cols) continue;
        irow = row0 + rr;
        icol0 = col0 + 8 * g;
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = stage[rr][8 * g + e];
      } else {
        // iterate rows = caller columns col0 + cc, columns = caller rows row0 + 8 g ..
        const int g = p / kEwCols, cc = p % kEwCols;
        if (cc >= cols || 8 * g >= rows) continue;
        irow = col0 + cc;
        icol0 = row0 + 8 * g;
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = stage[8 * g + e][cc];
      }
      Bf16x4 h0, h1, l0, l1;
      split4({v[0], v[1], v[2], v[3]}, h0, l0);
      split4({v[4], v[5], v[6], v[7]}, h1, l1);
      __nv_bfloat16* dst = xl + lo_index(lo_kind, gr, ldc, irow, icol0);  // 16-byte aligned
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
    for (int w = 0; w < kEwWarps; ++w) s += warp_part[w];
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
  for (int64_t k = tid; k < md.ew_tiles; k += kEwThreads)
    acc += static_cast<double>(__ldcg(a.partial + md.ew_tile_begin + k));
  acc = warp_sum_d(acc);
  if ((tid & 31) == 0) warp_part_d[tid >> 5] = acc;
  __syncthreads();
  if (tid == 0) {
    double s = 0.0;
    for (int w = 0; w < kEwWarps; ++w) s += warp_part_d[w];
    a.scale[mi] = static_cast<float>(1.0 / (sqrt(s) + static_cast<double>(a.eps)));
    if (a.diag) a.diag[2 * md.caller] = static_cast<float>(sqrt(s));
    a.counter[mi] = 0u;
    if (a.dep) a.dep[mi] = 0u;  // the chained stage launch that follows counts from zero
  }
}

cudaError_t launch_elementwise(const EwArgs& args, cudaStream_t stream) {
  if (args.total_tiles <= 0) return cudaSuccess;
  if (args.total_tiles > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  ew_kernel<<<static_cast<unsigned>(args.total_tiles), kEwThreads, 0, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace muon
