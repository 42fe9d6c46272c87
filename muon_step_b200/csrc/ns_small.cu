// Newton-Schulz for small matrices, one CTA per matrix, all steps on chip.
//
// For matrices with min(n, m) <= 128 and max(n, m) <= 128 the grouped stage
// kernels would spend their time on padding and per-launch latency (30
// dependent launches of mostly empty 256 x 256 tiles). Here one CTA of 128
// threads (thread = iterate row = TMEM lane) runs every step of the schedule
// for one matrix and then writes the update. 256 threads: thread t owns
// iterate row t % 128 (its TMEM lane) and half t / 128 of its columns, so
// each product's epilogue is two 32-column chunks per thread:
//
//   shared memory  X, A and B as bf16 128 x 128 tiles in the 128-byte-swizzle
//                  K-major layout (two 64-column chunks of 128 rows). The
//                  same X buffer is the K-major operand of the Gram product
//                  and the MN-major operand of the Apply product.
//   registers      the fp32 iterate, half a row per thread (aX term).
//   TMEM           one 128-column fp32 accumulator reused by the three
//                  products: A = X X^T, B = b A + c A A^T, X' = a X + B X
//                  ("Ch 06 · Muon" §3 and §5 Algorithm 1, regrouped), with
//                  tcgen05.mma kind::f16, M = N = 128, K = 128 (zero padded).
//
// The elementwise kernel has already written the unscaled N (bf16 high and low parts)
// and the normalisation scale s; step one folds s^2 into A and s into X'.
// After the last step the update W <- W (1 - lr wd) - lr gamma sqrt(max(n, m))
// O' goes to the caller's matrix in its orientation ("Muon 优化器完全拆解…",
// Algorithm 1 steps four and five). Two CTAs share an SM, so one's products
// overlap the other's epilogues. Every wait is bounded.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx_sm100.cuh"
#include "stage_common.cuh"

namespace muon {

namespace {

constexpr int kS = kSmallMax;                  // 128: rows, columns, K of every product
constexpr int kChunkBytes = kS * 128;          // one 64-column chunk: 128 rows x 128 B
constexpr int kTileBytes = 2 * kChunkBytes;    // 32 KB
constexpr size_t kSmem = 1024 + 3 * kTileBytes + 64;
constexpr int kTmemCols = 128;
constexpr uint32_t kIdescKK = ptx::idesc_bf16(kS, kS, 0, 0);
constexpr uint32_t kIdescKMN = ptx::idesc_bf16(kS, kS, 0, 1);

struct alignas(16) Bf16x8 {
  __nv_bfloat162 v[4];
};

// byte offset of 16-byte piece p (8 bf16, p = 0..15 over 128 columns) of row i
__device__ __forceinline__ int piece_off(int i, int p) {
  return (p >> 3) * kChunkBytes + i * 128 + (((p & 7) ^ (i & 7)) << 4);
}

// D = A * B over K = 128: eight instructions of K = 16.
__device__ __forceinline__ void gemm128(uint32_t d, uint32_t a_base, uint32_t b_base, bool b_mn) {
#pragma unroll
  for (int k = 0; k < kS / 16; ++k) {
    const uint64_t ad = ptx::desc_sw128(a_base + (k >> 2) * kChunkBytes + (k & 3) * 32, 16, 1024);
    const uint64_t bd = b_mn ? ptx::desc_sw128(b_base + k * 16 * 128, kChunkBytes, 1024)
                             : ptx::desc_sw128(b_base + (k >> 2) * kChunkBytes + (k & 3) * 32, 16, 1024);
    ptx::umma_bf16(d, ad, bd, b_mn ? kIdescKMN : kIdescKK, k != 0);
  }
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Write 32 values of row `i` (columns 32 ch .. 32 ch + 31) as bf16.
__device__ __forceinline__ void put_row32(uint8_t* tile, int i, int ch, const float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    Bf16x8 p;
#pragma unroll
    for (int h = 0; h < 4; ++h) p.v[h] = __floats2bfloat162_rn(v[8 * q + 2 * h], v[8 * q + 2 * h + 1]);
    *reinterpret_cast<Bf16x8*>(tile + piece_off(i, 4 * ch + q)) = p;
  }
}

}  // namespace

constexpr int kThreads = 256;
constexpr int kHalfCols = kS / 2;  // columns per thread

__global__ void __launch_bounds__(kThreads, 2) ns_small_kernel(const __grid_constant__ SmallArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ float red[kThreads / 32];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Xs = base;
  uint8_t* As = Xs + kTileBytes;
  uint8_t* Bs = As + kTileBytes;
  uint64_t* bar_ld = reinterpret_cast<uint64_t*>(Bs + kTileBytes);
  uint64_t* bar_mma = bar_ld + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_mma + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int row = tid & (kS - 1);     // iterate row = TMEM lane
  const int half = tid >> 7;          // which 64 columns
  const int ch0 = half * (kHalfCols / 32);  // first 32-column chunk
  if (tid == 0) {
    ptx::mbar_init(bar_ld, 1);
    ptx::mbar_init(bar_mma, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // this warp's lanes (warps w and w + 4 share lanes 32 (w % 4) ...)
  const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
  const uint32_t sX = ptx::smem_u32(Xs), sA = ptx::smem_u32(As), sB = ptx::smem_u32(Bs);
  const uint64_t limit = a.wait_limit_ns;
  uint32_t ld_phase = 0, mma_phase = 0;
  bool ok = true;

  // every thread waits for the product; on expiry the CTA stops
  auto wait_mma = [&]() {
    if (!ptx::mbar_wait(bar_mma, mma_phase, limit, abort_flag)) {
      *abort_flag = 1;
      atomicOr(a.err, kErrTimeout);
      ok = false;
    }
    mma_phase ^= 1u;
    ptx::tc_fence_after();
  };
  // make this thread's shared-memory tile writes and TMEM reads visible to
  // the next product, then let thread 0 issue it
  auto hand_over = [&]() {
    ptx::fence_async_shared();
    ptx::tc_fence_before();
    __syncthreads();
  };

  for (int64_t idx = blockIdx.x; ok && idx < a.nsmall; idx += gridDim.x) {
    const int mat = a.small_mats[idx];
    const MatDesc& md = a.mats[mat];
    const GroupDesc& gd = a.groups[md.group];
    const int r = gd.r, c = gd.c;
    const int64_t ldc = gd.ldc;

    if (tid == 0) {
      const void* tm = static_cast<const char*>(a.tmaps) +
                       (static_cast<int64_t>(md.group) * kTmPerGroup + kTmXb0K) * 128;
      ptx::fence_tmap_acquire(tm);
      ptx::mbar_arrive_expect_tx(bar_ld, kTileBytes);
      ptx::tma_load_3d(Xs, tm, bar_ld, 0, 0, md.index);
      ptx::tma_load_3d(Xs + kChunkBytes, tm, bar_ld, 64, 0, md.index);
    }
    // this thread's half row of the iterate into fp32 registers, high + low
    // bf16 parts (zero outside the matrix)
    float x[kHalfCols];
    const int col_base = half * kHalfCols;
    const int64_t row_off = (static_cast<int64_t>(md.index) * r + row) * ldc + col_base;
    const __nv_bfloat16* xh = reinterpret_cast<const __nv_bfloat16*>(a.ws + gd.xb_off[0]) + row_off;
    const __nv_bfloat16* xl = reinterpret_cast<const __nv_bfloat16*>(a.ws + gd.xlo_off) + row_off;
    // 16-byte loads: rows start 16-byte aligned (ldc is a multiple of 8) and
    // the 8-element groups that start below c lie inside the row's ldc
#pragma unroll
    for (int q = 0; q < kHalfCols / 8; ++q) {
      uint4 hv = make_uint4(0u, 0u, 0u, 0u), lv = hv;
      if (row < r && col_base + 8 * q < c) {
        hv = *reinterpret_cast<const uint4*>(xh + 8 * q);
        lv = *reinterpret_cast<const uint4*>(xl + 8 * q);
      }
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hv);
      const __nv_bfloat162* l2 = reinterpret_cast<const __nv_bfloat162*>(&lv);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 fh = __bfloat1622float2(h2[k]);
        const float2 fl = __bfloat1622float2(l2[k]);
        const int e = 8 * q + 2 * k;
        // columns c .. ldc of the buffers are not written
        x[e] = col_base + e < c ? fh.x + fl.x : 0.f;
        x[e + 1] = col_base + e + 1 < c ? fh.y + fl.y : 0.f;
      }
    }
    if (!ptx::mbar_wait(bar_ld, ld_phase, limit, abort_flag)) {
      *abort_flag = 1;
      atomicOr(a.err, kErrTimeout);
      ok = false;
      break;
    }
    ld_phase ^= 1u;
    const float s = a.scale[mat];

    for (int k = 0; ok && k < a.steps; ++k) {
      const float alpha = (k == 0) ? s : 1.f;
      const float ca = a.abc[3 * k], cb = a.abc[3 * k + 1], cc = a.abc[3 * k + 2];

      // Gram: A = alpha^2 X X^T
      if (tid == 0) {
        ptx::tc_fence_after();
        gemm128(tmem, sX, sX, false);
        ptx::umma_commit(bar_mma);
      }
      wait_mma();
      if (!ok) break;
#pragma unroll
      for (int ch = ch0; ch < ch0 + kHalfCols / 32; ++ch) {
        float v[32];
        ptx::tmem_ld32(trow + ch * 32, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] *= alpha * alpha;
        put_row32(As, row, ch, v);
      }
      hand_over();

      // Poly: B = b A + c A A^T
      if (tid == 0) {
        ptx::tc_fence_after();
        gemm128(tmem, sA, sA, false);
        ptx::umma_commit(bar_mma);
      }
      wait_mma();
      if (!ok) break;
#pragma unroll
      for (int ch = ch0; ch < ch0 + kHalfCols / 32; ++ch) {
        float v[32];
        ptx::tmem_ld32(trow + ch * 32, v);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const Bf16x8 p = *reinterpret_cast<const Bf16x8*>(As + piece_off(row, 4 * ch + q));
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float2 f = __bfloat1622float2(p.v[h]);
            v[8 * q + 2 * h] = fmaf(cb, f.x, cc * v[8 * q + 2 * h]);
            v[8 * q + 2 * h + 1] = fmaf(cb, f.y, cc * v[8 * q + 2 * h + 1]);
          }
        }
        put_row32(Bs, row, ch, v);
      }
      hand_over();

      // Apply: X' = alpha (a X + B X)
      if (tid == 0) {
        ptx::tc_fence_after();
        gemm128(tmem, sB, sX, true);
        ptx::umma_commit(bar_mma);
      }
      const bool last = (k + 1 == a.steps);
      if (last && md.W) {
        // the caller's weight into L2 while the last product and its
        // epilogue run: the update below then waits on L2, not DRAM
        const int64_t lines = (md.n * md.m + 31) / 32;  // 128-byte lines of W
        for (int64_t ln = tid; ln < lines; ln += kThreads) prefetch_l2(md.W + ln * 32);
      }
      wait_mma();
      if (!ok) break;
#pragma unroll
      for (int j = 0; j < kHalfCols / 32; ++j) {
        float v[32];
        ptx::tmem_ld32(trow + (ch0 + j) * 32, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          x[32 * j + e] = alpha * fmaf(ca, x[32 * j + e], v[e]);
          v[e] = x[32 * j + e];
        }
        if (!last) put_row32(Xs, row, ch0 + j, v);
      }
      hand_over();
    }
    if (!ok) break;

    // The update, in the caller's orientation. O' goes to shared memory as a
    // 128 x 128 fp32 tile (the A and B tiles are free now), word (i, j) at
    // i * 128 + (j ^ (i % 32)): conflict-free for row writes and for reads
    // along either index. Each warp then updates whole caller rows, every
    // global access one contiguous segment.
    float* T = reinterpret_cast<float*>(As);
#pragma unroll
    for (int e = 0; e < kHalfCols; ++e) {
      const int col = col_base + e;
      T[row * kS + (col ^ (row & 31))] = x[e];
    }
    if (a.scale_mode == kScaleUnitRms || a.diag) {
      // RMS(O') over the matrix (zeros outside it), in a fixed order
      float ssq = 0.f;
#pragma unroll
      for (int e = 0; e < kHalfCols; ++e) ssq = fmaf(x[e], x[e], ssq);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
      if ((tid & 31) == 0) red[warp] = ssq;
    }
    __syncthreads();
    {
      // unit-RMS: O = O' gamma / RMS(O'), a plain scale once RMS is known
      float gam = a.gamma;
      int mode = a.scale_mode;
      float tot = 0.f;
      if (mode == kScaleUnitRms || a.diag)
        for (int w = 0; w < kThreads / 32; ++w) tot += red[w];
      const float rms = (mode == kScaleUnitRms || a.diag) ? sqrtf(tot / (static_cast<float>(r) * c)) : 0.f;
      if (mode == kScaleUnitRms) {
        gam = rms > 0.f ? a.gamma / rms : 0.f;
        mode = kScaleNone;
      }
      if (a.diag && tid == 0) {
        // RMS of the applied update O = step / lr * O'
        const UpdateConsts u1 = update_consts_raw(1.f, 0.f, gam, c, mode);
        a.diag[2 * md.caller + 1] = u1.step * rms;
      }
      const UpdateConsts uc = update_consts_raw(a.lr, a.wd, gam, c, mode);
      const int lane = tid & 31;
      const bool tr = md.transposed != 0;
      const int rows = tr ? c : r;  // caller rows
      const int cols = tr ? r : c;  // caller columns
      // two caller rows per pass (crow, crow + 8), every load before the
      // first store, so that their round trips overlap
      constexpr int kRowStride = kThreads / 32;
      for (int crow0 = warp; crow0 < rows; crow0 += 2 * kRowStride) {
        float w[2][kS / 32], o[2][kS / 32];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int crow = crow0 + u * kRowStride;
          const float* Wr = (md.W && crow < rows) ? md.W + static_cast<int64_t>(crow) * md.m : nullptr;
#pragma unroll
          for (int q = 0; q < kS / 32; ++q) {
            const int col = 32 * q + lane;
            const int i = tr ? col : crow;  // iterate coordinates of caller (crow, col)
            const int j = tr ? crow : col;
            o[u][q] = T[(i & (kS - 1)) * kS + ((j & (kS - 1)) ^ (i & 31))];
            w[u][q] = (col < cols && Wr) ? Wr[col] : 0.f;
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int crow = crow0 + u * kRowStride;
          if (crow >= rows) break;
          float* Wr = md.W ? md.W + static_cast<int64_t>(crow) * md.m : nullptr;
          float* Or = md.O ? md.O + static_cast<int64_t>(crow) * md.m : nullptr;
#pragma unroll
          for (int q = 0; q < kS / 32; ++q) {
            const int col = 32 * q + lane;
            if (col >= cols) continue;
            if (Or) Or[col] = o[u][q];
            if (Wr) Wr[col] = fmaf(w[u][q], uc.keep, -uc.step * o[u][q]);
          }
        }
      }
    }
    __syncthreads();  // the next matrix writes the A tile again
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

cudaError_t launch_small(const SmallArgs& args, int grid, cudaStream_t stream) {
  if (args.nsmall <= 0) return cudaSuccess;
  static_assert(kSmem <= 113 * 1024, "two CTAs per SM");
  cudaError_t e = cudaFuncSetAttribute(ns_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmem));
  if (e != cudaSuccess) return e;
  ns_small_kernel<<<grid, kThreads, kSmem, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace muon
