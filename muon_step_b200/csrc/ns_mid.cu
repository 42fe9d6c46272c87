// Newton-Schulz for matrices with min(n, m) <= 128 < max(n, m) <= 512, one
// CTA per matrix, every step on chip.
//
// Such matrices (128 x 512 attention or expert slices, for instance) waste
// half or more of every 256 x 256 CTA-pair tile of the grouped kernels, and
// their three stage launches per step are short. Here one CTA of 512 threads
// runs the whole schedule for one matrix (r = min(n, m) rows, c = max(n, m)
// columns, rows <= 128, "Ch 06 · Muon" §3 and §5 Algorithm 1, regrouped as
// X' = a X + (b A + c A^2) X with A = X X^T):
//
//   shared memory  the iterate's bf16 high part X (128 x c, up to 128 KB) in
//                  the 128-byte-swizzle K-major layout: the K-major operand
//                  of the Gram product and, read as 64-column chunks, the
//                  MN-major operand of the Apply product; A and B as 128 x 128
//                  bf16 tiles (64 KB).
//   TMEM           columns 0 .. 255: the 128 x 128 accumulators of the Gram
//                  and Poly products and, one column half at a time, the
//                  128 x 256 accumulator of the Apply product (one N = 256
//                  instruction per K = 16); columns 256 .. 511: the iterate's
//                  bf16 low part (iterate = high + low), two elements a
//                  column, loaded from global memory once per matrix and
//                  rewritten in place by each Apply epilogue.
//
// Thread t owns iterate row t % 128 (its TMEM lane) and column quarter t / 128:
// 32 columns of A and B; in each Apply half, 64 columns of X. The elementwise kernel has written
// N as high + low parts and the scale s; step one folds s^2 into A and s into
// X'. After the last step the update W <- W (1 - lr wd) - lr gamma
// sqrt(max(n, m)) O' ("Muon 优化器完全拆解…", Algorithm 1 steps four and five, or
// the unit-RMS / no-rescale rules) goes to the caller's matrix in 128-column
// blocks of the iterate staged as fp32 in shared memory, so every global
// access is a contiguous row segment. Every wait is bounded.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx_sm100.cuh"
#include "stage_common.cuh"

namespace muon {

namespace {

constexpr int kR = kSmallMax;                       // 128 rows (TMEM lanes)
constexpr int kMaxC = kMidMaxC;                     // 512 columns
constexpr int kChunkBytes = kR * 128;               // 64 columns x 128 rows of bf16
constexpr int kXBytes = (kMaxC / 64) * kChunkBytes; // 128 KB
constexpr int kTileBytes = 2 * kChunkBytes;         // 128 x 128 bf16
constexpr int kThreads = 512;
constexpr size_t kSmem = 1024 + kXBytes + 2 * kTileBytes + 64;
constexpr int kTmemCols = 512;
constexpr int kLoCol = 256;  // TMEM columns 256 .. 511: the iterate's low part, two bf16 a column
constexpr uint32_t kIdescKK = ptx::idesc_bf16(kR, kR, 0, 0);   // M = N = 128, both K-major
constexpr uint32_t kIdescApply = ptx::idesc_bf16(kR, 256, 0, 1);  // M = 128, N = 256, B MN-major

struct alignas(16) Bf16x8 {
  __nv_bfloat162 v[4];
};

// byte offset of 16-byte piece p (8 bf16; p = column / 8) of row i
__device__ __forceinline__ int piece_off(int i, int p) {
  return (p >> 3) * kChunkBytes + i * 128 + (((p & 7) ^ (i & 7)) << 4);
}

// A = X X^T over K = 64 nch (zero columns past c).
__device__ __forceinline__ void gemm_gram(uint32_t d, uint32_t sx, int nch) {
  for (int kc = 0; kc < nch; ++kc) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint64_t desc = ptx::desc_sw128(sx + kc * kChunkBytes + k * 32, 16, 1024);
      ptx::umma_bf16(d, desc, desc, kIdescKK, (kc | k) != 0);
    }
  }
}

// D = A A^T (A symmetric) over K = 128.
__device__ __forceinline__ void gemm_poly(uint32_t d, uint32_t sa) {
#pragma unroll
  for (int k = 0; k < kR / 16; ++k) {
    const uint64_t desc = ptx::desc_sw128(sa + (k >> 2) * kChunkBytes + (k & 3) * 32, 16, 1024);
    ptx::umma_bf16(d, desc, desc, kIdescKK, k != 0);
  }
}

// D[:, 0 .. 256) = B X[:, 256 h ..] over K = 128: column half h of the Apply
// product (one N = 256 instruction per K = 16).
__device__ __forceinline__ void gemm_apply_half(uint32_t d, uint32_t sb, uint32_t sx, int h) {
#pragma unroll
  for (int k = 0; k < kR / 16; ++k) {
    const uint64_t ad = ptx::desc_sw128(sb + (k >> 2) * kChunkBytes + (k & 3) * 32, 16, 1024);
    const uint64_t bd = ptx::desc_sw128(sx + h * 4 * kChunkBytes + k * 16 * 128, kChunkBytes, 1024);
    ptx::umma_bf16(d, ad, bd, kIdescApply, k != 0);
  }
}

// tcgen05.ld / tcgen05.st of 16 consecutive 32-bit TMEM columns of this
// warp's 32 lanes (one row per thread).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ __nv_bfloat162 as_bf2(uint32_t u) {
  __nv_bfloat162 b;
  memcpy(&b, &u, 4);
  return b;
}

__device__ __forceinline__ uint32_t as_u32(__nv_bfloat162 b) {
  uint32_t u;
  memcpy(&u, &b, 4);
  return u;
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Write 32 values of row i, columns 32 ch .., as bf16 into a swizzled tile.
__device__ __forceinline__ void put_row32(uint8_t* tile, int i, int ch, const float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    Bf16x8 p;
#pragma unroll
    for (int h = 0; h < 4; ++h) p.v[h] = __floats2bfloat162_rn(v[8 * q + 2 * h], v[8 * q + 2 * h + 1]);
    *reinterpret_cast<Bf16x8*>(tile + piece_off(i, 4 * ch + q)) = p;
  }
}

// One 32-column chunk of the Apply epilogue for iterate row `row`:
// X' = alpha (a X + v) with X = high (shared) + low (`lw`: word i holds
// columns col0 + 2 i and col0 + 2 i + 1), written back as high and low parts.
// kFirst folds alpha (step one), kLast accumulates the sum of squares, kMask
// zeroes what lies outside the matrix (ragged chunks).
template <bool kFirst, bool kLast, bool kMask>
__device__ __forceinline__ void apply_chunk(uint8_t* Xs, int row, int col0, int c, bool row_in, float alpha,
                                            float ca, const float (&v)[32], uint32_t (&lw)[16], float& ssq) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int p = col0 / 8 + q;
    Bf16x8 h8 = *reinterpret_cast<const Bf16x8*>(Xs + piece_off(row, p));
#pragma unroll
    for (int hh = 0; hh < 4; ++hh) {
      const int e = 8 * q + 2 * hh;
      const float2 fh = __bfloat1622float2(h8.v[hh]);
      const float2 fl = __bfloat1622float2(as_bf2(lw[4 * q + hh]));
      float x0 = fh.x + fl.x, x1 = fh.y + fl.y;
      if (kMask) {
        // columns c .. ldc of the low part are not written by the elementwise kernel
        x0 = (row_in && col0 + e < c) ? x0 : 0.f;
        x1 = (row_in && col0 + e + 1 < c) ? x1 : 0.f;
      }
      float y0 = fmaf(ca, x0, v[e]), y1 = fmaf(ca, x1, v[e + 1]);
      if (kFirst) {
        y0 *= alpha;
        y1 *= alpha;
      }
      if (kLast) ssq = fmaf(y0, y0, fmaf(y1, y1, ssq));
      h8.v[hh] = __floats2bfloat162_rn(y0, y1);
      const float2 nh2 = __bfloat1622float2(h8.v[hh]);
      lw[4 * q + hh] = as_u32(__floats2bfloat162_rn(y0 - nh2.x, y1 - nh2.y));
    }
    *reinterpret_cast<Bf16x8*>(Xs + piece_off(row, p)) = h8;
  }
}

// The epilogue of column half h: thread quarter cq takes iterate columns
// 256 h + 64 cq .. + 63 (two chunks); the accumulator holds the half at TMEM
// columns 0 .. 255, the low part sits at column kLoCol + col / 2.
template <bool kFirst, bool kLast>
__device__ __forceinline__ void apply_epilogue(uint8_t* Xs, uint32_t trow, int row, int cq, int h, int c,
                                               bool row_in, float alpha, float ca, float& ssq) {
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int acc = 64 * cq + 32 * j;  // accumulator column
    const int col0 = 256 * h + acc;    // iterate column
    if (col0 >= c) break;              // the same for the whole warp
    float v[32];
    uint32_t lw[16];
    ptx::tmem_ld32(trow + acc, v);
    tmem_ld16(trow + kLoCol + (col0 >> 1), lw);
    if (row_in && col0 + 32 <= c)
      apply_chunk<kFirst, kLast, false>(Xs, row, col0, c, row_in, alpha, ca, v, lw, ssq);
    else
      apply_chunk<kFirst, kLast, true>(Xs, row, col0, c, row_in, alpha, ca, v, lw, ssq);
    tmem_st16(trow + kLoCol + (col0 >> 1), lw);
  }
  tmem_wait_st();
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) ns_mid_kernel(const __grid_constant__ SmallArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ float red[kThreads / 32];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Xs = base;
  uint8_t* As = Xs + kXBytes;
  uint8_t* Bs = As + kTileBytes;
  uint64_t* bar_ld = reinterpret_cast<uint64_t*>(Bs + kTileBytes);
  uint64_t* bar_mma = bar_ld + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_mma + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int row = tid & (kR - 1);  // iterate row = TMEM lane
  const int cq = tid >> 7;         // column quarter: 32 columns of A / B, 128 of X
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
  // warps w, w + 4, w + 8, w + 12 share lanes 32 (w % 4) ...
  const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
  const uint32_t sX = ptx::smem_u32(Xs), sA = ptx::smem_u32(As), sB = ptx::smem_u32(Bs);
  const uint64_t limit = a.wait_limit_ns;
  uint32_t ld_phase = 0, mma_phase = 0;
  bool ok = true;

  auto wait_mma = [&]() {
    if (!ptx::mbar_wait(bar_mma, mma_phase, limit, abort_flag)) {
      *abort_flag = 1;
      atomicOr(a.err, kErrTimeout);
      ok = false;
    }
    mma_phase ^= 1u;
    ptx::tc_fence_after();
  };
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
    const int nch = (c + 63) / 64;    // 64-column chunks of X
    const int nh = (c + 255) / 256;   // N = 256 halves of the Apply product

    if (tid == 0) {
      const void* tm = static_cast<const char*>(a.tmaps) +
                       (static_cast<int64_t>(md.group) * kTmPerGroup + kTmXb0K) * 128;
      ptx::fence_tmap_acquire(tm);
      ptx::mbar_arrive_expect_tx(bar_ld, static_cast<uint32_t>(nch * kChunkBytes));
      for (int q = 0; q < nch; ++q) ptx::tma_load_3d(Xs + q * kChunkBytes, tm, bar_ld, 64 * q, 0, md.index);
    }
    // the iterate's low part, in 8-column groups (lo_index): the 16-byte piece
    // of this thread's row for columns 8 g .. 8 g + 7 is at xl + 8 g r
    __nv_bfloat16* xl = reinterpret_cast<__nv_bfloat16*>(a.ws + gd.xlo_off) +
                        static_cast<int64_t>(md.index) * r * ldc + static_cast<int64_t>(row) * 8;
    const bool row_in = row < r;
    // the low part into TMEM columns kLoCol + col / 2: this thread's row,
    // columns 128 cq .. 128 cq + 127 (8-column groups past the matrix: zero)
    ptx::tc_fence_after();
#pragma unroll 1
    for (int g = 0; g < 4; ++g) {
      const int col0 = 128 * cq + 32 * g;
      uint32_t lw[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 lraw = make_uint4(0u, 0u, 0u, 0u);
        if (row_in && col0 + 8 * q < c)
          lraw = *reinterpret_cast<const uint4*>(xl + static_cast<int64_t>((col0 >> 3) + q) * r * 8);
        lw[4 * q] = lraw.x;
        lw[4 * q + 1] = lraw.y;
        lw[4 * q + 2] = lraw.z;
        lw[4 * q + 3] = lraw.w;
      }
      tmem_st16(trow + kLoCol + (col0 >> 1), lw);
    }
    tmem_wait_st();
    if (!ptx::mbar_wait(bar_ld, ld_phase, limit, abort_flag)) {
      *abort_flag = 1;
      atomicOr(a.err, kErrTimeout);
      ok = false;
      break;
    }
    ld_phase ^= 1u;
    const float s = a.scale[mat];
    float ssq = 0.f;

    for (int k = 0; ok && k < a.steps; ++k) {
      const float alpha = (k == 0) ? s : 1.f;
      const float ca = a.abc[3 * k], cb = a.abc[3 * k + 1], cc = a.abc[3 * k + 2];

      // Gram: A = alpha^2 X X^T
      if (tid == 0) {
        ptx::tc_fence_after();
        gemm_gram(tmem, sX, nch);
        ptx::umma_commit(bar_mma);
      }
      wait_mma();
      if (!ok) break;
      {
        float v[32];
        ptx::tmem_ld32(trow + cq * 32, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] *= alpha * alpha;
        put_row32(As, row, cq, v);
      }
      hand_over();

      // Poly: B = b A + c A A^T
      if (tid == 0) {
        ptx::tc_fence_after();
        gemm_poly(tmem, sA);
        ptx::umma_commit(bar_mma);
      }
      wait_mma();
      if (!ok) break;
      {
        float v[32];
        ptx::tmem_ld32(trow + cq * 32, v);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const Bf16x8 p = *reinterpret_cast<const Bf16x8*>(As + piece_off(row, 4 * cq + q));
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float2 f = __bfloat1622float2(p.v[h]);
            v[8 * q + 2 * h] = fmaf(cb, f.x, cc * v[8 * q + 2 * h]);
            v[8 * q + 2 * h + 1] = fmaf(cb, f.y, cc * v[8 * q + 2 * h + 1]);
          }
        }
        put_row32(Bs, row, cq, v);
      }
      hand_over();

      // Apply: X' = alpha (a X + B X), X = high (shared) + low (TMEM), one
      // column half at a time: the product of half 1 reads X columns 256 ..
      // only, which the epilogue of half 0 leaves alone
      const bool last = (k + 1 == a.steps);
      if (last && md.W) {
        // the caller's weight into L2 for the update while the products run
        const int64_t lines = (md.n * md.m + 31) / 32;  // 128-byte lines of W
        for (int64_t ln = tid; ln < lines; ln += kThreads) prefetch_l2(md.W + ln * 32);
      }
      for (int h = 0; ok && h < nh; ++h) {
        if (tid == 0) {
          ptx::tc_fence_after();
          gemm_apply_half(tmem, sB, sX, h);
          ptx::umma_commit(bar_mma);
        }
        wait_mma();
        if (!ok) break;
        // variants without the step-one scale, sums or masks where they are not needed
        if (k == 0) {
          if (last) apply_epilogue<true, true>(Xs, trow, row, cq, h, c, row_in, alpha, ca, ssq);
          else apply_epilogue<true, false>(Xs, trow, row, cq, h, c, row_in, alpha, ca, ssq);
        } else {
          if (last) apply_epilogue<false, true>(Xs, trow, row, cq, h, c, row_in, alpha, ca, ssq);
          else apply_epilogue<false, false>(Xs, trow, row, cq, h, c, row_in, alpha, ca, ssq);
        }
        hand_over();
      }
    }
    if (!ok) break;

    // RMS of O' (unit-RMS scale, diagnostics), in a fixed order
    const bool need_rms = a.scale_mode == kScaleUnitRms || a.diag;
    if (need_rms) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
      if (lane == 0) red[warp] = ssq;
    }
    __syncthreads();
    float gam = a.gamma;
    int mode = a.scale_mode;
    float rms = 0.f;
    if (need_rms) {
      float tot = 0.f;
      for (int w = 0; w < kThreads / 32; ++w) tot += red[w];
      rms = sqrtf(tot / (static_cast<float>(r) * c));
    }
    if (mode == kScaleUnitRms) {
      gam = rms > 0.f ? a.gamma / rms : 0.f;
      mode = kScaleNone;
    }
    if (a.diag && tid == 0) {
      const UpdateConsts u1 = update_consts_raw(1.f, 0.f, gam, c, mode);
      a.diag[2 * md.caller + 1] = u1.step * rms;
    }
    const UpdateConsts uc = update_consts_raw(a.lr, a.wd, gam, c, mode);

    // The update, 128 iterate columns at a time: O' (high + low) staged as a
    // 128 x 128 fp32 tile in the A / B area, word (i, j) at i * 128 + (j ^ (i % 32)),
    // then each warp updates whole caller rows with contiguous accesses.
    float* T = reinterpret_cast<float*>(As);
    ptx::tc_fence_after();  // the low part was last written by other warps
    const bool tr = md.transposed != 0;
    for (int p0 = 0; p0 < c; p0 += 128) {
      const int bw = (c - p0) < 128 ? (c - p0) : 128;  // block width
      const int col0 = p0 + 32 * cq;
      if (col0 < c) {  // the same for the whole warp
        uint32_t lw[16];
        tmem_ld16(trow + kLoCol + (col0 >> 1), lw);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const Bf16x8 h8 = *reinterpret_cast<const Bf16x8*>(Xs + piece_off(row, col0 / 8 + q));
#pragma unroll
          for (int hh = 0; hh < 4; ++hh) {
            const int e = 8 * q + 2 * hh;
            const float2 fh = __bfloat1622float2(h8.v[hh]);
            const float2 fl = __bfloat1622float2(as_bf2(lw[4 * q + hh]));
            const int jj = 32 * cq + e;  // column within the block
            T[row * 128 + (jj ^ (row & 31))] = (row_in && col0 + e < c) ? fh.x + fl.x : 0.f;
            T[row * 128 + ((jj + 1) ^ (row & 31))] = (row_in && col0 + e + 1 < c) ? fh.y + fl.y : 0.f;
          }
        }
      }
      __syncthreads();
      if (!tr) {
        // caller rows = iterate rows (r), caller columns p0 .. p0 + bw
        // two caller rows per warp pass: all loads before the stores
        for (int cb = 2 * warp; cb < r; cb += 2 * (kThreads / 32)) {
          float w[2][4];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int crow = cb + u;
            float* Wr = (md.W && crow < r) ? md.W + static_cast<int64_t>(crow) * md.m + p0 : nullptr;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int lc = 32 * q + lane;
              w[u][q] = (lc < bw && Wr) ? Wr[lc] : 0.f;
            }
          }
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int crow = cb + u;
            if (crow >= r) break;
            float* Wr = md.W ? md.W + static_cast<int64_t>(crow) * md.m + p0 : nullptr;
            float* Or = md.O ? md.O + static_cast<int64_t>(crow) * md.m + p0 : nullptr;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int lc = 32 * q + lane;
              if (lc >= bw) continue;
              const float o = T[crow * 128 + (lc ^ (crow & 31))];
              if (Or) Or[lc] = o;
              if (Wr) Wr[lc] = fmaf(w[u][q], uc.keep, -uc.step * o);
            }
          }
        }
      } else {
        // caller rows p0 .. p0 + bw = iterate columns, caller columns = iterate rows (r)
        for (int cb = 2 * warp; cb < bw; cb += 2 * (kThreads / 32)) {
          float w[2][4];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int cr = cb + u;
            float* Wr = (md.W && cr < bw) ? md.W + (p0 + cr) * md.m : nullptr;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int col = 32 * q + lane;  // iterate row
              w[u][q] = (col < r && Wr) ? Wr[col] : 0.f;
            }
          }
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int cr = cb + u;
            if (cr >= bw) break;
            float* Wr = md.W ? md.W + (p0 + cr) * md.m : nullptr;
            float* Or = md.O ? md.O + (p0 + cr) * md.m : nullptr;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int col = 32 * q + lane;
              if (col >= r) continue;
              const float o = T[col * 128 + (cr ^ (col & 31))];
              if (Or) Or[col] = o;
              if (Wr) Wr[col] = fmaf(w[u][q], uc.keep, -uc.step * o);
            }
          }
        }
      }
      __syncthreads();  // the next block rewrites the staging tile
    }
    // the next matrix loads X by TMA over what this one read, and its low
    // part into TMEM over what this one's update read
    ptx::fence_async_shared();
    ptx::tc_fence_before();
    __syncthreads();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

cudaError_t launch_mid(const SmallArgs& args, int grid, cudaStream_t stream) {
  if (args.nsmall <= 0) return cudaSuccess;
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(ns_mid_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmem));
  if (e != cudaSuccess) return e;
  ns_mid_kernel<<<grid, kThreads, kSmem, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace muon
