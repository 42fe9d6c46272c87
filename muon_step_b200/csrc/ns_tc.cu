// Newton-Schulz stages on the sm_100a tensor cores.
//
// One persistent, warp-specialised kernel per stage kind walks the output
// tiles of every matrix of the plan (all shape groups, one launch):
//
//   warp 0     TMA producer: 3-D tiled loads (128-byte swizzle) of the two
//              operands into a 4-deep shared-memory ring, one mbarrier per
//              slot counting the bytes.
//   warp 1     MMA issuer: tcgen05.mma kind::f16 (bf16 x bf16 -> fp32),
//              M = 128, N = 256, K = 16 per instruction, accumulating in
//              TMEM; tcgen05.commit frees ring slots and hands finished
//              accumulators to the epilogue. Two 256-column accumulators
//              (all 512 TMEM columns) let the epilogue of one tile overlap
//              the main loop of the next.
//   warps 2-5  epilogue: tcgen05.ld of 32 columns at a time, one tile row
//              per thread, fused arithmetic and stores.
//
// Stages ("Ch 06 · Muon" §3 and §5 Algorithm 1, regrouped as
// a X + (b A + c A^2) X with A = X X^T):
//
//   Gram   A = X X^T, symmetric: only tiles on or below the diagonal are
//          computed (128 x 128 blocks, 256-wide tiles), each block stored
//          and mirrored. Step one folds s^2 (X_0 = s N).
//   Poly   B = b A + c A A^T (A symmetric); the epilogue reads A's tile.
//          Lower tiles only, mirrored, like Gram.
//   Apply  X' = a X + B X: B is the K-major left operand, the iterate X the
//          MN-major right operand (row-major X read as K x N). The epilogue
//          reads the fp32 iterate, writes the fp32 iterate and its bf16
//          operand copy; on the last step it writes the update
//          W <- W (1 - lr wd) - lr gamma sqrt(max(n, m)) X in the caller's
//          orientation (and O' when requested).
//
// Every spin-wait is bounded; on expiry the kernel sets the error word,
// stops issuing work, waits (bounded) for copies and MMAs already in
// flight, frees TMEM and returns.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx_sm100.cuh"
#include "stage_common.cuh"

namespace muon {

namespace {

constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;             // 16 KB
constexpr int kBBytes = kBN * kBK * 2;             // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;     // 48 KB
constexpr int kTmemCols = 512;                     // two 256-column accumulators
constexpr int kTmapBytes = 128;
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr size_t kBarrierBytes = 256;
constexpr size_t kSmemBytes = 1024 + kStages * kStageBytes + kBarrierBytes;

constexpr uint32_t kIdescKK = ptx::idesc_bf16(kBM, kBN, 0, 0);   // both K-major
constexpr uint32_t kIdescKMN = ptx::idesc_bf16(kBM, kBN, 0, 1);  // B MN-major

struct TileCoord {
  int g;
  int64_t b;    // matrix within the group
  int i;        // 128-row block
  int j;        // 256-column tile
  int kblocks;  // K / 64, rounded up
};

// Lower-triangle tile enumeration for the symmetric stages: row block i
// (128 rows) has tiles j = 0 .. floor(i / 2) (256 columns each). Row pair p
// (rows 2p, 2p + 1) holds 2 (p + 1) tiles; the first p pairs hold p (p + 1).
__device__ __forceinline__ void syrk_tile(int64_t u, int& i, int& j) {
  int64_t p = static_cast<int64_t>((sqrt(4.0 * static_cast<double>(u) + 1.0) - 1.0) * 0.5);
  while (p * (p + 1) > u) --p;
  while ((p + 1) * (p + 2) <= u) ++p;
  const int64_t off = u - p * (p + 1);
  if (off <= p) {
    i = static_cast<int>(2 * p);
    j = static_cast<int>(off);
  } else {
    i = static_cast<int>(2 * p + 1);
    j = static_cast<int>(off - (p + 1));
  }
}

template <int KIND>
__device__ __forceinline__ TileCoord decode_tile(const StageArgs& a, int64_t t) {
  TileCoord tc;
  tc.g = stage_group<KIND>(a, t);
  const GroupDesc& gd = a.groups[tc.g];
  const int64_t local = t - gd.tile_base[KIND];
  const int64_t per = gd.tiles_per_mat[KIND];
  tc.b = local / per;
  const int64_t u = local % per;
  if (KIND == kApply) {
    const int64_t rb = (gd.r + kBM - 1) / kBM;
    tc.i = static_cast<int>(u % rb);
    tc.j = static_cast<int>(u / rb);
    tc.kblocks = (gd.r + kBK - 1) / kBK;
  } else {
    syrk_tile(u, tc.i, tc.j);
    tc.kblocks = ((KIND == kGram ? gd.c : gd.r) + kBK - 1) / kBK;
  }
  return tc;
}

__device__ __forceinline__ const void* tmap(const StageArgs& a, int g, int slot) {
  return static_cast<const char*>(a.tmaps) + (static_cast<int64_t>(g) * kTmPerGroup + slot) * kTmapBytes;
}

__device__ __forceinline__ void raise_abort(const StageArgs& a, volatile int* abort_flag) {
  *abort_flag = 1;
  atomicOr(a.err, kErrTimeout);
}

struct alignas(16) Bf16x8 {
  __nv_bfloat162 v[4];
};

// -------------------------------------------------------------- epilogues

// Gram / Poly: 32 columns of one row of a lower (or diagonal) 128 x 128 block.
template <int KIND>
__device__ __forceinline__ void epi_symmetric(const StageArgs& a, const GroupDesc& gd,
                                              const TileCoord& tc, int trow, int ch,
                                              const float (&v)[32]) {
  const int bj = 2 * tc.j + (ch >> 2);
  if (bj > tc.i) return;  // block above the diagonal: its mirror is stored elsewhere
  const int64_t r = gd.r, ldr = gd.ldr;
  const int64_t row = static_cast<int64_t>(tc.i) * kBM + trow;
  const int64_t col0 = static_cast<int64_t>(tc.j) * kBN + ch * 32;
  if (row >= r || col0 >= r) return;
  const int ncol = static_cast<int>(r - col0 < 32 ? r - col0 : 32);
  const int64_t moff = tc.b * r * ldr;
  __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.ws + (KIND == kGram ? gd.a_off : gd.b_off)) + moff;

  float out[32];
  if (KIND == kGram) {
    float s2 = 1.f;
    if (a.first) {
      const float s = a.scale[gd.first_mat + tc.b];
      s2 = s * s;
    }
#pragma unroll
    for (int e = 0; e < 32; ++e) out[e] = s2 * v[e];
  } else {
    const __nv_bfloat16* Asrc = reinterpret_cast<const __nv_bfloat16*>(a.ws + gd.a_off) + moff + row * ldr + col0;
    if (ncol == 32) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const Bf16x8 p = *reinterpret_cast<const Bf16x8*>(Asrc + 8 * q);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float2 f = __bfloat1622float2(p.v[h]);
          out[8 * q + 2 * h] = fmaf(a.b, f.x, a.c * v[8 * q + 2 * h]);
          out[8 * q + 2 * h + 1] = fmaf(a.b, f.y, a.c * v[8 * q + 2 * h + 1]);
        }
      }
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        out[e] = (e < ncol) ? fmaf(a.b, __bfloat162float(Asrc[e]), a.c * v[e]) : 0.f;
    }
  }

  __nv_bfloat16* drow = dst + row * ldr + col0;
  if (ncol == 32) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      Bf16x8 p;
#pragma unroll
      for (int h = 0; h < 4; ++h) p.v[h] = __floats2bfloat162_rn(out[8 * q + 2 * h], out[8 * q + 2 * h + 1]);
      *reinterpret_cast<Bf16x8*>(drow + 8 * q) = p;
    }
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (e < ncol) drow[e] = __float2bfloat16_rn(out[e]);
  }
  if (bj < tc.i) {
    // mirror: lanes hold consecutive rows, so each store is 64 contiguous bytes
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (e < ncol) dst[(col0 + e) * ldr + row] = __float2bfloat16_rn(out[e]);
  }
}

// Apply: X' = alpha (a X + acc) for 32 columns of one row.
__device__ __forceinline__ void epi_apply(const StageArgs& a, const GroupDesc& gd,
                                          const TileCoord& tc, int trow, int ch,
                                          const float (&v)[32]) {
  const int64_t r = gd.r, c = gd.c, ldc = gd.ldc;
  const int64_t row = static_cast<int64_t>(tc.i) * kBM + trow;
  const int64_t col0 = static_cast<int64_t>(tc.j) * kBN + ch * 32;
  if (row >= r || col0 >= c) return;
  const int ncol = static_cast<int>(c - col0 < 32 ? c - col0 : 32);
  const int mat = gd.first_mat + static_cast<int>(tc.b);
  const float alpha = a.first ? a.scale[mat] : 1.f;
  float* xf = reinterpret_cast<float*>(a.ws + gd.xf_off[0]) + tc.b * r * ldc + row * ldc + col0;

  float x[32];
  if (ncol == 32) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 p = *reinterpret_cast<const float4*>(xf + 4 * q);
      x[4 * q + 0] = alpha * fmaf(a.a, p.x, v[4 * q + 0]);
      x[4 * q + 1] = alpha * fmaf(a.a, p.y, v[4 * q + 1]);
      x[4 * q + 2] = alpha * fmaf(a.a, p.z, v[4 * q + 2]);
      x[4 * q + 3] = alpha * fmaf(a.a, p.w, v[4 * q + 3]);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e) x[e] = (e < ncol) ? alpha * fmaf(a.a, xf[e], v[e]) : 0.f;
  }

  if (!a.last) {
    __nv_bfloat16* xb = reinterpret_cast<__nv_bfloat16*>(a.ws + gd.xb_off[a.xsrc ^ 1]) + tc.b * r * ldc + row * ldc + col0;
    if (ncol == 32) {
#pragma unroll
      for (int q = 0; q < 8; ++q)
        *reinterpret_cast<float4*>(xf + 4 * q) = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        Bf16x8 p;
#pragma unroll
        for (int h = 0; h < 4; ++h) p.v[h] = __floats2bfloat162_rn(x[8 * q + 2 * h], x[8 * q + 2 * h + 1]);
        *reinterpret_cast<Bf16x8*>(xb + 8 * q) = p;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (e < ncol) {
          xf[e] = x[e];
          xb[e] = __float2bfloat16_rn(x[e]);
        }
    }
    return;
  }

  // last step: the update, in the caller's orientation
  const MatDesc& md = a.mats[mat];
  const UpdateConsts uc = update_consts(a, static_cast<int>(c));
  if (!md.transposed && ncol == 32 && (md.m & 3) == 0 &&
      ((reinterpret_cast<uintptr_t>(md.W) | reinterpret_cast<uintptr_t>(md.O)) & 15) == 0) {
    const int64_t base = row * md.m + col0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 o4 = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
      if (md.O) *reinterpret_cast<float4*>(md.O + base + 4 * q) = o4;
      if (md.W) {
        float4 w = *reinterpret_cast<const float4*>(md.W + base + 4 * q);
        w.x = fmaf(w.x, uc.keep, -uc.step * o4.x);
        w.y = fmaf(w.y, uc.keep, -uc.step * o4.y);
        w.z = fmaf(w.z, uc.keep, -uc.step * o4.z);
        w.w = fmaf(w.w, uc.keep, -uc.step * o4.w);
        *reinterpret_cast<float4*>(md.W + base + 4 * q) = w;
      }
    }
  } else {
    // transposed: for each column, the warp's lanes write consecutive addresses
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (e < ncol) write_update(md, uc, row, col0 + e, x[e]);
  }
}

// -------------------------------------------------------------- kernel

template <int KIND>
__global__ void __launch_bounds__(kThreads, 1) stage_tc_kernel(const __grid_constant__ StageArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&tfull[s], 1);
      ptx::mbar_init(&tempty[s], kEpiThreads);
    }
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t limit = a.wait_limit_ns;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- producer
    for (int g = 0; g < a.ngroups; ++g)
      for (int s = 0; s < kTmPerGroup; ++s) {
        ptx::fence_tmap_acquire(tmap(a, g, s));
        ptx::prefetch_tmap(tmap(a, g, s));
      }
    uint32_t stage = 0, phase = 0;
    uint32_t armed = 0, armed_phase = 0;  // bit s: slot s armed; its last armed parity
    bool ok = true;
    for (int64_t t = blockIdx.x; ok && t < a.total_tiles; t += gridDim.x) {
      const TileCoord tc = decode_tile<KIND>(a, t);
      const int bz = static_cast<int>(tc.b);
      for (int kb = 0; kb < tc.kblocks; ++kb) {
        if (!ptx::mbar_wait(&empty[stage], phase ^ 1, limit, abort_flag)) {
          raise_abort(a, abort_flag);
          ok = false;
          break;
        }
        uint8_t* sa = smem + stage * kStageBytes;
        uint8_t* sb = sa + kABytes;
        ptx::mbar_arrive_expect_tx(&full[stage], kStageBytes);
        armed |= 1u << stage;
        armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
        const int k0 = kb * kBK;
        if (KIND == kApply) {
          ptx::tma_load_3d(sa, tmap(a, tc.g, kTmB), &full[stage], k0, tc.i * kBM, bz);
          const void* tx = tmap(a, tc.g, a.xsrc ? kTmXb1MN : kTmXb0MN);
#pragma unroll
          for (int q = 0; q < kBN / 64; ++q)
            ptx::tma_load_3d(sb + q * (64 * kBK * 2), tx, &full[stage], tc.j * kBN + q * 64, k0, bz);
        } else {
          const void* tm = (KIND == kGram) ? tmap(a, tc.g, a.xsrc ? kTmXb1K : kTmXb0K)
                                           : tmap(a, tc.g, kTmA);
          ptx::tma_load_3d(sa, tm, &full[stage], k0, tc.i * kBM, bz);
          ptx::tma_load_3d(sb, tm, &full[stage], k0, tc.j * kBN, bz);
          ptx::tma_load_3d(sb + kABytes, tm, &full[stage], k0, tc.j * kBN + kBM, bz);
        }
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (!ok) {
      // let the copies already issued land before the CTA exits
      volatile int never = 0;
      for (int s = 0; s < kStages; ++s)
        if (armed & (1u << s)) ptx::mbar_wait(&full[s], (armed_phase >> s) & 1u, limit, &never);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    const uint32_t idesc = (KIND == kApply) ? kIdescKMN : kIdescKK;
    uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
    bool ok = true;
    bool issued = false;
    for (int64_t t = blockIdx.x; ok && t < a.total_tiles; t += gridDim.x) {
      const TileCoord tc = decode_tile<KIND>(a, t);
      if (!ptx::mbar_wait(&tempty[acc], acc_phase ^ 1, limit, abort_flag)) {
        raise_abort(a, abort_flag);
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t d = tmem_base + acc * kBN;
      for (int kb = 0; kb < tc.kblocks; ++kb) {
        if (!ptx::mbar_wait(&full[stage], phase, limit, abort_flag)) {
          raise_abort(a, abort_flag);
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t sa = ptx::smem_u32(smem + stage * kStageBytes);
        const uint32_t sb = sa + kABytes;
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k) {
          const uint64_t ad = ptx::desc_sw128(sa + k * 32, 16, 1024);
          const uint64_t bd = (KIND == kApply) ? ptx::desc_sw128(sb + k * 16 * 128, 64 * kBK * 2, 1024)
                                               : ptx::desc_sw128(sb + k * 32, 16, 1024);
          ptx::umma_bf16(d, ad, bd, idesc, (kb | k) != 0);
        }
        issued = true;
        ptx::umma_commit(&empty[stage]);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      ptx::umma_commit(&tfull[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if (!ok && issued) {
      // wait for the MMAs in flight before TMEM is released
      volatile int never = 0;
      ptx::umma_commit(drain);
      ptx::mbar_wait(drain, 0, limit, &never);
    }
  } else if (warp >= 2) {
    // ---------------------------------------------------------- epilogue
    const int lane_base = (warp & 3) * 32;  // TMEM lanes this warp may read
    const int trow = lane_base + lane;
    uint32_t acc = 0, acc_phase = 0;
    for (int64_t t = blockIdx.x; t < a.total_tiles; t += gridDim.x) {
      const TileCoord tc = decode_tile<KIND>(a, t);
      if (!ptx::mbar_wait(&tfull[acc], acc_phase, limit, abort_flag)) {
        raise_abort(a, abort_flag);
        break;
      }
      ptx::tc_fence_after();
      const GroupDesc& gd = a.groups[tc.g];
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(lane_base) << 16) + acc * kBN;
#pragma unroll 1
      for (int ch = 0; ch < kBN / 32; ++ch) {
        float v[32];
        __syncwarp();
        ptx::tmem_ld32(taddr + ch * 32, v);
        if (KIND == kApply) epi_apply(a, gd, tc, trow, ch, v);
        else epi_symmetric<KIND>(a, gd, tc, trow, ch, v);
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

size_t stage_tc_smem_bytes() { return kSmemBytes; }

cudaError_t launch_stage_tc(StageKind kind, const StageArgs& args, int grid, cudaStream_t stream) {
  if (args.total_tiles <= 0) return cudaSuccess;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  cudaError_t e = cudaSuccess;
  switch (kind) {
    case kGram:
      e = cudaFuncSetAttribute(stage_tc_kernel<kGram>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
      if (e == cudaSuccess) stage_tc_kernel<kGram><<<grid, kThreads, kSmemBytes, stream>>>(args);
      break;
    case kPoly:
      e = cudaFuncSetAttribute(stage_tc_kernel<kPoly>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
      if (e == cudaSuccess) stage_tc_kernel<kPoly><<<grid, kThreads, kSmemBytes, stream>>>(args);
      break;
    case kApply:
      e = cudaFuncSetAttribute(stage_tc_kernel<kApply>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
      if (e == cudaSuccess) stage_tc_kernel<kApply><<<grid, kThreads, kSmemBytes, stream>>>(args);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace muon
