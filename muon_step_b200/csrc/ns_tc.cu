// Newton-Schulz stages on the sm_100a tensor cores, one CTA pair per tile.
//
// One persistent, warp-specialised kernel per stage kind walks the 256 x 256
// output tiles of every matrix of the plan (all shape groups, one launch).
// CTAs run in clusters of two; the pair computes a tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16, bf16 x bf16 -> fp32):
// each CTA holds 128 rows of the left operand and a 128-wide half of the
// right operand in its shared memory, and 128 rows x 256 columns of the
// accumulator in its TMEM. Per SM that is 32 KB of operands per 4.2 MFLOP,
// two thirds of what a one-CTA 128 x 256 tile needs.
//
//   warp 0     TMA producer (both CTAs): 3-D tiled loads with 128-byte
//              swizzle into a 5- or 6-deep ring; the bytes of both CTAs are
//              counted on the pair leader's mbarrier.
//   warp 1     TMEM allocation (both CTAs); MMA issue (leader only):
//              tcgen05.commit multicasts slot releases and finished
//              accumulators to both CTAs. Two 256-column accumulators let
//              the epilogue of one tile overlap the main loop of the next.
//   warps 2-5  epilogue (both CTAs): each warp owns 32 accumulator rows,
//              reads 32 columns at a time from TMEM, stages results in
//              swizzled shared memory and writes them with TMA tensor stores
//              (whole lines, clipped at the matrix edge); inputs the
//              epilogue needs (the iterate, the Gram tile, the weight)
//              arrive by double-buffered TMA loads.
//
// The iterate is stored as two bf16 parts, X = high + low: the high part is
// the tensor-core operand (ping-pong, since every Apply tile reads the
// current one), the low part, rn(X - high), is updated in place by the tile
// that owns it. The pair carries 16 significant bits, enough for the a X term
// (the same O' error as an fp32 iterate in a CPU emulation of the rounding),
// and the Apply stage moves 4 bytes of iterate in and 4 out per element
// instead of 4 + 4 + 2 with an fp32 master beside a bf16 operand copy.
//
// Stages ("Ch 06 · Muon" §3 and §5 Algorithm 1, regrouped as
// a X + (b A + c A^2) X with A = X X^T):
//
//   Gram       A = X X^T. Symmetric: only pair tiles on or below the diagonal
//              run; each 128 x 128 block on or below the diagonal is stored
//              and, below the diagonal, mirrored. Step one folds s^2
//              (X_0 = s N).
//   Poly       B = b A + c A A^T (A symmetric), same tiling as Gram.
//   Apply      X' = a X + B X: B is the K-major left operand, the iterate's
//              high part the MN-major right operand (row-major X read as
//              K x N); the epilogue adds a (high + low). Step one folds s.
//   ApplyLast  the last step's Apply: O' = a X + B X, then the update of
//              "Muon 优化器完全拆解…", Algorithm 1 steps four and five,
//              W <- W (1 - lr wd) - lr gamma sqrt(max(n, m)) O', in the
//              caller's orientation (and O' when requested). W and O move by
//              TMA when their rows are 16-byte aligned, else by coalesced
//              plain loads and stores.
//
// Every spin-wait is bounded; on expiry the kernel raises the error word and
// an abort flag in both CTAs, stops issuing work, drains what is in flight,
// frees TMEM and returns.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx_sm100.cuh"
#include "stage_common.cuh"

namespace muon {

namespace {

constexpr int kApplyLast = 3;  // kernel kind beyond StageKind: the last Apply

constexpr int kHalf = 128;                        // rows of each operand half held by one CTA
constexpr int kABytes = kHalf * kBK * 2;          // 16 KB
constexpr int kBBytes = kHalf * kBK * 2;          // 16 KB
constexpr int kStageBytes = kABytes + kBBytes;    // 32 KB
constexpr uint32_t kPairTx = 2 * kStageBytes;     // bytes both CTAs land per ring slot
constexpr int kPairTile = 256;
constexpr int kTmemCols = 512;
constexpr int kEpiF32 = 32 * 32 * 4;              // fp32 32 x 32, 128-byte swizzle
constexpr int kEpiB16 = 32 * 32 * 2;              // bf16 32 x 32, 64-byte swizzle
constexpr size_t kBarrierBytes = 512;
constexpr int kTmapBytes = 128;

// Per-kind layout: ring depth and the epilogue staging slots (kEpiSlots per
// warp; four epilogue warps, one per TMEM lane quarter, or eight for Apply,
// two per quarter). The Apply-like kinds load an input per 32 x 32 chunk
// ahead of the chunk being processed. Slot sizes:
//   Gram       [bf16 out | bf16 mirror out]                            4 KB
//   Poly       [bf16 A in | bf16 out | bf16 mirror out]                6 KB
//   Apply      [bf16 iterate high in / out | bf16 low in / out]        4 KB
//   ApplyLast  [bf16 high in | bf16 low in, then fp32 O out | fp32 W in / out]  8 KB
// The iterate is kept as two bf16 parts, X = high + low (16 significant
// bits); the high part is the tensor-core operand.
//
// Wide variants run eight epilogue warps, two per TMEM lane quarter, each
// taking half of the columns, for one ring stage less. Apply is always wide
// (its epilogue moves the most data); Gram, Poly and ApplyLast are wide when
// the plan's tiles have short main loops, where the epilogue sets the tile
// rate (the host picks, by the mean K of the launch's tiles).
template <int KIND, bool WIDE = false>
struct Cfg {
  static constexpr bool kWide = WIDE || KIND == kApply;
  static constexpr int kEpiWarps = kWide ? 8 : 4;
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
  static constexpr int kStages = (KIND == kGram)   ? (kWide ? 5 : 6)
                                 : (KIND == kPoly) ? (kWide ? 4 : 5)
                                 : (KIND == kApply) ? 5
                                                    : (kWide ? 3 : 4);
  static constexpr int kSlot = (KIND == kApplyLast) ? 2 * kEpiF32
                               : (KIND == kPoly)    ? 3 * kEpiB16
                                                    : 2 * kEpiB16;
  static constexpr int kEpiSlots = (KIND == kApplyLast && !kWide) ? 3 : 2;
  static constexpr int kEpiBytes = kEpiWarps * kEpiSlots * kSlot;
  static constexpr size_t kSmem = 1024 + kStages * kStageBytes + kEpiBytes + kBarrierBytes;
  static constexpr bool kApplyLike = (KIND == kApply || KIND == kApplyLast);
  static constexpr int kTiles = kApplyLike ? kApply : KIND;  // which tile tables to walk
  static constexpr int kChunksPerWarp = (kPairTile / 32) / (kEpiWarps / 4);
  // symmetric kinds: where the direct and mirrored outputs sit in a slot
  static constexpr int kOffSymOut = (KIND == kPoly) ? kEpiB16 : 0;
  static constexpr int kOffSymMirror = kOffSymOut + kEpiB16;
};

constexpr int kOffLow = kEpiB16;   // low part of the iterate in Apply-like slots
constexpr int kSumsqSlots = 8;     // sum-of-squares slots per CTA and tile (most epilogue warps)
constexpr int kOffLastW = kEpiF32;

constexpr uint32_t kIdescKK = ptx::idesc_bf16(kPairTile, kPairTile, 0, 0);   // both K-major
constexpr uint32_t kIdescKMN = ptx::idesc_bf16(kPairTile, kPairTile, 0, 1);  // B MN-major

struct TileCoord {
  int g;
  int64_t b;    // matrix within the group
  int I, J;     // 256-row block, 256-column block
  int kblocks;  // K / 64, rounded up
};

// Lower-triangle pair tiles of the symmetric stages: (I, J) with J <= I,
// row-major: u = I (I + 1) / 2 + J.
__device__ __forceinline__ void lower_tile(int64_t u, int& I, int& J) {
  int64_t i = static_cast<int64_t>((sqrt(8.0 * static_cast<double>(u) + 1.0) - 1.0) * 0.5);
  while (i * (i + 1) / 2 > u) --i;
  while ((i + 1) * (i + 2) / 2 <= u) ++i;
  I = static_cast<int>(i);
  J = static_cast<int>(u - i * (i + 1) / 2);
}

template <int KIND>
__device__ __forceinline__ TileCoord decode_tile(const StageArgs& a, int64_t t) {
  constexpr int T = Cfg<KIND>::kTiles;
  TileCoord tc;
  tc.g = stage_group<T>(a, t);
  const GroupDesc& gd = a.groups[tc.g];
  const int64_t local = t - gd.tile_base[T];
  const int64_t per = gd.tiles_per_mat[T];
  tc.b = local / per;
  const int64_t u = local % per;
  if (T == kApply) {
    const int64_t rb = (gd.r + kPairTile - 1) / kPairTile;
    tc.I = static_cast<int>(u % rb);
    tc.J = static_cast<int>(u / rb);
    tc.kblocks = (gd.r + kBK - 1) / kBK;
  } else {
    lower_tile(u, tc.I, tc.J);
    tc.kblocks = ((T == kGram ? gd.c : gd.r) + kBK - 1) / kBK;
  }
  return tc;
}

__device__ __forceinline__ const void* tmap(const StageArgs& a, int g, int slot) {
  return static_cast<const char*>(a.tmaps) +
         (static_cast<int64_t>(g) * kTmPerGroup + slot) * kTmapBytes;
}

__device__ __forceinline__ const void* mat_tmap(const StageArgs& a, int mat, int slot) {
  return static_cast<const char*>(a.mat_tmaps) +
         (static_cast<int64_t>(mat) * kMtPerMat + slot) * kTmapBytes;
}

struct alignas(16) Bf16x8 {
  __nv_bfloat162 v[4];
};

// Byte offsets inside the swizzled staging tiles (buffers aligned to the
// swizzle period): 128-byte rows of fp32 (16-byte chunk q of row r lands at
// chunk q ^ (r % 8)); 64-byte rows of bf16 (chunk q ^ ((r / 2) % 4)).
__device__ __forceinline__ int sw128_chunk(int row, int q) { return row * 128 + ((q ^ (row & 7)) << 4); }
__device__ __forceinline__ int sw64_chunk(int row, int q) { return row * 64 + ((q ^ ((row >> 1) & 3)) << 4); }
// fp32 element (row, col) of a 32 x 32 tile with 128-byte swizzle
__device__ __forceinline__ int sw128_f32(int row, int col) { return sw128_chunk(row, col >> 2) + ((col & 3) << 2); }

// -------------------------------------------------------------- shared state

struct Smem {
  uint8_t* ring;   // stages x (A half | B half)
  uint8_t* epi;    // epilogue warps x 2 slots
  uint64_t* full;
  uint64_t* empty;
  uint64_t* tfull;
  uint64_t* tempty;
  uint64_t* drain;
  uint64_t* eload;  // epilogue warps x kEpiSlots
  uint32_t* tmem_slot;
  volatile int* abort_flag;
};

template <typename C>
__device__ __forceinline__ Smem carve(uint8_t* raw) {
  Smem s;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.ring = base;
  s.epi = base + C::kStages * kStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(s.epi + C::kEpiBytes);
  s.full = bars;
  s.empty = s.full + C::kStages;
  s.tfull = s.empty + C::kStages;
  s.tempty = s.tfull + 2;
  s.drain = s.tempty + 2;
  s.eload = s.drain + 1;
  s.tmem_slot = reinterpret_cast<uint32_t*>(s.eload + C::kEpiSlots * C::kEpiWarps);
  s.abort_flag = reinterpret_cast<volatile int*>(s.tmem_slot + 1);
  return s;
}

// Raise the abort flag in both CTAs of the pair and the device error word.
__device__ __forceinline__ void raise_abort(const StageArgs& a, const Smem& s) {
  const uint32_t local = ptx::smem_u32(const_cast<int*>(s.abort_flag));
  ptx::st_cluster_u32(ptx::mapa_shared(local, 0), 1u);
  ptx::st_cluster_u32(ptx::mapa_shared(local, 1), 1u);
  atomicOr(a.err, kErrTimeout);
}

// -------------------------------------------------------------- epilogue pieces

// Gram / Poly: one warp's 32 x 32 chunk of a block on or below the diagonal.
template <int KIND>
__device__ __forceinline__ void epi_symmetric(const StageArgs& a, const GroupDesc& gd,
                                              const TileCoord& tc, int row0, int col0, bool mirror,
                                              uint8_t* slot, const float (&v)[32], int lane) {
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
    // the A chunk, bf16 with 64-byte swizzle, in the slot's input area
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const Bf16x8 p = *reinterpret_cast<const Bf16x8*>(slot + sw64_chunk(lane, q));
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float2 f = __bfloat1622float2(p.v[h]);
        out[8 * q + 2 * h] = fmaf(a.b, f.x, a.c * v[8 * q + 2 * h]);
        out[8 * q + 2 * h + 1] = fmaf(a.b, f.y, a.c * v[8 * q + 2 * h + 1]);
      }
    }
  }
  uint8_t* st_direct = slot + Cfg<KIND>::kOffSymOut;
  uint8_t* st_mirror = slot + Cfg<KIND>::kOffSymMirror;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    Bf16x8 p;
#pragma unroll
    for (int h = 0; h < 4; ++h) p.v[h] = __floats2bfloat162_rn(out[8 * q + 2 * h], out[8 * q + 2 * h + 1]);
    *reinterpret_cast<Bf16x8*>(st_direct + sw64_chunk(lane, q)) = p;
  }
  if (mirror) {
    // transposed chunk: row e of the mirror holds column e of this chunk
    __nv_bfloat16* m16 = reinterpret_cast<__nv_bfloat16*>(st_mirror);
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int off = sw64_chunk(e, lane >> 3) + (lane & 7) * 2;
      m16[off >> 1] = __float2bfloat16_rn(out[e]);
    }
  }
  ptx::fence_async_shared();
  __syncwarp();
  if (lane == 0) {
    const void* tm = tmap(a, tc.g, KIND == kGram ? kTmAE : kTmBE);
    ptx::tma_store_3d(tm, st_direct, col0, row0, static_cast<int>(tc.b));
    if (mirror) ptx::tma_store_3d(tm, st_mirror, row0, col0, static_cast<int>(tc.b));
  }
}

// X' (or O') = alpha (a X + acc) for one warp's 32 x 32 chunk; X = high +
// low parts from the slot's two bf16 input areas.
__device__ __forceinline__ void apply_values(const StageArgs& a, float alpha, const uint8_t* slot,
                                             const float (&v)[32], int lane, float (&x)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const Bf16x8 h = *reinterpret_cast<const Bf16x8*>(slot + sw64_chunk(lane, q));
    const Bf16x8 l = *reinterpret_cast<const Bf16x8*>(slot + kOffLow + sw64_chunk(lane, q));
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 fh = __bfloat1622float2(h.v[k]);
      const float2 fl = __bfloat1622float2(l.v[k]);
      const int e = 8 * q + 2 * k;
      x[e] = alpha * fmaf(a.a, fh.x + fl.x, v[e]);
      x[e + 1] = alpha * fmaf(a.a, fh.y + fl.y, v[e + 1]);
    }
  }
}

// Apply: write the new iterate as bf16 high part (the next operand) and low
// part, high = rn(x'), low = rn(x' - high); x' - high is exact in fp32.
// `ssq` accumulates this lane's sum of squares of the new iterate (used by
// the unit-RMS update scale on the last step).
__device__ __forceinline__ void epi_apply(const StageArgs& a, const GroupDesc& gd, const TileCoord& tc,
                                          int row0, int col0, uint8_t* slot, const float (&v)[32],
                                          int lane, float& ssq) {
  const int mat = gd.first_mat + static_cast<int>(tc.b);
  const float alpha = a.first ? a.scale[mat] : 1.f;
  float x[32];
  apply_values(a, alpha, slot, v, lane, x);
  if (a.sumsq_per_tile > 0) {
    // rows and columns past the matrix hold zeros (zero-filled operands)
#pragma unroll
    for (int e = 0; e < 32; ++e) ssq = fmaf(x[e], x[e], ssq);
  }
  // each lane rewrites its own row of both areas: no other lane reads them
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    Bf16x8 h, l;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int e = 8 * q + 2 * k;
      h.v[k] = __floats2bfloat162_rn(x[e], x[e + 1]);
      const float2 fh = __bfloat1622float2(h.v[k]);
      l.v[k] = __floats2bfloat162_rn(x[e] - fh.x, x[e + 1] - fh.y);
    }
    *reinterpret_cast<Bf16x8*>(slot + sw64_chunk(lane, q)) = h;
    *reinterpret_cast<Bf16x8*>(slot + kOffLow + sw64_chunk(lane, q)) = l;
  }
  ptx::fence_async_shared();
  __syncwarp();
  if (lane == 0) {
    ptx::tma_store_3d(tmap(a, tc.g, a.xsrc ? kTmXb0E : kTmXb1E), slot, col0, row0,
                      static_cast<int>(tc.b));
    ptx::tma_store_3d(tmap(a, tc.g, kTmXloE), slot + kOffLow, col0, row0, static_cast<int>(tc.b));
  }
}

// Whether the last step moves this matrix's W and O by TMA.
__device__ __forceinline__ bool last_by_tma(const MatDesc& md) {
  return (!md.W || (md.flags & kMatWTma)) && (!md.O || (md.flags & kMatOTma));
}

// Caller coordinates (x = column, y = row) of the chunk at iterate (row0, col0).
__device__ __forceinline__ void caller_xy(const MatDesc& md, int row0, int col0, int& x, int& y) {
  x = md.transposed ? row0 : col0;
  y = md.transposed ? col0 : row0;
}

// ApplyLast: O' and the update, W <- W keep - step O', in the caller's
// orientation. With TMA the W chunk is in the slot's second area, in the
// caller's orientation (transposed relative to the iterate when n > m).
__device__ __forceinline__ void epi_apply_last(const StageArgs& a, const GroupDesc& gd,
                                               const TileCoord& tc, int row0, int col0, uint8_t* slot,
                                               const float (&v)[32], int lane, float& ssq) {
  const int mat = gd.first_mat + static_cast<int>(tc.b);
  const float alpha = a.first ? a.scale[mat] : 1.f;
  float x[32];
  apply_values(a, alpha, slot, v, lane, x);
  if (a.sumsq_per_tile > 0) {
    // update-RMS diagnostics; rows and columns past the matrix hold zeros
#pragma unroll
    for (int e = 0; e < 32; ++e) ssq = fmaf(x[e], x[e], ssq);
  }
  const MatDesc& md = a.mats[mat];
  const UpdateConsts uc = update_consts(a, gd.c);
  const bool tr = md.transposed != 0;

  if (last_by_tma(md)) {
    // element (iterate row lane, col e) sits at (lane, e), or at (e, lane) when transposed
    if (md.W) {
      uint8_t* Ws = slot + kOffLastW;
      if (!tr) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float4* p = reinterpret_cast<float4*>(Ws + sw128_chunk(lane, q));
          float4 w = *p;
          w.x = fmaf(w.x, uc.keep, -uc.step * x[4 * q + 0]);
          w.y = fmaf(w.y, uc.keep, -uc.step * x[4 * q + 1]);
          w.z = fmaf(w.z, uc.keep, -uc.step * x[4 * q + 2]);
          w.w = fmaf(w.w, uc.keep, -uc.step * x[4 * q + 3]);
          *p = w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          float* p = reinterpret_cast<float*>(Ws + sw128_f32(e, lane));
          *p = fmaf(*p, uc.keep, -uc.step * x[e]);
        }
      }
    }
    if (md.O) {
      __syncwarp();  // every lane has read its iterate values: the area takes O'
      if (!tr) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<float4*>(slot + sw128_chunk(lane, q)) =
              make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) *reinterpret_cast<float*>(slot + sw128_f32(e, lane)) = x[e];
      }
    }
    ptx::fence_async_shared();
    __syncwarp();
    if (lane == 0) {
      int cx, cy;
      caller_xy(md, row0, col0, cx, cy);
      if (md.W) ptx::tma_store_3d(mat_tmap(a, mat, kMtW), slot + kOffLastW, cx, cy, 0);
      if (md.O) ptx::tma_store_3d(mat_tmap(a, mat, kMtO), slot, cx, cy, 0);
    }
    return;
  }

  // Plain loads and stores (rows not 16-byte aligned).
  const int mrows = (gd.r - row0) < 32 ? (gd.r - row0) : 32;
  const int ncol = (gd.c - col0) < 32 ? (gd.c - col0) : 32;
  if (tr) {
    // caller element (col, row): for each column the lanes (rows) hit consecutive addresses
    if (lane < mrows) {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (e < ncol) write_update(md, uc, row0 + lane, col0 + e, x[e]);
    }
    return;
  }
  // Row-major caller matrix: move O' to "lane = column" layout through a
  // 32 x 32 transpose in shared memory (word (r, c) at r * 32 + (c ^ r):
  // conflict-free both ways); then every global access of the warp is one
  // contiguous row segment, all 32 rows' loads in flight at once. The slot's
  // second area is unused on this path.
  float* T = reinterpret_cast<float*>(slot + kOffLastW);
#pragma unroll
  for (int e = 0; e < 32; ++e) T[lane * 32 + (e ^ lane)] = x[e];
  __syncwarp();
  float xc[32];
#pragma unroll
  for (int rr = 0; rr < 32; ++rr) xc[rr] = T[rr * 32 + (lane ^ rr)];
  const bool col_ok = lane < ncol;
  float* Wp = md.W ? md.W + static_cast<int64_t>(row0) * md.m + col0 + lane : nullptr;
  float* Op = md.O ? md.O + static_cast<int64_t>(row0) * md.m + col0 + lane : nullptr;
  if (Op) {
#pragma unroll
    for (int rr = 0; rr < 32; ++rr)
      if (col_ok && rr < mrows) Op[static_cast<int64_t>(rr) * md.m] = xc[rr];
  }
  if (Wp) {
    float w[32];
#pragma unroll
    for (int rr = 0; rr < 32; ++rr) w[rr] = (col_ok && rr < mrows) ? Wp[static_cast<int64_t>(rr) * md.m] : 0.f;
#pragma unroll
    for (int rr = 0; rr < 32; ++rr)
      if (col_ok && rr < mrows) Wp[static_cast<int64_t>(rr) * md.m] = fmaf(w[rr], uc.keep, -uc.step * xc[rr]);
  }
  // a later TMA load may overwrite this slot: order these accesses before it
  ptx::fence_async_shared();
  __syncwarp();
}

// -------------------------------------------------------------- kernel

template <int KIND, bool WIDE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg<KIND, WIDE>::kThreads, 1)
    stage_tc_kernel(const __grid_constant__ StageArgs a) {
  using C = Cfg<KIND, WIDE>;
  constexpr int kStages = C::kStages;
  constexpr int kEpiWarps = C::kEpiWarps;
  extern __shared__ uint8_t smem_raw[];
  const Smem s = carve<C>(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const int64_t pair = blockIdx.x >> 1;
  const int64_t npairs = gridDim.x >> 1;
  const uint64_t limit = a.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      ptx::mbar_init(&s.full[i], 1);
      ptx::mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&s.tfull[i], 1);
      ptx::mbar_init(&s.tempty[i], 2 * kEpiWarps);
    }
    ptx::mbar_init(s.drain, 1);
    for (int i = 0; i < C::kEpiSlots * kEpiWarps; ++i) ptx::mbar_init(&s.eload[i], 1);
    *s.abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(s.tmem_slot, kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();  // barriers of both CTAs initialised before any remote use
  ptx::tc_fence_after();
  const uint32_t tmem_base = *s.tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- producer
    for (int g = 0; g < a.ngroups; ++g)
      for (int k = 0; k < kTmPerGroup; ++k) {
        ptx::fence_tmap_acquire(tmap(a, g, k));
        ptx::prefetch_tmap(tmap(a, g, k));
      }
    uint32_t leader_full[kStages];
    for (int i = 0; i < kStages; ++i) leader_full[i] = ptx::mapa_shared(ptx::smem_u32(&s.full[i]), 0);
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    for (int64_t t = a.tile_begin + pair; ok && t < a.total_tiles; t += npairs) {
      const TileCoord tc = decode_tile<KIND>(a, t);
      const int bz = static_cast<int>(tc.b);
      for (int kb = 0; kb < tc.kblocks; ++kb) {
        if (!ptx::mbar_wait(&s.empty[stage], phase ^ 1, limit, s.abort_flag)) {
          raise_abort(a, s);
          ok = false;
          break;
        }
        uint8_t* sa = s.ring + stage * kStageBytes;
        uint8_t* sb = sa + kABytes;
        const bool diag = !C::kApplyLike && tc.I == tc.J;
        if (rank == 0) ptx::mbar_arrive_expect_tx(&s.full[stage], diag ? kPairTx / 2 : kPairTx);
        const int k0 = kb * kBK;
        if (C::kApplyLike) {
          ptx::tma_load_3d_pair(sa, tmap(a, tc.g, kTmB), leader_full[stage], k0,
                                tc.I * kPairTile + rank * kHalf, bz);
          const void* tx = tmap(a, tc.g, a.xsrc ? kTmXb1MN : kTmXb0MN);
#pragma unroll
          for (int q = 0; q < kHalf / 64; ++q)
            ptx::tma_load_3d_pair(sb + q * (64 * kBK * 2), tx, leader_full[stage],
                                  tc.J * kPairTile + rank * kHalf + q * 64, k0, bz);
        } else {
          const void* tm = (KIND == kGram) ? tmap(a, tc.g, a.xsrc ? kTmXb1K : kTmXb0K)
                                           : tmap(a, tc.g, kTmA);
          ptx::tma_load_3d_pair(sa, tm, leader_full[stage], k0, tc.I * kPairTile + rank * kHalf, bz);
          // on a diagonal tile each CTA's right-operand half is its left-operand rows
          if (tc.I != tc.J)
            ptx::tma_load_3d_pair(sb, tm, leader_full[stage], k0, tc.J * kPairTile + rank * kHalf, bz);
        }
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (!ok) {
      // give copies already issued time to land before the pair exits
      const uint64_t t0 = ptx::globaltimer_ns();
      while (ptx::globaltimer_ns() - t0 < 20000) {
      }
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ---------------------------------------------------------- MMA issuer (pair leader)
    const uint32_t idesc = C::kApplyLike ? kIdescKMN : kIdescKK;
    uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
    bool ok = true;
    bool issued = false;
    for (int64_t t = a.tile_begin + pair; ok && t < a.total_tiles; t += npairs) {
      const TileCoord tc = decode_tile<KIND>(a, t);
      if (!ptx::mbar_wait(&s.tempty[acc], acc_phase ^ 1, limit, s.abort_flag)) {
        raise_abort(a, s);
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t d = tmem_base + acc * kPairTile;
      for (int kb = 0; kb < tc.kblocks; ++kb) {
        if (!ptx::mbar_wait(&s.full[stage], phase, limit, s.abort_flag)) {
          raise_abort(a, s);
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t sa = ptx::smem_u32(s.ring + stage * kStageBytes);
        const uint32_t sb = (!C::kApplyLike && tc.I == tc.J) ? sa : sa + kABytes;
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k) {
          const uint64_t ad = ptx::desc_sw128(sa + k * 32, 16, 1024);
          const uint64_t bd = C::kApplyLike ? ptx::desc_sw128(sb + k * 16 * 128, 64 * kBK * 2, 1024)
                                            : ptx::desc_sw128(sb + k * 32, 16, 1024);
          ptx::umma_bf16_pair(d, ad, bd, idesc, (kb | k) != 0);
        }
        issued = true;
        ptx::umma_commit_pair(&s.empty[stage]);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      ptx::umma_commit_pair(&s.tfull[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if (!ok && issued) {
      // let the MMAs in flight finish before TMEM is released
      volatile int never = 0;
      ptx::umma_commit_pair_self(s.drain);
      ptx::mbar_wait(s.drain, 0, limit, &never);
    }
  } else if (warp >= 2) {
    // ---------------------------------------------------------- epilogue
    const int ew = warp - 2;
    const int quarter = warp & 3;  // TMEM lanes this warp may read: 32 * quarter ...
    const int ch_begin = (ew / 4) * C::kChunksPerWarp;  // this warp's share of the columns
    const int ch_end = ch_begin + C::kChunksPerWarp;
    constexpr int S = C::kEpiSlots;
    uint8_t* slots = s.epi + ew * S * C::kSlot;
    uint64_t* eload = s.eload + S * ew;
    uint32_t eload_phase = 0u;  // bit i: phase of slot i's load barrier
    uint32_t leader_tempty[2];
    for (int i = 0; i < 2; ++i) leader_tempty[i] = ptx::mapa_shared(ptx::smem_u32(&s.tempty[i]), 0);
    constexpr bool kInput = (KIND != kGram);
    // input loads in flight ahead of the current chunk: with three or more
    // slots the newest chunk's stores may still be reading their slot when the
    // next load is issued (no wait on them); with two they must have finished
    constexpr int D = !kInput ? 0 : (S >= 3 ? S - 2 : S - 1);
    constexpr int kReuseWait = S - 1 - D;  // store groups that may still be pending
    uint32_t acc = 0, acc_phase = 0;
    bool ok = true;
    for (int64_t t = a.tile_begin + pair; ok && t < a.total_tiles; t += npairs) {
      const TileCoord tc = decode_tile<KIND>(a, t);
      const GroupDesc& gd = a.groups[tc.g];
      const int row0 = tc.I * kPairTile + static_cast<int>(rank) * kHalf + quarter * 32;
      const int bi = (tc.I * kPairTile + static_cast<int>(rank) * kHalf) / kHalf;
      const int bz = static_cast<int>(tc.b);
      const int mat = gd.first_mat + bz;
      // Apply-like: the current iterate's high part (the operand buffer) and low part
      const void* in_map = tmap(a, tc.g, C::kApplyLike ? (a.xsrc ? kTmXb1E : kTmXb0E) : kTmAE);
      float ssq = 0.f;  // sum of squares of this warp's share of X' (unit-RMS scale)
      // the last step also brings the weight chunk, in the caller's orientation
      bool w_in = false;
      bool w_tr = false;
      if (KIND == kApplyLast) {
        const MatDesc& md = a.mats[mat];
        w_in = md.W && last_by_tma(md);
        w_tr = md.transposed != 0;
        if (lane == 0 && last_by_tma(md)) {
          if (md.W) ptx::fence_tmap_acquire(mat_tmap(a, mat, kMtW));
          if (md.O) ptx::fence_tmap_acquire(mat_tmap(a, mat, kMtO));
        }
      }
      const uint32_t in_bytes = (KIND == kPoly ? kEpiB16 : 2 * kEpiB16) + (w_in ? kEpiF32 : 0);
      const int limit_c = C::kApplyLike ? gd.c : gd.r;
      // rows or columns past the matrix: nothing to load or store for a chunk
      auto live_chunk = [&](int ch) {
        return ch < ch_end && row0 < gd.r && tc.J * kPairTile + ch * 32 < limit_c;
      };
      auto issue_load = [&](int ch) {  // the caller has made sure the slot is free
        const int sl = (ch - ch_begin) % S;
        uint8_t* slot = slots + sl * C::kSlot;
        uint64_t* bar = &eload[sl];
        const int col0 = tc.J * kPairTile + ch * 32;
        ptx::mbar_arrive_expect_tx(bar, in_bytes);
        ptx::tma_load_3d(slot, in_map, bar, col0, row0, bz);
        if (C::kApplyLike) ptx::tma_load_3d(slot + kOffLow, tmap(a, tc.g, kTmXloE), bar, col0, row0, bz);
        if (KIND == kApplyLast && w_in)
          ptx::tma_load_3d(slot + kOffLastW, mat_tmap(a, mat, kMtW), bar, w_tr ? row0 : col0,
                           w_tr ? col0 : row0, 0);
      };
      if (kInput && lane == 0) {
        ptx::bulk_wait_read<0>();  // the previous tile's stores have read every slot
        for (int ch = ch_begin; ch < ch_begin + D; ++ch)
          if (live_chunk(ch)) issue_load(ch);
      }
      if (!ptx::mbar_wait(&s.tfull[acc], acc_phase, limit, s.abort_flag)) {
        raise_abort(a, s);
        ok = false;
      }
      ptx::tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * kPairTile;
#pragma unroll 1
      for (int ch = ch_begin; ok && ch < ch_end; ++ch) {
        const int sl = (ch - ch_begin) % S;
        uint8_t* slot = slots + sl * C::kSlot;
        const int col0 = tc.J * kPairTile + ch * 32;
        const bool live = live_chunk(ch);
        if (lane == 0) {
          // the load D chunks ahead reuses the slot of chunk ch + D - S, whose
          // stores are older than the newest kReuseWait groups
          if (kInput && live_chunk(ch + D)) {
            ptx::bulk_wait_read<kReuseWait>();
            issue_load(ch + D);
          }
          if (!kInput) ptx::bulk_wait_read<1>();  // two slots: chunk ch - 2's stores have read it
        }
        __syncwarp();
        float v[32];
        ptx::tmem_ld32(taddr + ch * 32, v);
        if (kInput && live) {
          if (!ptx::mbar_wait(&eload[sl], (eload_phase >> sl) & 1u, limit, s.abort_flag)) {
            raise_abort(a, s);
            ok = false;
            break;
          }
          eload_phase ^= 1u << sl;
        }
        if (live) {
          if (KIND == kApply) {
            epi_apply(a, gd, tc, row0, col0, slot, v, lane, ssq);
          } else if (KIND == kApplyLast) {
            epi_apply_last(a, gd, tc, row0, col0, slot, v, lane, ssq);
          } else {
            const int bj = col0 / kHalf;
            if (bj <= bi) epi_symmetric<KIND>(a, gd, tc, row0, col0, bj < bi, slot, v, lane);
          }
        }
        // one bulk group per chunk (possibly empty), so "all but the newest
        // group" always means "every chunk before the previous one"
        __syncwarp();
        if (lane == 0) ptx::bulk_commit();
      }
      if ((KIND == kApply || KIND == kApplyLast) && a.sumsq_per_tile > 0) {
        // one slot per (tile, CTA of the pair, epilogue warp); every slot is written
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
        // kSumsqSlots per CTA and tile; a kind with fewer epilogue warps zeroes the rest
        if (lane == 0) {
          float* dst = a.sumsq + (t * 2 + rank) * kSumsqSlots;
          dst[ew] = ssq;
          for (int e = ew + kEpiWarps; e < kSumsqSlots; e += kEpiWarps) dst[e] = 0.f;
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(leader_tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if (lane == 0) ptx::bulk_wait<0>();
    if (!ok) {
      // give an input load still in flight time to land before the pair exits
      const uint64_t t0 = ptx::globaltimer_ns();
      while (ptx::globaltimer_ns() - t0 < 20000) {
      }
    }
    __syncwarp();
  }

  __syncwarp();
  ptx::tc_fence_before();
  ptx::cluster_sync();  // neither CTA leaves while its partner may still use its memory
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

template <int KIND, bool WIDE>
cudaError_t launch_kind(const StageArgs& args, int grid, cudaStream_t stream) {
  using C = Cfg<KIND, WIDE>;
  constexpr size_t smem = C::kSmem;
  static_assert(smem <= 227 * 1024, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(stage_tc_kernel<KIND, WIDE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  stage_tc_kernel<KIND, WIDE><<<grid, C::kThreads, smem, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace

size_t stage_tc_smem_bytes() { return Cfg<kGram>::kSmem; }

cudaError_t launch_stage_tc(StageKind kind, const StageArgs& args, int grid, bool wide,
                            cudaStream_t stream) {
  if (args.total_tiles <= args.tile_begin) return cudaSuccess;
  if (grid < 2 || (grid & 1)) return cudaErrorInvalidConfiguration;
  switch (kind) {
    case kGram:
      return wide ? launch_kind<kGram, true>(args, grid, stream) : launch_kind<kGram, false>(args, grid, stream);
    case kPoly:
      return wide ? launch_kind<kPoly, true>(args, grid, stream) : launch_kind<kPoly, false>(args, grid, stream);
    case kApply:
      if (!args.last) return launch_kind<kApply, true>(args, grid, stream);
      return wide ? launch_kind<kApplyLast, true>(args, grid, stream)
                  : launch_kind<kApplyLast, false>(args, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace muon
