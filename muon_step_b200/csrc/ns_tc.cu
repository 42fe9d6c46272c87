// Newton-Schulz stages on the sm_100a tensor cores, one CTA pair per tile.
//
// Persistent, warp-specialised kernels walk 256 x 256 output tiles of every
// matrix of the plan (all shape groups). CTAs run in clusters of two; the
// pair computes a tile with tcgen05.mma.cta_group::2 (M = 256, N = 256,
// K = 16, bf16 x bf16 -> fp32): each CTA holds 128 rows of the left operand
// and a 128-wide half of the right operand in its shared memory, and 128 rows
// x 256 columns of the accumulator in its TMEM. Per SM that is 32 KB of
// operands per 4.2 MFLOP, two thirds of what a one-CTA 128 x 256 tile needs.
//
//   warp 0     TMA producer (both CTAs): 3-D tiled loads with 128-byte
//              swizzle into a ring of 32 KB stages; the bytes of both CTAs
//              are counted on the pair leader's mbarrier.
//   warp 1     TMEM allocation (both CTAs); MMA issue (leader only):
//              tcgen05.commit with .multicast::cluster arrives on an mbarrier
//              in both CTAs of the pair (ring slot released, accumulator
//              ready); it is an mbarrier signal inside the CTA pair, not a
//              memory load. Two 256-column accumulators let the epilogue of
//              one tile overlap the main loop of the next.
//   warps 2-   epilogue (both CTAs): each warp owns 32 accumulator rows,
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
//              run, and only they are stored (the lower triangle of 256-row
//              blocks, diagonal blocks in full). Step one folds s^2
//              (X_0 = s N).
//   Poly       B = b A + c A A^T (A symmetric), same tiling and storage as
//              Gram. A K block of A above its row block's diagonal is read
//              from the transposed, stored position as an MN-major operand.
//   Apply      X' = a X + B X: B is the left operand (K-major, or MN-major
//              above the diagonal as in Poly), the iterate's high part the
//              MN-major right operand (row-major X read as K x N); the
//              epilogue adds a (high + low). Step one folds s.
//   ApplyLast  the last step's Apply: O' = a X + B X, then the update of
//              "Muon 优化器完全拆解…", Algorithm 1 steps four and five,
//              W <- W (1 - lr wd) - lr gamma sqrt(max(n, m)) O', in the
//              caller's orientation (and O' when requested). W and O move by
//              TMA when their rows are 16-byte aligned, else by coalesced
//              plain loads and stores.
//
// Two kernels share the per-tile work (producer loads, MMA issue, epilogue):
//
//   stage_tc_kernel<KIND>  one stage of one step over every matrix (one
//                          launch per stage);
//   stage_chain_kernel     every Gram, Poly and Apply stage of the schedule
//                          in one persistent launch. Tiles are taken in the
//                          order of a host-built list that keeps a window of
//                          matrices in flight, so their buffers stay in L2
//                          from one stage to the next. A matrix's stages
//                          depend on each other only: per matrix, a counter
//                          in global memory counts the epilogue warps that
//                          have finished a tile (after their TMA stores have
//                          landed: wait, proxy fence, release add), and a
//                          tile's producer and epilogue warps wait (acquire)
//                          until every tile of the matrix's earlier stages
//                          has finished. CTA pairs take list indices from
//                          a global counter as they become free (the pair
//                          leader's producer fetches and publishes each to
//                          both CTAs' roles through a small queue), so the
//                          earliest unfinished tile is always held by a
//                          running pair and can run, however many pairs the
//                          device holds at once.
//
// Every spin-wait is bounded; on expiry the kernel raises the error word and
// an abort flag in both CTAs, stops issuing work, drains what is in flight,
// frees TMEM and returns. The chained kernel's dependency waits also give up
// as soon as any CTA has raised the error word.
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
constexpr int kTileQ = 4;  // chained launch: tile indices published ahead of their use

// Facts of a tile kind that do not depend on the launch layout. Slot use:
//   Gram       [bf16 out | unused]                                     4 KB
//   Poly       [bf16 A in | bf16 out]                                  4 KB
//   Apply      [bf16 iterate high in / out | bf16 low in / out]        4 KB
//   ApplyLast  [bf16 high in | bf16 low in, then fp32 O out | fp32 W in / out]  8 KB
template <int KIND>
struct KindT {
  static constexpr bool kApplyLike = (KIND == kApply || KIND == kApplyLast);
  static constexpr int kTiles = kApplyLike ? kApply : KIND;  // which tile tables to walk
  static constexpr bool kInput = (KIND != kGram);            // the epilogue loads inputs
  static constexpr int kSlotUse = (KIND == kApplyLast) ? 2 * kEpiF32 : 2 * kEpiB16;
  // symmetric kinds: where the output sits in a slot (Poly's A input takes the first area)
  static constexpr int kOffSymOut = (KIND == kPoly) ? kEpiB16 : 0;
};

// Launch layout: ring depth, epilogue warps (one per TMEM lane quarter, or
// two, each with half of the columns), staging slot size and slots per warp.
template <int STAGES, int EPI_WARPS, int SLOT, int SLOTS>
struct Layout {
  static constexpr int kStages = STAGES;
  static constexpr int kEpiWarps = EPI_WARPS;
  static constexpr int kThreads = 64 + 32 * EPI_WARPS;
  static constexpr int kSlot = SLOT;
  static constexpr int kEpiSlots = SLOTS;
  static constexpr int kEpiBytes = EPI_WARPS * SLOTS * SLOT;
  static constexpr size_t kSmem = 1024 + STAGES * kStageBytes + kEpiBytes + kBarrierBytes;
  static constexpr int kChunksPerWarp = (kPairTile / 32) / (EPI_WARPS / 4);
  // mbarriers (ring, accumulators, drain, epilogue loads, tile queue), then
  // the TMEM address, the abort flag and the tile queue's entries
  static_assert(8 * (2 * STAGES + 5 + SLOTS * EPI_WARPS + 2 * kTileQ) + 8 + 4 * kTileQ <= kBarrierBytes,
                "barrier area");
};

// Layout of the one-stage kernels. Wide variants run eight epilogue warps
// for one ring stage less. Apply is always wide (its epilogue moves the most
// data); Gram, Poly and ApplyLast are wide when the plan's tiles have short
// main loops, where the epilogue sets the tile rate (the host picks, by the
// mean K of the launch's tiles).
template <int KIND, bool WIDE>
struct StageLayout {
  static constexpr bool kWide = WIDE || KIND == kApply;
  static constexpr int kStages = (KIND == kGram || KIND == kPoly) ? (kWide ? 5 : 6)
                                 : (KIND == kApply)                ? 5
                                                                   : (kWide ? 3 : 4);
  static constexpr int kEpiSlots = (KIND == kApplyLast && !kWide) ? 3 : 2;
  using L = Layout<kStages, kWide ? 8 : 4, KindT<KIND>::kSlotUse, kEpiSlots>;
};

// The chained launch runs Gram, Poly and Apply tiles with one layout: eight
// epilogue warps, two 4 KB slots each, five ring stages.
using ChainL = Layout<5, 8, 2 * kEpiB16, 2>;
static_assert(ChainL::kSmem <= 227 * 1024, "shared memory budget");

constexpr int kOffLow = kEpiB16;   // low part of the iterate in Apply-like slots
constexpr int kSumsqSlots = 8;     // sum-of-squares slots per CTA and tile (most epilogue warps)
constexpr int kOffLastW = kEpiF32;

// instruction descriptors by operand major-ness (A side, B side; 1 = MN-major)
__device__ __forceinline__ uint32_t idesc_of(bool a_mn, bool b_mn) {
  return ptx::idesc_bf16(kPairTile, kPairTile, a_mn ? 1 : 0, b_mn ? 1 : 0);
}

struct TileCoord {
  int g;
  int64_t b;    // matrix within the group
  int I, J;     // 256-row block, 256-column block
  int kblocks;  // K / 64, rounded up
};

// The step a tile belongs to, as its epilogue needs it.
struct StepP {
  int32_t first;   // step one: fold the normalisation scale
  int32_t xsrc;    // ping-pong buffer holding the current iterate
  int32_t record;  // Apply kinds: record sums of squares of X'
  float a, b, c;   // the step's coefficients
};

__device__ __forceinline__ StepP step_of(const StageArgs& a) {
  StepP p;
  p.first = a.first;
  p.xsrc = a.xsrc;
  p.record = a.sumsq_per_tile > 0;
  p.a = a.a;
  p.b = a.b;
  p.c = a.c;
  return p;
}

// Lower-triangle pair tiles of the symmetric stages: (I, J) with J <= I,
// row-major: u = I (I + 1) / 2 + J.
__device__ __forceinline__ void lower_tile(int64_t u, int& I, int& J) {
  int64_t i = static_cast<int64_t>((sqrt(8.0 * static_cast<double>(u) + 1.0) - 1.0) * 0.5);
  while (i * (i + 1) / 2 > u) --i;
  while ((i + 1) * (i + 2) / 2 <= u) ++i;
  I = static_cast<int>(i);
  J = static_cast<int>(u - i * (i + 1) / 2);
}

// Tile u of matrix b of group g in the table of stage kind T.
template <int T>
__device__ __forceinline__ TileCoord coord_of(const GroupDesc& gd, int g, int64_t b, int64_t u) {
  TileCoord tc;
  tc.g = g;
  tc.b = b;
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

template <int KIND>
__device__ __forceinline__ TileCoord decode_tile(const StageArgs& a, int64_t t) {
  constexpr int T = KindT<KIND>::kTiles;
  const int g = stage_group<T>(a, t);
  const GroupDesc& gd = a.groups[g];
  const int64_t local = t - gd.tile_base[T];
  const int64_t per = gd.tiles_per_mat[T];
  return coord_of<T>(gd, g, local / per, local % per);
}

// Where a tile of the chained list sits, and what it waits for.
struct ChainPos {
  TileCoord tc;
  int kind;         // Gram, Poly or Apply
  int step;
  uint32_t need;    // dependency counter value at which every earlier stage is done
  int64_t t_apply;  // Apply tiles: index in the Apply table (sum-of-squares slots)
};

__device__ __forceinline__ ChainPos chain_pos(const StageArgs& a, const ChainTile& ct) {
  ChainPos cp;
  const MatDesc& md = a.mats[ct.mat];
  const GroupDesc& gd = a.groups[md.group];
  cp.kind = ct.stage % 3;
  cp.step = ct.stage / 3;
  if (cp.kind == kApply) cp.tc = coord_of<kApply>(gd, md.group, md.index, ct.tile);
  else if (cp.kind == kPoly) cp.tc = coord_of<kPoly>(gd, md.group, md.index, ct.tile);
  else cp.tc = coord_of<kGram>(gd, md.group, md.index, ct.tile);
  const int64_t g0 = gd.tiles_per_mat[kGram], p0 = gd.tiles_per_mat[kPoly], a0 = gd.tiles_per_mat[kApply];
  const int64_t prefix = cp.step * (g0 + p0 + a0) + (cp.kind >= 1 ? g0 : 0) + (cp.kind >= 2 ? p0 : 0);
  cp.need = static_cast<uint32_t>(prefix * kChainArrivals);
  cp.t_apply = gd.tile_base[kApply] + static_cast<int64_t>(md.index) * a0 + ct.tile;
  return cp;
}

__device__ __forceinline__ StepP chain_step(const StageArgs& a, const ChainTile& ct, int step) {
  StepP p;
  p.first = step == 0;
  p.xsrc = step & 1;
  p.record = ct.stage == a.chain_sumsq_stage;
  p.a = a.abc[3 * step];
  p.b = a.abc[3 * step + 1];
  p.c = a.abc[3 * step + 2];
  return p;
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
  uint8_t* epi;    // epilogue warps x slots
  uint64_t* full;
  uint64_t* empty;
  uint64_t* tfull;
  uint64_t* tempty;
  uint64_t* drain;
  uint64_t* eload;  // epilogue warps x slots
  uint64_t* tq_full;   // chained launch: tile queue, entry published (both CTAs)
  uint64_t* tq_empty;  // ... entry read by every consumer (pair leader)
  uint32_t* tmem_slot;
  volatile int* abort_flag;
  volatile uint32_t* tq;  // tile indices
};

template <typename L>
__device__ __forceinline__ Smem carve(uint8_t* raw) {
  Smem s;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.ring = base;
  s.epi = base + L::kStages * kStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(s.epi + L::kEpiBytes);
  s.full = bars;
  s.empty = s.full + L::kStages;
  s.tfull = s.empty + L::kStages;
  s.tempty = s.tfull + 2;
  s.drain = s.tempty + 2;
  s.eload = s.drain + 1;
  s.tq_full = s.eload + L::kEpiSlots * L::kEpiWarps;
  s.tq_empty = s.tq_full + kTileQ;
  s.tmem_slot = reinterpret_cast<uint32_t*>(s.tq_empty + kTileQ);
  s.abort_flag = reinterpret_cast<volatile int*>(s.tmem_slot + 1);
  s.tq = reinterpret_cast<volatile uint32_t*>(s.abort_flag + 1);
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
__device__ __forceinline__ void epi_symmetric(const StageArgs& a, const StepP& p, const GroupDesc& gd,
                                              const TileCoord& tc, int row0, int col0, uint8_t* slot,
                                              const float (&v)[32], int lane) {
  float out[32];
  if (KIND == kGram) {
    // step one folds s^2; later steps store the product as it is (s^2 = 1)
    if (p.first) {
      const float sc = a.scale[gd.first_mat + tc.b];
      const float s2 = sc * sc;
#pragma unroll
      for (int e = 0; e < 32; ++e) out[e] = s2 * v[e];
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) out[e] = v[e];
    }
  } else {
    // the A chunk, bf16 with 64-byte swizzle, in the slot's input area
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const Bf16x8 pa = *reinterpret_cast<const Bf16x8*>(slot + sw64_chunk(lane, q));
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float2 f = __bfloat1622float2(pa.v[h]);
        out[8 * q + 2 * h] = fmaf(p.b, f.x, p.c * v[8 * q + 2 * h]);
        out[8 * q + 2 * h + 1] = fmaf(p.b, f.y, p.c * v[8 * q + 2 * h + 1]);
      }
    }
  }
  uint8_t* st_direct = slot + KindT<KIND>::kOffSymOut;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    Bf16x8 pk;
#pragma unroll
    for (int h = 0; h < 4; ++h) pk.v[h] = __floats2bfloat162_rn(out[8 * q + 2 * h], out[8 * q + 2 * h + 1]);
    *reinterpret_cast<Bf16x8*>(st_direct + sw64_chunk(lane, q)) = pk;
  }
  ptx::fence_async_shared();
  __syncwarp();
  if (lane == 0) {
    const void* tm = tmap(a, tc.g, KIND == kGram ? kTmAE : kTmBE);
    ptx::tma_store_3d(tm, st_direct, col0, row0, static_cast<int>(tc.b));
  }
}

// X' (or O') = alpha (a X + acc) for one warp's 32 x 32 chunk; X = high +
// low parts from the slot's two bf16 input areas. alpha is the step-one
// scale s, and 1 on later steps (no multiply then: the same values).
__device__ __forceinline__ void apply_values(const StepP& p, float alpha, const uint8_t* slot,
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
      x[e] = fmaf(p.a, fh.x + fl.x, v[e]);
      x[e + 1] = fmaf(p.a, fh.y + fl.y, v[e + 1]);
    }
  }
  if (p.first) {
#pragma unroll
    for (int e = 0; e < 32; ++e) x[e] = alpha * x[e];
  }
}

// Apply: write the new iterate as bf16 high part (the next operand) and low
// part, high = rn(x'), low = rn(x' - high); x' - high is exact in fp32.
// `ssq` accumulates this lane's sum of squares of the new iterate (used by
// the unit-RMS update scale on the last step).
__device__ __forceinline__ void epi_apply(const StageArgs& a, const StepP& p, const GroupDesc& gd,
                                          const TileCoord& tc, int row0, int col0, uint8_t* slot,
                                          const float (&v)[32], int lane, float& ssq) {
  const int mat = gd.first_mat + static_cast<int>(tc.b);
  const float alpha = p.first ? a.scale[mat] : 1.f;
  float x[32];
  apply_values(p, alpha, slot, v, lane, x);
  if (p.record) {
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
    ptx::tma_store_3d(tmap(a, tc.g, p.xsrc ? kTmXb0E : kTmXb1E), slot, col0, row0,
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
__device__ __forceinline__ void epi_apply_last(const StageArgs& a, const StepP& p, const GroupDesc& gd,
                                               const TileCoord& tc, int row0, int col0, uint8_t* slot,
                                               const float (&v)[32], int lane, float& ssq) {
  const int mat = gd.first_mat + static_cast<int>(tc.b);
  const float alpha = p.first ? a.scale[mat] : 1.f;
  float x[32];
  apply_values(p, alpha, slot, v, lane, x);
  if (p.record) {
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
          float4* pw = reinterpret_cast<float4*>(Ws + sw128_chunk(lane, q));
          float4 w = *pw;
          w.x = fmaf(w.x, uc.keep, -uc.step * x[4 * q + 0]);
          w.y = fmaf(w.y, uc.keep, -uc.step * x[4 * q + 1]);
          w.z = fmaf(w.z, uc.keep, -uc.step * x[4 * q + 2]);
          w.w = fmaf(w.w, uc.keep, -uc.step * x[4 * q + 3]);
          *pw = w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          float* pw = reinterpret_cast<float*>(Ws + sw128_f32(e, lane));
          *pw = fmaf(*pw, uc.keep, -uc.step * x[e]);
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

// -------------------------------------------------------------- per-tile roles

// A and B are stored as their lower triangle of 256-row blocks only (the
// Gram and Poly tiles with J <= I, diagonal blocks in full). A K block of a
// symmetric operand's row block `blk` at or below the diagonal (k0 / 256 <=
// blk) is read K-major from the stored rows; one above it is read from its
// transposed position, block (k0 / 256, blk), as an MN-major operand: the
// same values, since the matrix is symmetric.
__device__ __forceinline__ bool sym_mn(int k0, int blk) { return k0 / kPairTile > blk; }

// One CTA's half (rows blk * 256 + rank * 128 ..) of a symmetric operand's K block k0.
__device__ __forceinline__ void load_sym_half(uint8_t* dst, const void* tm_k, const void* tm_mn,
                                              uint32_t bar, int blk, int k0, uint32_t rank, int bz) {
  const int row = blk * kPairTile + static_cast<int>(rank) * kHalf;
  if (sym_mn(k0, blk)) {
#pragma unroll
    for (int q = 0; q < kHalf / 64; ++q)
      ptx::tma_load_3d_pair(dst + q * (64 * kBK * 2), tm_mn, bar, row + q * 64, k0, bz);
  } else {
    ptx::tma_load_3d_pair(dst, tm_k, bar, k0, row, bz);
  }
}

// Producer (one thread per CTA): the operand loads of one tile into the ring.
// Returns false when a wait gives up (the caller aborts the pair).
template <int KIND, int STAGES>
__device__ __forceinline__ bool produce_tile(const StageArgs& a, const Smem& s, const TileCoord& tc,
                                             int xsrc, uint32_t rank, const uint32_t* leader_full,
                                             uint32_t& stage, uint32_t& phase, uint64_t limit) {
  using K = KindT<KIND>;
  const int bz = static_cast<int>(tc.b);
  for (int kb = 0; kb < tc.kblocks; ++kb) {
    if (!ptx::mbar_wait(&s.empty[stage], phase ^ 1, limit, s.abort_flag)) return false;
    uint8_t* sa = s.ring + stage * kStageBytes;
    uint8_t* sb = sa + kABytes;
    const bool diag = !K::kApplyLike && tc.I == tc.J;
    if (rank == 0) ptx::mbar_arrive_expect_tx(&s.full[stage], diag ? kPairTx / 2 : kPairTx);
    const int k0 = kb * kBK;
    if (K::kApplyLike) {
      // B (symmetric) rows I, then the iterate's column block J (MN-major)
      load_sym_half(sa, tmap(a, tc.g, kTmB), tmap(a, tc.g, kTmBMN), leader_full[stage], tc.I, k0, rank, bz);
      const void* tx = tmap(a, tc.g, xsrc ? kTmXb1MN : kTmXb0MN);
#pragma unroll
      for (int q = 0; q < kHalf / 64; ++q)
        ptx::tma_load_3d_pair(sb + q * (64 * kBK * 2), tx, leader_full[stage],
                              tc.J * kPairTile + rank * kHalf + q * 64, k0, bz);
    } else if (KIND == kGram) {
      const void* tm = tmap(a, tc.g, xsrc ? kTmXb1K : kTmXb0K);
      ptx::tma_load_3d_pair(sa, tm, leader_full[stage], k0, tc.I * kPairTile + rank * kHalf, bz);
      // on a diagonal tile each CTA's right-operand half is its left-operand rows
      if (tc.I != tc.J)
        ptx::tma_load_3d_pair(sb, tm, leader_full[stage], k0, tc.J * kPairTile + rank * kHalf, bz);
    } else {
      // Poly: A (symmetric) rows I and rows J
      const void* tk = tmap(a, tc.g, kTmA);
      const void* tmn = tmap(a, tc.g, kTmAMN);
      load_sym_half(sa, tk, tmn, leader_full[stage], tc.I, k0, rank, bz);
      if (tc.I != tc.J) load_sym_half(sb, tk, tmn, leader_full[stage], tc.J, k0, rank, bz);
    }
    if (++stage == STAGES) {
      stage = 0;
      phase ^= 1;
    }
  }
  return true;
}

// MMA issuer (pair leader, one thread): one tile into accumulator `acc`.
template <int KIND, int STAGES>
__device__ __forceinline__ bool mma_tile(const Smem& s, const TileCoord& tc, uint32_t tmem_base,
                                         uint32_t& stage, uint32_t& phase, uint32_t& acc,
                                         uint32_t& acc_phase, bool& issued, uint64_t limit) {
  using K = KindT<KIND>;
  if (!ptx::mbar_wait(&s.tempty[acc], acc_phase ^ 1, limit, s.abort_flag)) return false;
  ptx::tc_fence_after();
  const uint32_t d = tmem_base + acc * kPairTile;
  for (int kb = 0; kb < tc.kblocks; ++kb) {
    if (!ptx::mbar_wait(&s.full[stage], phase, limit, s.abort_flag)) return false;
    ptx::tc_fence_after();
    const uint32_t sa = ptx::smem_u32(s.ring + stage * kStageBytes);
    const uint32_t sb = (!K::kApplyLike && tc.I == tc.J) ? sa : sa + kABytes;
    // major-ness of each side for this K block (Gram: X, always K-major;
    // Poly: A both sides; Apply: B, then the iterate MN-major)
    const int k0 = kb * kBK;
    const bool a_mn = KIND != kGram && sym_mn(k0, tc.I);
    const bool b_mn = K::kApplyLike || (KIND == kPoly && sym_mn(k0, tc.J));
    const uint32_t idesc = idesc_of(a_mn, b_mn);
#pragma unroll
    for (int k = 0; k < kBK / 16; ++k) {
      const uint64_t ad = a_mn ? ptx::desc_sw128(sa + k * 16 * 128, 64 * kBK * 2, 1024)
                               : ptx::desc_sw128(sa + k * 32, 16, 1024);
      const uint64_t bd = b_mn ? ptx::desc_sw128(sb + k * 16 * 128, 64 * kBK * 2, 1024)
                               : ptx::desc_sw128(sb + k * 32, 16, 1024);
      ptx::umma_bf16_pair(d, ad, bd, idesc, (kb | k) != 0);
    }
    issued = true;
    ptx::umma_commit_pair(&s.empty[stage]);
    if (++stage == STAGES) {
      stage = 0;
      phase ^= 1;
    }
  }
  ptx::umma_commit_pair(&s.tfull[acc]);
  if (++acc == 2) {
    acc = 0;
    acc_phase ^= 1;
  }
  return true;
}

// State an epilogue warp carries from tile to tile.
struct EpiState {
  uint32_t acc = 0, acc_phase = 0;
  uint32_t eload_phase = 0;  // bit i: phase of slot i's load barrier
};

// Epilogue warp: one tile. With `dep` set (chained launch) the warp first
// waits until the tile's inputs have landed (counter >= need) and, once its
// own stores have landed, adds one to the matrix's counter. Returns false
// when a wait gives up (the pair has been aborted).
template <int KIND, typename L>
__device__ __forceinline__ bool epilogue_tile(const StageArgs& a, const StepP& p, const Smem& s,
                                              const TileCoord& tc, int64_t t_apply, uint32_t rank,
                                              int ew, int warp, int lane, uint32_t tmem_base,
                                              EpiState& es, const uint32_t* leader_tempty,
                                              uint64_t limit, unsigned* dep, uint32_t need) {
  using K = KindT<KIND>;
  const int quarter = warp & 3;  // TMEM lanes this warp may read: 32 * quarter ...
  const int ch_begin = (ew / 4) * L::kChunksPerWarp;  // this warp's share of the columns
  const int ch_end = ch_begin + L::kChunksPerWarp;
  constexpr int S = L::kEpiSlots;
  uint8_t* slots = s.epi + ew * S * L::kSlot;
  uint64_t* eload = s.eload + S * ew;
  constexpr bool kInput = K::kInput;
  // input loads in flight ahead of the current chunk: with three or more
  // slots the newest chunk's stores may still be reading their slot when the
  // next load is issued (no wait on them); with two they must have finished
  constexpr int D = !kInput ? 0 : (S >= 3 ? S - 2 : S - 1);
  constexpr int kReuseWait = S - 1 - D;  // store groups that may still be pending
  const GroupDesc& gd = a.groups[tc.g];
  const int row0 = tc.I * kPairTile + static_cast<int>(rank) * kHalf + quarter * 32;
  const int bz = static_cast<int>(tc.b);
  const int mat = gd.first_mat + bz;
  // Apply-like: the current iterate's high part (the operand buffer) and low part
  const void* in_map = tmap(a, tc.g, K::kApplyLike ? (p.xsrc ? kTmXb1E : kTmXb0E) : kTmAE);
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
  const int limit_c = K::kApplyLike ? gd.c : gd.r;
  // rows or columns past the matrix: nothing to load or store for a chunk
  auto live_chunk = [&](int ch) {
    return ch < ch_end && row0 < gd.r && tc.J * kPairTile + ch * 32 < limit_c;
  };
  auto issue_load = [&](int ch) {  // the caller has made sure the slot is free
    const int sl = (ch - ch_begin) % S;
    uint8_t* slot = slots + sl * L::kSlot;
    uint64_t* bar = &eload[sl];
    const int col0 = tc.J * kPairTile + ch * 32;
    ptx::mbar_arrive_expect_tx(bar, in_bytes);
    ptx::tma_load_3d(slot, in_map, bar, col0, row0, bz);
    if (K::kApplyLike) ptx::tma_load_3d(slot + kOffLow, tmap(a, tc.g, kTmXloE), bar, col0, row0, bz);
    if (KIND == kApplyLast && w_in)
      ptx::tma_load_3d(slot + kOffLastW, mat_tmap(a, mat, kMtW), bar, w_tr ? row0 : col0,
                       w_tr ? col0 : row0, 0);
  };
  bool ok = true;
  if (kInput && lane == 0) {
    // chained launch: the inputs come from this matrix's earlier stages
    if (dep != nullptr && !ptx::dep_wait(dep + mat, need, a.err, limit, s.abort_flag)) {
      raise_abort(a, s);
      ok = false;
    }
    if (ok) {
      // the previous tile's stores have read every slot: fill them all, so
      // that the first chunks' inputs travel while the accumulator is awaited
      ptx::bulk_wait_read<0>();
      for (int ch = ch_begin; ch < ch_begin + S; ++ch)
        if (live_chunk(ch)) issue_load(ch);
    }
  }
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (!ok) return false;
  if (!ptx::mbar_wait(&s.tfull[es.acc], es.acc_phase, limit, s.abort_flag)) {
    raise_abort(a, s);
    return false;
  }
  ptx::tc_fence_after();
  const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + es.acc * kPairTile;
#pragma unroll 1
  for (int ch = ch_begin; ch < ch_end; ++ch) {
    const int sl = (ch - ch_begin) % S;
    uint8_t* slot = slots + sl * L::kSlot;
    const int col0 = tc.J * kPairTile + ch * 32;
    const bool live = live_chunk(ch);
    if (lane == 0) {
      // the load D chunks ahead reuses the slot of chunk ch + D - S, whose
      // stores are older than the newest kReuseWait groups
      if (kInput && ch + D >= ch_begin + S && live_chunk(ch + D)) {
        ptx::bulk_wait_read<kReuseWait>();
        issue_load(ch + D);
      }
      if (!kInput) ptx::bulk_wait_read<1>();  // two slots: chunk ch - 2's stores have read it
    }
    __syncwarp();
    float v[32];
    ptx::tmem_ld32(taddr + ch * 32, v);
    if (kInput && live) {
      if (!ptx::mbar_wait(&eload[sl], (es.eload_phase >> sl) & 1u, limit, s.abort_flag)) {
        raise_abort(a, s);
        return false;
      }
      es.eload_phase ^= 1u << sl;
    }
    if (live) {
      if (KIND == kApply) {
        epi_apply(a, p, gd, tc, row0, col0, slot, v, lane, ssq);
      } else if (KIND == kApplyLast) {
        epi_apply_last(a, p, gd, tc, row0, col0, slot, v, lane, ssq);
      } else {
        epi_symmetric<KIND>(a, p, gd, tc, row0, col0, slot, v, lane);
      }
    }
    // one bulk group per chunk (possibly empty), so "all but the newest
    // group" always means "every chunk before the previous one"
    __syncwarp();
    if (lane == 0) ptx::bulk_commit();
  }
  if (K::kApplyLike && p.record) {
    // one slot per (tile, CTA of the pair, epilogue warp); every slot is written
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
    // kSumsqSlots per CTA and tile; a kind with fewer epilogue warps zeroes the rest
    if (lane == 0) {
      float* dst = a.sumsq + (t_apply * 2 + rank) * kSumsqSlots;
      dst[ew] = ssq;
      for (int e = ew + L::kEpiWarps; e < kSumsqSlots; e += L::kEpiWarps) dst[e] = 0.f;
    }
  }
  ptx::tc_fence_before();
  __syncwarp();
  if (lane == 0) ptx::mbar_arrive_cluster(leader_tempty[es.acc]);
  if (++es.acc == 2) {
    es.acc = 0;
    es.acc_phase ^= 1;
  }
  if (dep != nullptr && lane == 0) {
    // this warp's share of the tile is in global memory: count it
    ptx::bulk_wait<0>();
    ptx::fence_proxy_async_global();
    ptx::red_release_gpu_add(dep + mat, 1u);
  }
  __syncwarp();
  return true;
}

// -------------------------------------------------------------- kernels

// Barrier set-up and TMEM allocation shared by both kernels.
template <typename L>
__device__ __forceinline__ uint32_t prologue(const Smem& s, int warp) {
  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kStages; ++i) {
      ptx::mbar_init(&s.full[i], 1);
      ptx::mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&s.tfull[i], 1);
      ptx::mbar_init(&s.tempty[i], 2 * L::kEpiWarps);
    }
    ptx::mbar_init(s.drain, 1);
    for (int i = 0; i < L::kEpiSlots * L::kEpiWarps; ++i) ptx::mbar_init(&s.eload[i], 1);
    // chained launch's tile queue: published by the leader's producer; read by
    // the leader's MMA warp, the peer's producer and both CTAs' epilogue warps
    for (int i = 0; i < kTileQ; ++i) {
      ptx::mbar_init(&s.tq_full[i], 1);
      ptx::mbar_init(&s.tq_empty[i], 2 + 2 * L::kEpiWarps);
    }
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
  return *s.tmem_slot;
}

__device__ __forceinline__ void teardown(int warp, uint32_t tmem_base) {
  __syncwarp();
  ptx::tc_fence_before();
  ptx::cluster_sync();  // neither CTA leaves while its partner may still use its memory
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// Give copies already issued time to land before the pair exits.
__device__ __forceinline__ void linger() {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (ptx::globaltimer_ns() - t0 < 20000) {
  }
}

// Let the MMAs in flight finish before TMEM is released.
__device__ __forceinline__ void drain_mma(const Smem& s, uint64_t limit) {
  volatile int never = 0;
  ptx::umma_commit_pair_self(s.drain);
  ptx::mbar_wait(s.drain, 0, limit, &never);
}

template <typename L>
__device__ __forceinline__ void load_tmaps_and_full(const StageArgs& a, const Smem& s, uint32_t* leader_full) {
  for (int g = 0; g < a.ngroups; ++g)
    for (int k = 0; k < kTmPerGroup; ++k) {
      ptx::fence_tmap_acquire(tmap(a, g, k));
      ptx::prefetch_tmap(tmap(a, g, k));
    }
  for (int i = 0; i < L::kStages; ++i) leader_full[i] = ptx::mapa_shared(ptx::smem_u32(&s.full[i]), 0);
}

template <int KIND, bool WIDE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(StageLayout<KIND, WIDE>::L::kThreads, 1)
    stage_tc_kernel(const __grid_constant__ StageArgs a) {
  using L = typename StageLayout<KIND, WIDE>::L;
  extern __shared__ uint8_t smem_raw[];
  const Smem s = carve<L>(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const int64_t pair = blockIdx.x >> 1;
  const int64_t npairs = gridDim.x >> 1;
  const uint64_t limit = a.wait_limit_ns;
  const uint32_t tmem_base = prologue<L>(s, warp);
  const StepP p = step_of(a);

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- producer
    uint32_t leader_full[L::kStages];
    load_tmaps_and_full<L>(a, s, leader_full);
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    for (int64_t t = a.tile_begin + pair; ok && t < a.total_tiles; t += npairs) {
      const TileCoord tc = decode_tile<KIND>(a, t);
      if (!produce_tile<KIND, L::kStages>(a, s, tc, p.xsrc, rank, leader_full, stage, phase, limit)) {
        raise_abort(a, s);
        ok = false;
      }
    }
    if (!ok) linger();
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ---------------------------------------------------------- MMA issuer (pair leader)
    uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
    bool issued = false;
    for (int64_t t = a.tile_begin + pair; t < a.total_tiles; t += npairs) {
      const TileCoord tc = decode_tile<KIND>(a, t);
      if (!mma_tile<KIND, L::kStages>(s, tc, tmem_base, stage, phase, acc, acc_phase, issued, limit)) {
        raise_abort(a, s);
        if (issued) drain_mma(s, limit);
        break;
      }
    }
  } else if (warp >= 2) {
    // ---------------------------------------------------------- epilogue
    const int ew = warp - 2;
    uint32_t leader_tempty[2];
    for (int i = 0; i < 2; ++i) leader_tempty[i] = ptx::mapa_shared(ptx::smem_u32(&s.tempty[i]), 0);
    EpiState es;
    bool ok = true;
    for (int64_t t = a.tile_begin + pair; ok && t < a.total_tiles; t += npairs) {
      const TileCoord tc = decode_tile<KIND>(a, t);
      ok = epilogue_tile<KIND, L>(a, p, s, tc, t, rank, ew, warp, lane, tmem_base, es, leader_tempty,
                                  limit, nullptr, 0u);
    }
    if (lane == 0) ptx::bulk_wait<0>();
    if (!ok) linger();
    __syncwarp();
  }
  teardown(warp, tmem_base);
}

// The chained launch's tile queue. The pair leader's producer takes the next
// tile index from the global counter and publishes it to both CTAs; every
// other role of the pair takes the indices from its CTA's queue in the same
// order. An index at or past the end of the list ends every role's loop.
struct TileQueue {
  uint32_t slot = 0, phase = 0;
  __device__ void advance() {
    if (++slot == kTileQ) {
      slot = 0;
      phase ^= 1;
    }
  }
};

// Leader producer: fetch, then publish to both CTAs (the queue entry must
// have been read by all consumers of its previous use).
__device__ __forceinline__ bool tq_publish(const StageArgs& a, const Smem& s, TileQueue& q, uint64_t limit,
                                           uint32_t& t) {
  t = atomicAdd(a.next_tile, 1u);
  if (!ptx::mbar_wait_cluster(&s.tq_empty[q.slot], q.phase ^ 1, limit, s.abort_flag)) return false;
  const uint32_t entry = ptx::smem_u32(const_cast<uint32_t*>(s.tq + q.slot));
  const uint32_t full = ptx::smem_u32(&s.tq_full[q.slot]);
  for (uint32_t r = 0; r < 2; ++r) {
    ptx::st_cluster_u32(ptx::mapa_shared(entry, r), t);
    ptx::mbar_arrive_release_cluster(ptx::mapa_shared(full, r));
  }
  q.advance();
  return true;
}

// Any other role: the next published index of this CTA's queue.
__device__ __forceinline__ bool tq_take(const Smem& s, TileQueue& q, uint64_t limit, uint32_t& t) {
  if (!ptx::mbar_wait_cluster(&s.tq_full[q.slot], q.phase, limit, s.abort_flag)) return false;
  t = s.tq[q.slot];
  ptx::mbar_arrive_release_cluster(ptx::mapa_shared(ptx::smem_u32(&s.tq_empty[q.slot]), 0));
  q.advance();
  return true;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(ChainL::kThreads, 1)
    stage_chain_kernel(const __grid_constant__ StageArgs a) {
  using L = ChainL;
  extern __shared__ uint8_t smem_raw[];
  const Smem s = carve<L>(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const uint64_t limit = a.wait_limit_ns;
  const uint32_t total = static_cast<uint32_t>(a.total_tiles);
  const uint32_t tmem_base = prologue<L>(s, warp);

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- producer
    uint32_t leader_full[L::kStages];
    load_tmaps_and_full<L>(a, s, leader_full);
    uint32_t stage = 0, phase = 0;
    TileQueue q;
    bool ok = true;
    for (;;) {
      uint32_t t = 0;
      if (!(rank == 0 ? tq_publish(a, s, q, limit, t) : tq_take(s, q, limit, t))) {
        raise_abort(a, s);
        ok = false;
        break;
      }
      if (t >= total) break;
      const ChainTile ct = a.chain[t];
      if (ct.stage >= a.chain_stages) continue;  // skipped by every role of the pair
      const ChainPos cp = chain_pos(a, ct);
      const int xsrc = cp.step & 1;
      // every tile of the matrix's earlier stages has finished
      if (!ptx::dep_wait(a.dep + ct.mat, cp.need, a.err, limit, s.abort_flag)) {
        raise_abort(a, s);
        ok = false;
        break;
      }
      bool r;
      if (cp.kind == kGram) r = produce_tile<kGram, L::kStages>(a, s, cp.tc, xsrc, rank, leader_full, stage, phase, limit);
      else if (cp.kind == kPoly) r = produce_tile<kPoly, L::kStages>(a, s, cp.tc, xsrc, rank, leader_full, stage, phase, limit);
      else r = produce_tile<kApply, L::kStages>(a, s, cp.tc, xsrc, rank, leader_full, stage, phase, limit);
      if (!r) {
        raise_abort(a, s);
        ok = false;
        break;
      }
    }
    if (!ok) linger();
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ---------------------------------------------------------- MMA issuer (pair leader)
    uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
    bool issued = false;
    TileQueue q;
    for (;;) {
      uint32_t t = 0;
      bool r = tq_take(s, q, limit, t);
      if (r && t >= total) break;
      if (r) {
        const ChainTile ct = a.chain[t];
        if (ct.stage >= a.chain_stages) continue;
        const ChainPos cp = chain_pos(a, ct);
        if (cp.kind == kApply) r = mma_tile<kApply, L::kStages>(s, cp.tc, tmem_base, stage, phase, acc, acc_phase, issued, limit);
        else if (cp.kind == kPoly) r = mma_tile<kPoly, L::kStages>(s, cp.tc, tmem_base, stage, phase, acc, acc_phase, issued, limit);
        else r = mma_tile<kGram, L::kStages>(s, cp.tc, tmem_base, stage, phase, acc, acc_phase, issued, limit);
      }
      if (!r) {
        raise_abort(a, s);
        if (issued) drain_mma(s, limit);
        break;
      }
    }
  } else if (warp >= 2) {
    // ---------------------------------------------------------- epilogue
    const int ew = warp - 2;
    uint32_t leader_tempty[2];
    for (int i = 0; i < 2; ++i) leader_tempty[i] = ptx::mapa_shared(ptx::smem_u32(&s.tempty[i]), 0);
    EpiState es;
    TileQueue q;
    bool ok = true;
    for (;;) {
      uint32_t t = 0;
      int took = 1;
      if (lane == 0) took = tq_take(s, q, limit, t) ? 1 : 0;
      else q.advance();  // every lane follows the queue position (lane 0 reads it)
      took = __shfl_sync(0xffffffffu, took, 0);
      t = __shfl_sync(0xffffffffu, t, 0);
      if (!took) {
        if (lane == 0) raise_abort(a, s);
        ok = false;
        break;
      }
      if (t >= total) break;
      const ChainTile ct = a.chain[t];
      if (ct.stage >= a.chain_stages) continue;
      const ChainPos cp = chain_pos(a, ct);
      const StepP p = chain_step(a, ct, cp.step);
      if (cp.kind == kGram)
        ok = epilogue_tile<kGram, L>(a, p, s, cp.tc, cp.t_apply, rank, ew, warp, lane, tmem_base, es,
                                     leader_tempty, limit, a.dep, cp.need);
      else if (cp.kind == kPoly)
        ok = epilogue_tile<kPoly, L>(a, p, s, cp.tc, cp.t_apply, rank, ew, warp, lane, tmem_base, es,
                                     leader_tempty, limit, a.dep, cp.need);
      else
        ok = epilogue_tile<kApply, L>(a, p, s, cp.tc, cp.t_apply, rank, ew, warp, lane, tmem_base, es,
                                      leader_tempty, limit, a.dep, cp.need);
      if (!ok) break;
    }
    if (lane == 0) ptx::bulk_wait<0>();
    if (!ok) linger();
    __syncwarp();
  }
  teardown(warp, tmem_base);
}

template <int KIND, bool WIDE>
cudaError_t launch_kind(const StageArgs& args, int grid, cudaStream_t stream) {
  using L = typename StageLayout<KIND, WIDE>::L;
  constexpr size_t smem = L::kSmem;
  static_assert(smem <= 227 * 1024, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(stage_tc_kernel<KIND, WIDE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  stage_tc_kernel<KIND, WIDE><<<grid, L::kThreads, smem, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace

size_t stage_tc_smem_bytes() { return StageLayout<kGram, false>::L::kSmem; }

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

cudaError_t chain_max_pairs(int* pairs) {
  constexpr size_t smem = ChainL::kSmem;
  cudaError_t e = cudaFuncSetAttribute(stage_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(ChainL::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr{};
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  e = cudaOccupancyMaxActiveClusters(&clusters, stage_chain_kernel, &cfg);
  if (e != cudaSuccess) return e;
  *pairs = clusters;
  return cudaSuccess;
}

cudaError_t launch_stage_chain(const StageArgs& args, int grid, cudaStream_t stream) {
  if (args.total_tiles <= args.tile_begin) return cudaSuccess;
  if (grid < 2 || (grid & 1)) return cudaErrorInvalidConfiguration;
  constexpr size_t smem = ChainL::kSmem;
  cudaError_t e = cudaFuncSetAttribute(stage_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  stage_chain_kernel<<<grid, ChainL::kThreads, smem, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace muon
