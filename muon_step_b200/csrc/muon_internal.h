// Internal descriptor tables shared by the host planner and the device kernels.
//
// A Muon step (or an ns_orthogonalize call) over many matrices is planned once
// on the host: matrices are grouped by their Newton-Schulz shape (r, c) with
// r = min(n, m) <= c = max(n, m); each group's working buffers sit in one
// contiguous slab of the caller's workspace so that one 3-D TMA tensor map per
// buffer covers the whole group. Tile counts per stage kind are prefix-summed
// over the groups so that a single persistent launch per stage walks every
// matrix's tiles.
#pragma once

#include <cstdint>

namespace muon {

constexpr int kMaxGroups = 64;
constexpr int kMaxSteps = 64;

// tcgen05 tiles: 256 x 256 output tiles per CTA pair, K blocks of 64 bf16 (128 B).
constexpr int kPairM = 256;
constexpr int kPairN = 256;
constexpr int kBK = 64;

// Matrices with min(n, m) <= kSmallMax and max(n, m) <= kSmallMax run the
// whole Newton-Schulz iteration in one CTA (bf16 precision).
constexpr int kSmallMax = 128;
// Matrices with min(n, m) <= kSmallMax < max(n, m) <= kMidMaxC run the whole
// iteration in one 512-thread CTA with the iterate in shared memory.
constexpr int kMidMaxC = 512;
// In the bf16 precision, matrices of at most kTinyMaxElems elements run the
// whole iteration with fp32 operands in one CTA (too few elements for bf16
// operand rounding to average out over the Frobenius norm).
constexpr int kTinyMaxElems = 4096;

// fp32 validation tile shape.
constexpr int kSBM = 64;
constexpr int kSBN = 64;
constexpr int kSBK = 16;

// elementwise (momentum / norm / cast) tile: 64 rows x 128 columns. 64 rows
// make the transposed writes of the bf16 iterate parts whole 128-byte lines
// (two caller rows per lane).
constexpr int kEwRows = 64;
constexpr int kEwCols = 128;

enum StageKind : int { kGram = 0, kPoly = 1, kApply = 2, kNumKinds = 3 };

// MatDesc.flags
enum MatFlags : int { kMatWTma = 1, kMatOTma = 2 };
// per-matrix tensor maps: fp32 {32, 32} boxes, 128-byte swizzle, over the caller's W and O
enum MatTmapSlot : int { kMtW = 0, kMtO = 1, kMtPerMat = 2 };

// tensor maps per group (bf16 mode)
enum TmapSlot : int {
  kTmXb0K = 0,   // X bf16 buffer 0, box {64 cols, 128 rows}: K-major operand
  kTmXb1K = 1,   // X bf16 buffer 1
  kTmXb0MN = 2,  // X bf16 buffer 0, box {64 cols, 64 rows}: MN-major operand
  kTmXb1MN = 3,  // X bf16 buffer 1
  kTmA = 4,      // Gram matrix A, box {64, 128}
  kTmB = 5,      // polynomial B = bA + cA^2, box {64, 128}
  // epilogue maps, box {32, 32}: loads and stores of one warp's 32 x 32 chunk
  kTmXloE = 6,   // bf16 low part of the iterate, 64-byte swizzle
  kTmXb0E = 7,   // bf16 iterate buffer 0, 64-byte swizzle
  kTmXb1E = 8,   // bf16 iterate buffer 1, 64-byte swizzle
  kTmAE = 9,     // A, 64-byte swizzle
  kTmBE = 10,    // B, 64-byte swizzle
  kTmAMN = 11,   // A, box {64, 64}: MN-major operand (a K block above the diagonal, read transposed)
  kTmBMN = 12,   // B, box {64, 64}
  kTmPerGroup = 13
};

struct GroupDesc {
  int32_t r, c;          // Newton-Schulz shape, r <= c
  int32_t ldc, ldr;      // leading dimensions (elements) of r x c and r x r buffers
  int32_t count;         // matrices in this group
  int32_t first_mat;     // internal index of the group's first matrix
  int32_t small;         // 1: small-matrix kernel, 2: mid-size kernel, 3: tiny fp32 kernel
                         // (no stage tiles for any of them)
  int32_t pad0;
  int64_t xf_off[2];     // byte offsets in the workspace: fp32 iterate, ping-pong (fp32 mode)
  int64_t xb_off[2];     // bf16 iterate (bf16 mode: its high part, the MMA operand), ping-pong
  int64_t xlo_off;       // bf16 mode: low part, iterate = high + low (updated in place)
  int64_t a_off, b_off;  // A = X X^T and B = bA + cA^2 (bf16, or fp32 in fp32 mode)
  int64_t tiles_per_mat[kNumKinds];
  int64_t tile_base[kNumKinds];
  int64_t tile_flops[kNumKinds];  // useful FLOPs per matrix per stage (host statistics)
};

struct MatDesc {
  float* W;              // caller's weight (n x m, row-major), updated in place
  const float* G;        // caller's gradient, or the ns_orthogonalize input X
  float* M;              // caller's momentum buffer (NULL for ns_orthogonalize)
  float* O;              // optional output O' in the caller's orientation
  int64_t n, m;          // caller's shape
  int32_t transposed;    // Newton-Schulz runs on the transpose (n > m)
  int32_t group;         // shape group
  int32_t index;         // index within the group
  int32_t flags;         // kMatWTma / kMatOTma: W / O reachable by TMA (16-byte rows)
  int32_t caller;        // position in the caller's list (diagnostics output)
  int32_t pad1;
  int64_t ew_tile_begin; // first elementwise tile of this matrix
  int64_t ew_tiles;      // number of elementwise tiles
};

// One tile of the chained launch's list: stage = 3 * step + kind (Gram 0,
// Poly 1, Apply 2), tile = index within the matrix's table of that kind.
struct ChainTile {
  int32_t mat;    // internal matrix index
  int32_t stage;
  int32_t tile;
  int32_t pad;
};

// Epilogue warps per tile of the chained launch (8 per CTA, two CTAs): each
// adds one to its matrix's dependency counter when its stores have landed.
constexpr int kChainArrivals = 16;

// Per-launch arguments of the Newton-Schulz stage kernels.
struct StageArgs {
  const GroupDesc* groups;
  const MatDesc* mats;
  const void* tmaps;      // CUtensorMap[ngroups][kTmPerGroup], 64-byte aligned
  const void* mat_tmaps;  // CUtensorMap[nmats][kMtPerMat] (W / O of the last step)
  char* ws;               // workspace base
  const float* scale;     // per-matrix 1 / (||N||_F + eps)
  int* err;               // device error word
  int64_t tile_begin;     // this launch walks tiles [tile_begin, total_tiles) of the kind's table
  int64_t total_tiles;
  int32_t ngroups;
  int32_t first;          // first Newton-Schulz step: fold the normalisation scale
  int32_t last;           // last step: write O' and update W instead of the iterate
  int32_t xsrc;           // which ping-pong buffer holds the current iterate
  float a, b, c;          // this step's coefficients
  float lr, wd, gamma;    // update hyper-parameters (last step)
  int32_t scale_mode;     // muon_scale_mode_t of the update
  int32_t sumsq_per_tile; // > 0: the last step records sums of squares of X' (per tile slots)
  float* sumsq;           // ... into sumsq[tile * sumsq_per_tile + slot]
  uint64_t wait_limit_ns; // bound on every spin-wait
  // chained launch: every Gram / Poly / Apply stage of the schedule in one
  // persistent kernel, tiles taken in the order of a host-built list
  const ChainTile* chain; // [total_tiles]
  unsigned* dep;          // per matrix: epilogue-warp tile completions so far this execute
  unsigned* next_tile;    // the list index the next CTA pair to ask takes (zero at launch)
  int32_t chain_sumsq_stage;  // stage whose Apply records sums of squares (-1: none)
  int32_t chain_stages;       // tiles of later stages in the list are skipped
  float abc[kMaxSteps * 3];   // every step's coefficients
};

// Elementwise-stage arguments (momentum + Nesterov + Frobenius partials + cast).
struct EwArgs {
  const GroupDesc* groups;
  const MatDesc* mats;
  char* ws;
  const int32_t* tile_mat;  // matrix of each elementwise tile
  float* partial;         // one partial sum of squares per elementwise tile
  unsigned* counter;      // per-matrix arrival counter (left at zero)
  float* scale;           // per-matrix output 1 / (||N||_F + eps)
  int* err;
  int64_t total_tiles;
  int32_t nmats;
  int32_t mode;           // 0: Muon (momentum + Nesterov), 1: plain normalisation of G
  int32_t nesterov;
  int32_t split;          // bf16 mode: the iterate as bf16 high + low parts (else fp32)
  float mu, eps;
  float* diag;            // optional: diag[2 caller] = ||N||_F
  unsigned* dep;          // optional: chained-launch dependency counters, reset per matrix
  unsigned* next_tile;    // optional: chained-launch tile counter, reset by the first CTA
};

// Small-matrix kernel arguments (one CTA per matrix, every step on chip).
struct SmallArgs {
  const GroupDesc* groups;
  const MatDesc* mats;
  const void* tmaps;      // group tensor maps (the bf16 iterate, K-major box)
  char* ws;
  const float* scale;
  const int32_t* small_mats;  // internal indices of the small matrices
  int* err;
  int64_t nsmall;
  int32_t steps;
  float lr, wd, gamma;    // update hyper-parameters
  int32_t scale_mode;     // muon_scale_mode_t of the update
  uint64_t wait_limit_ns;
  float* diag;            // optional: diag[2 caller + 1] = RMS of the applied update O
  int32_t mode;           // tiny kernel: 0 Muon step (N from M_t and G), 1 ns_orthogonalize (N = G)
  int32_t nesterov;       // tiny kernel: N = mu M_t + G (else N = M_t)
  float mu;               // tiny kernel: momentum coefficient
  float abc[kMaxSteps * 3];
};

// Update pass of the unit-RMS scale mode (matrices on the grouped or fp32
// path): W <- W keep - lr factor[mat] O', O' read from the iterate buffers.
struct FinishArgs {
  const GroupDesc* groups;
  const MatDesc* mats;
  const int32_t* tile_mat;  // elementwise tiling of the caller matrices
  char* ws;
  const float* sumsq;       // per-tile slots of sum of squares of O'
  float* factor;            // per matrix gamma / RMS(O') (0 when O' = 0)
  int64_t total_tiles;      // elementwise tiles
  int32_t nmats;
  int32_t xf_slot;          // which iterate buffer holds O' (fp32, or the bf16 high part)
  int32_t split;            // bf16 mode: O' = high + low parts
  int32_t sumsq_per_tile;
  int32_t apply_kind;       // tile table the sums were recorded on
  int32_t scale_mode;       // muon_scale_mode_t of the update
  float lr, wd, gamma;
  float* diag;              // optional: diag[2 caller + 1] = RMS of the applied update O
};

// Element offset of iterate element (row, col) in a matrix's bf16 low-part
// buffer (r x ldc elements). Row-major, except for the mid-size kernel's
// matrices (GroupDesc.small == 2), whose low part is stored as 8-column
// groups, [col / 8][row][col % 8], so that the threads that own consecutive
// rows read and write one contiguous 16-byte piece each.
__host__ __device__ __forceinline__ int64_t lo_index(int small, int r, int64_t ldc, int64_t row,
                                                     int64_t col) {
  return small == 2 ? ((col >> 3) * r + row) * 8 + (col & 7) : row * ldc + col;
}

// error bits in the device error word
enum ErrBits : int { kErrTimeout = 1, kErrBadTile = 2 };

}  // namespace muon
