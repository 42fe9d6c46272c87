// Host planner and C ABI (include/muon_step.h).
//
// Planning groups matrices by Newton-Schulz shape (r, c) = (min, max), lays
// the per-group working buffers out in the caller's workspace, enumerates the
// tiles of every stage, and keeps a host image of the descriptor tables. An
// execute copies that image into the workspace the first time it sees the
// workspace pointer (TMA tensor maps are encoded then, since they embed the
// buffers' addresses), and then launches 1 + 3 * steps kernels.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <new>
#include <utility>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "kernels.cuh"
#include "muon_step.h"
#include "ptx_sm100.cuh"

using namespace muon;

namespace {

__device__ int g_device_error;  // per device: error bits of the library's kernels

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
int* g_err_ptr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};
int g_cc_major[kMaxDevices] = {};
int g_chain_pairs[kMaxDevices] = {};  // CTA pairs of the chained launch resident at once
std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};  // set from any host thread

// Per-device setup: the error word's device address and the SM count.
muon_status_t device_setup(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MUON_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_err_ptr[dev]) {
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MUON_ERR_CUDA;
    g_cc_major[dev] = major;
    g_num_sms[dev] = sms;
    if (major == 10) {
      int pairs = 0;
      if (chain_max_pairs(&pairs) != cudaSuccess) return MUON_ERR_CUDA;
      g_chain_pairs[dev] = pairs;
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return MUON_ERR_CUDA;
    g_err_ptr[dev] = static_cast<int*>(p);
  }
  if (g_cc_major[dev] != 10) return MUON_ERR_UNSUPPORTED;
  *dev_out = dev;
  return MUON_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D tensor map over a group's [count][rows][ld] buffer, box {box0, box1, 1},
// zero fill outside [inner, rows, count] on loads, clipping on stores.
bool encode_3d(CUtensorMap* out, void* base, CUtensorMapDataType dtype, int elem_bytes, int64_t inner,
               int64_t rows, int64_t ld, int64_t count, int box0, int box1,
               CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(count)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld * elem_bytes),
                           static_cast<cuuint64_t>(rows * ld * elem_bytes)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box0), static_cast<cuuint32_t>(box1), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(out, dtype, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_bf16_3d(CUtensorMap* out, void* base, int64_t inner, int64_t rows, int64_t ld,
                    int64_t count, int box0, int box1, CUtensorMapSwizzle swizzle) {
  return encode_3d(out, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, inner, rows, ld, count, box0, box1,
                   swizzle);
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

const float kHybrid[10][3] = {{3.4445f, -4.7750f, 2.0315f}, {3.4445f, -4.7750f, 2.0315f},
                              {3.4445f, -4.7750f, 2.0315f}, {3.4445f, -4.7750f, 2.0315f},
                              {3.4445f, -4.7750f, 2.0315f}, {3.4445f, -4.7750f, 2.0315f},
                              {3.4445f, -4.7750f, 2.0315f}, {3.4445f, -4.7750f, 2.0315f},
                              {2.0f, -1.5f, 0.5f},          {2.0f, -1.5f, 0.5f}};

}  // namespace

struct muon_plan_s {
  int mode = 0;  // 0: Muon step, 1: ns_orthogonalize
  muon_precision_t prec = MUON_NS_BF16;
  int steps = 10;
  std::vector<float> abc;
  float eps = 1e-7f;
  std::vector<GroupDesc> groups;
  std::vector<MatDesc> mats;  // internal (group-major) order
  int64_t ew_tiles = 0;
  int64_t stage_tiles[kNumKinds] = {0, 0, 0};
  double flops[kNumKinds] = {0, 0, 0};
  size_t off_groups = 0, off_mats = 0, off_tmaps = 0, off_mat_tmaps = 0, off_tile_mat = 0,
         off_small = 0, off_partial = 0, off_counter = 0, off_scale = 0, desc_bytes = 0,
         ws_bytes = 0;
  std::vector<int32_t> small_mats;  // internal indices run by the small-matrix kernel
  std::vector<int32_t> mid_mats;    // internal indices run by the mid-size kernel
  std::vector<int32_t> tiny_mats;   // internal indices run by the tiny fp32 kernel
  size_t off_mid = 0, off_tiny = 0;
  std::vector<int> launch_kinds;    // 0 elementwise, 1 Gram, 2 Poly, 3 Apply, 4 ApplyLast, 5 small, 8 mid,
                                    // 9 tiny, 6 RMS reduction, 7 update pass (unit-RMS scale)
  int scale_mode = MUON_SCALE_SHAPE;
  int sumsq_per_tile = 1;           // sum-of-squares slots per Apply tile (unit-RMS scale)
  size_t off_sumsq = 0, off_factor = 0;
  float* diag = nullptr;            // caller's diagnostics output (2 floats per matrix) or NULL
  // L2 batching: the stage launches run batch by batch over consecutive
  // matrices whose Newton-Schulz working set fits the budget (0: one batch)
  size_t l2_batch_bytes = 0;
  std::vector<std::pair<int, int>> batches;  // internal matrix ranges [first, last)
  // chained launch of the Newton-Schulz stages (bf16, one pass): the tile
  // list and the per-matrix dependency counters live in the descriptor region
  bool chain_on = true;
  int chain_window = 0;             // matrices in flight (0: from the tile counts)
  int64_t chain_len = 0;            // tiles of every stage of every grouped matrix
  size_t off_chain = 0, off_dep = 0;
  std::vector<uint8_t> blob;
  // one-shot calls: the descriptor tables travel as kernel arguments, since
  // the plan (and its host image) ends when the call returns
  bool upload_by_value = false;
  void* uploaded_ws = nullptr;
  int uploaded_dev = -1;
  std::vector<void*> events;
};

namespace {

muon_status_t set_schedule(muon_plan_s* p, const muon_ns_schedule_t* s) {
  if (!s) {
    p->steps = 10;
    p->abc.assign(&kHybrid[0][0], &kHybrid[0][0] + 30);
    p->eps = 1e-7f;
    return MUON_OK;
  }
  if (s->steps < 1 || s->steps > MUON_MAX_NS_STEPS || !s->abc || !(s->eps > 0.f) ||
      !std::isfinite(s->eps))
    return MUON_ERR_INVALID_ARG;
  for (int k = 0; k < 3 * s->steps; ++k)
    if (!std::isfinite(s->abc[k])) return MUON_ERR_INVALID_ARG;
  p->steps = s->steps;
  p->abc.assign(s->abc, s->abc + 3 * s->steps);
  p->eps = s->eps;
  return MUON_OK;
}

// Workspace bytes one matrix's Newton-Schulz buffers take (the L2 working
// set of its stages): bf16 iterate high x 2 + low, A and B.
double ns_bytes(const muon_plan_s* p, const MatDesc& md) {
  const GroupDesc& gd = p->groups[md.group];
  if (gd.small) return 0.0;
  const double x = static_cast<double>(gd.r) * gd.ldc, a = static_cast<double>(gd.r) * gd.ldr;
  return p->prec == MUON_NS_BF16 ? 6.0 * x + 4.0 * a : 8.0 * x + 8.0 * a;
}

// Split the matrices (internal order) into batches for the stage launches.
void make_batches(muon_plan_s* p) {
  p->batches.clear();
  const int nm = static_cast<int>(p->mats.size());
  if (p->l2_batch_bytes == 0) {
    p->batches.emplace_back(0, nm);
    return;
  }
  int first = 0;
  double acc = 0.0;
  for (int i = 0; i < nm; ++i) {
    const double b = ns_bytes(p, p->mats[i]);
    if (i > first && acc + b > static_cast<double>(p->l2_batch_bytes)) {
      p->batches.emplace_back(first, i);
      first = i;
      acc = 0.0;
    }
    acc += b;
  }
  p->batches.emplace_back(first, nm);
}

// First tile of internal matrix i in stage kind k's table (the total for i = count).
int64_t first_tile(const muon_plan_s* p, int i, int k) {
  if (i >= static_cast<int>(p->mats.size())) return p->stage_tiles[k];
  const MatDesc& md = p->mats[i];
  const GroupDesc& gd = p->groups[md.group];
  return gd.tile_base[k] + static_cast<int64_t>(md.index) * gd.tiles_per_mat[k];
}

// Gram, Poly and the last Apply take the eight-epilogue-warp variant when the
// tile-weighted mean length of their main loops (K = c for Gram, r for the
// others) is at most 512 (1024 for the last Apply, whose epilogue also moves
// W): there the epilogue, not the operand feed, sets the tile rate. Measured
// on 512^2, 512 x 2048, 1024^2 and 2048^2 batches.
bool wide_epilogue(const muon_plan_s* p, const std::pair<int, int>& bt, int kind, bool last) {
  if (kind == kApply && !last) return true;
  const double kmax = (kind == kApply) ? 1024.0 : 512.0;
  double tiles = 0.0, ksum = 0.0;
  for (int i = bt.first; i < bt.second; ++i) {
    const GroupDesc& gd = p->groups[p->mats[i].group];
    const double t = static_cast<double>(gd.tiles_per_mat[kind]);
    tiles += t;
    ksum += t * (kind == kGram ? gd.c : gd.r);
  }
  return tiles > 0.0 && ksum <= kmax * tiles;
}

// Whether the stages run as one chained launch (bf16, no L2 batching).
bool chained(const muon_plan_s* p) {
  return p->chain_on && p->prec == MUON_NS_BF16 && p->l2_batch_bytes == 0 && p->stage_tiles[kApply] > 0;
}

// The launch list of one execute (depends on the scale mode and the batches).
void make_launch_list(muon_plan_s* p) {
  const bool unit = p->scale_mode == MUON_SCALE_UNIT_RMS;
  make_batches(p);
  p->launch_kinds.assign(1, 0);
  if (!p->small_mats.empty()) p->launch_kinds.push_back(5);
  if (!p->mid_mats.empty()) p->launch_kinds.push_back(8);
  if (!p->tiny_mats.empty()) p->launch_kinds.push_back(9);
  if (chained(p)) {
    // every stage in one launch; the last Apply fused with the update runs
    // after it (in the unit-RMS mode the chain holds the last Apply too)
    p->launch_kinds.push_back(10);
    if (unit) {
      p->launch_kinds.push_back(6);
      p->launch_kinds.push_back(7);
    } else {
      p->launch_kinds.push_back(4);
      if (p->diag) p->launch_kinds.push_back(6);
    }
    return;
  }
  if (p->stage_tiles[kApply] > 0) {
    for (const auto& bt : p->batches) {
      if (first_tile(p, bt.first, kApply) == first_tile(p, bt.second, kApply)) continue;
      for (int k = 0; k < p->steps; ++k) {
        p->launch_kinds.push_back(1);
        p->launch_kinds.push_back(2);
        p->launch_kinds.push_back(k + 1 == p->steps && !unit ? 4 : 3);
      }
    }
    if (unit) {
      p->launch_kinds.push_back(6);
      p->launch_kinds.push_back(7);
    } else if (p->diag) {
      p->launch_kinds.push_back(6);  // update-RMS diagnostics of the fused last step
    }
  }
}

// Build groups, tiles, flop counts and the workspace layout from `mats`
// (caller order; only pointers, n, m filled).
muon_status_t build_plan(muon_plan_s* p, const std::vector<MatDesc>& caller) {
  const bool tc = (p->prec == MUON_NS_BF16);
  std::map<std::pair<int64_t, int64_t>, int> gid;
  std::vector<std::vector<int>> members;
  for (size_t k = 0; k < caller.size(); ++k) {
    const int64_t r = std::min(caller[k].n, caller[k].m), c = std::max(caller[k].n, caller[k].m);
    auto key = std::make_pair(r, c);
    auto it = gid.find(key);
    if (it == gid.end()) {
      if (static_cast<int>(members.size()) >= kMaxGroups) return MUON_ERR_UNSUPPORTED;
      it = gid.emplace(key, static_cast<int>(members.size())).first;
      members.emplace_back();
    }
    members[it->second].push_back(static_cast<int>(k));
  }
  std::vector<std::pair<int64_t, int64_t>> shape(members.size());
  for (auto& kv : gid) shape[kv.second] = kv.first;

  p->groups.assign(members.size(), GroupDesc{});
  p->mats.clear();
  int64_t ew_total = 0;
  for (size_t g = 0; g < members.size(); ++g) {
    GroupDesc& gd = p->groups[g];
    const int64_t r = shape[g].first, c = shape[g].second;
    gd.r = static_cast<int32_t>(r);
    gd.c = static_cast<int32_t>(c);
    gd.ldc = static_cast<int32_t>(align_up(static_cast<size_t>(c), 8));
    gd.ldr = static_cast<int32_t>(align_up(static_cast<size_t>(r), 8));
    gd.count = static_cast<int32_t>(members[g].size());
    gd.first_mat = static_cast<int32_t>(p->mats.size());
    double fl[kNumKinds] = {0, 0, 0};
    gd.small = !tc                                   ? 0
               : (r * c <= kTinyMaxElems)              ? 3
               : (r <= kSmallMax && c <= kSmallMax)    ? 1
               : (r <= kSmallMax && c <= kMidMaxC)     ? 2
                                                       : 0;
    if (gd.small) {
      // one CTA per matrix, dense 128 x 128 products; count the useful FLOPs
      fl[kGram] = 2.0 * r * r * static_cast<double>(c);
      fl[kPoly] = 2.0 * r * r * static_cast<double>(r);
      for (int k = 0; k < kNumKinds; ++k) gd.tiles_per_mat[k] = 0;
    } else if (tc) {
      // pair tiles of 256 x 256; the symmetric stages run those on or below
      // the diagonal and keep the 128 x 128 blocks on or below it
      const int64_t rb = cdiv(r, 128);
      for (int64_t i = 0; i < rb; ++i) {
        const double rows = static_cast<double>(std::min<int64_t>(128, r - i * 128));
        for (int64_t bj = 0; bj <= i; ++bj) {
          const double cols = static_cast<double>(std::min<int64_t>(128, r - bj * 128));
          fl[kGram] += 2.0 * rows * cols * static_cast<double>(c);
          fl[kPoly] += 2.0 * rows * cols * static_cast<double>(r);
        }
      }
      const int64_t pb = cdiv(r, kPairM);
      gd.tiles_per_mat[kGram] = pb * (pb + 1) / 2;
      gd.tiles_per_mat[kPoly] = gd.tiles_per_mat[kGram];
      gd.tiles_per_mat[kApply] = pb * cdiv(c, kPairN);
    } else {
      gd.tiles_per_mat[kGram] = cdiv(r, kSBM) * cdiv(r, kSBN);
      gd.tiles_per_mat[kPoly] = gd.tiles_per_mat[kGram];
      gd.tiles_per_mat[kApply] = cdiv(r, kSBM) * cdiv(c, kSBN);
      fl[kGram] = 2.0 * r * r * static_cast<double>(c);
      fl[kPoly] = 2.0 * r * r * static_cast<double>(r);
    }
    fl[kApply] = 2.0 * r * static_cast<double>(c) * static_cast<double>(r);
    for (int k = 0; k < kNumKinds; ++k) {
      gd.tile_base[k] = p->stage_tiles[k];
      p->stage_tiles[k] += gd.tiles_per_mat[k] * gd.count;
      gd.tile_flops[k] = static_cast<int64_t>(fl[k]);
      p->flops[k] += fl[k] * gd.count * p->steps;
    }
    for (size_t idx = 0; idx < members[g].size(); ++idx) {
      MatDesc md = caller[members[g][idx]];
      md.transposed = md.n > md.m ? 1 : 0;
      md.group = static_cast<int32_t>(g);
      md.index = static_cast<int32_t>(idx);
      md.caller = static_cast<int32_t>(members[g][idx]);
      // the last step moves W and O by TMA when their rows are 16-byte aligned
      const bool rows16 = (md.m % 4) == 0;
      md.flags = 0;
      if (md.W && rows16 && (reinterpret_cast<uintptr_t>(md.W) & 15) == 0) md.flags |= kMatWTma;
      if (md.O && rows16 && (reinterpret_cast<uintptr_t>(md.O) & 15) == 0) md.flags |= kMatOTma;
      if (gd.small == 1) p->small_mats.push_back(static_cast<int32_t>(p->mats.size()));
      if (gd.small == 2) p->mid_mats.push_back(static_cast<int32_t>(p->mats.size()));
      if (gd.small == 3) p->tiny_mats.push_back(static_cast<int32_t>(p->mats.size()));
      md.ew_tile_begin = ew_total;
      md.ew_tiles = cdiv(md.n, kEwRows) * cdiv(md.m, kEwCols);
      ew_total += md.ew_tiles;
      p->mats.push_back(md);
    }
  }
  p->ew_tiles = ew_total;

  // workspace layout
  const size_t ng = p->groups.size(), nm = p->mats.size();
  size_t off = 0;
  p->off_groups = off;
  off = align_up(off + ng * sizeof(GroupDesc), 256);
  p->off_mats = off;
  off = align_up(off + nm * sizeof(MatDesc), 256);
  p->off_tmaps = off;
  off = align_up(off + (tc ? ng * kTmPerGroup * sizeof(CUtensorMap) : 0), 256);
  p->off_mat_tmaps = off;
  off = align_up(off + (tc ? nm * kMtPerMat * sizeof(CUtensorMap) : 0), 256);
  p->off_tile_mat = off;
  off = align_up(off + static_cast<size_t>(ew_total) * sizeof(int32_t), 256);
  p->off_small = off;
  off = align_up(off + p->small_mats.size() * sizeof(int32_t), 256);
  p->off_mid = off;
  off = align_up(off + p->mid_mats.size() * sizeof(int32_t), 256);
  p->off_tiny = off;
  off = align_up(off + p->tiny_mats.size() * sizeof(int32_t), 256);
  p->off_partial = off;
  off = align_up(off + static_cast<size_t>(ew_total) * sizeof(float), 256);
  p->off_counter = off;
  off = align_up(off + nm * sizeof(unsigned), 256);
  p->off_scale = off;
  off = align_up(off + nm * sizeof(float), 256);
  // unit-RMS scale: sums of squares of O' per Apply tile, then gamma / RMS per matrix
  p->sumsq_per_tile = tc ? 16 : 1;  // tensor cores: 2 CTAs x 8 slots (one per epilogue warp) per tile
  p->off_sumsq = off;
  off = align_up(off + static_cast<size_t>(p->stage_tiles[kApply]) * p->sumsq_per_tile * sizeof(float), 256);
  p->off_factor = off;
  off = align_up(off + nm * sizeof(float), 256);
  // chained launch: the tile list (every stage of every step of every grouped
  // matrix) and one dependency counter per matrix
  p->chain_len = 0;
  if (tc)
    for (const auto& md : p->mats) {
      const GroupDesc& gd = p->groups[md.group];
      p->chain_len += static_cast<int64_t>(p->steps) *
                      (gd.tiles_per_mat[kGram] + gd.tiles_per_mat[kPoly] + gd.tiles_per_mat[kApply]);
    }
  p->off_chain = off;
  off = align_up(off + static_cast<size_t>(p->chain_len) * sizeof(ChainTile), 256);
  p->off_dep = off;
  off = align_up(off + (tc ? (nm + 1) * sizeof(unsigned) : 0), 256);  // + the tile counter
  p->desc_bytes = off;
  off = align_up(off, 1024);
  for (auto& gd : p->groups) {
    const size_t cnt = static_cast<size_t>(gd.count);
    const size_t x_elems = cnt * static_cast<size_t>(gd.r) * gd.ldc;
    const size_t a_elems = cnt * static_cast<size_t>(gd.r) * gd.ldr;
    const size_t ab_bytes = tc ? 2 : 4;
    if (tc) {
      // bf16 mode: the iterate as high part (ping-pong: the Apply product reads
      // the current one whole) and low part (updated in place by its owner tile)
      gd.xf_off[0] = gd.xf_off[1] = 0;
      gd.xb_off[0] = static_cast<int64_t>(off);
      off = align_up(off + x_elems * 2, 1024);
      gd.xb_off[1] = static_cast<int64_t>(off);
      off = align_up(off + x_elems * 2, 1024);
      gd.xlo_off = static_cast<int64_t>(off);
      off = align_up(off + x_elems * 2, 1024);
    } else {
      gd.xf_off[0] = static_cast<int64_t>(off);
      off = align_up(off + x_elems * 4, 1024);
      gd.xf_off[1] = static_cast<int64_t>(off);
      off = align_up(off + x_elems * 4, 1024);
      gd.xb_off[0] = gd.xb_off[1] = 0;
      gd.xlo_off = 0;
    }
    gd.a_off = static_cast<int64_t>(off);
    off = align_up(off + a_elems * ab_bytes, 1024);
    gd.b_off = static_cast<int64_t>(off);
    off = align_up(off + a_elems * ab_bytes, 1024);
  }
  p->ws_bytes = off;

  p->blob.assign(p->desc_bytes, 0);
  std::memcpy(p->blob.data() + p->off_groups, p->groups.data(), ng * sizeof(GroupDesc));
  std::memcpy(p->blob.data() + p->off_mats, p->mats.data(), nm * sizeof(MatDesc));
  if (!p->small_mats.empty())
    std::memcpy(p->blob.data() + p->off_small, p->small_mats.data(), p->small_mats.size() * sizeof(int32_t));
  if (!p->mid_mats.empty())
    std::memcpy(p->blob.data() + p->off_mid, p->mid_mats.data(), p->mid_mats.size() * sizeof(int32_t));
  if (!p->tiny_mats.empty())
    std::memcpy(p->blob.data() + p->off_tiny, p->tiny_mats.data(), p->tiny_mats.size() * sizeof(int32_t));
  make_launch_list(p);
  auto* tile_mat = reinterpret_cast<int32_t*>(p->blob.data() + p->off_tile_mat);
  for (size_t k = 0; k < nm; ++k)
    for (int64_t t = 0; t < p->mats[k].ew_tiles; ++t)
      tile_mat[p->mats[k].ew_tile_begin + t] = static_cast<int32_t>(k);
  return MUON_OK;
}

// The planner keeps r, c and their leading dimensions (rounded up to 8) in
// 32-bit fields, so both sides stop 8 short of 2^31.
constexpr int64_t kMaxDim = 0x7fffffffLL - 7;

bool valid_shape(int64_t n, int64_t m) {
  return n >= 1 && m >= 1 && n <= kMaxDim && m <= kMaxDim;
}

// The chained launch's tile list: a window of W matrices in flight, in
// rounds; each round lists the next stage of every matrix in the window (all
// its tiles), and a matrix that has finished every stage leaves the window
// for the next one. A stage of a matrix is listed one round after the stage
// it depends on, with the other matrices' tiles in between, so CTA pairs that
// reach it seldom wait; the window's buffers are the working set that stays
// in L2. W defaults to the number of matrices whose average stage gives
// every CTA pair two and a half tiles per round, and at least two.
void build_chain(const muon_plan_s* p, int npairs, ChainTile* out) {
  std::vector<int> mats;
  double stage_tiles = 0.0;
  for (size_t i = 0; i < p->mats.size(); ++i) {
    const GroupDesc& gd = p->groups[p->mats[i].group];
    const int64_t per_step = gd.tiles_per_mat[kGram] + gd.tiles_per_mat[kPoly] + gd.tiles_per_mat[kApply];
    if (per_step == 0) continue;
    mats.push_back(static_cast<int>(i));
    stage_tiles += per_step / 3.0;
  }
  if (mats.empty()) return;
  int window = p->chain_window;
  if (window <= 0) {
    // at least two, so that another matrix's tiles sit between a stage and
    // the stage that depends on it, covering the first one's last tiles
    const double mean = stage_tiles / static_cast<double>(mats.size());
    window = std::max(2, static_cast<int>(std::ceil(2.5 * std::max(npairs, 1) / std::max(mean, 1.0))));
  }
  window = std::max(1, std::min<int>(window, static_cast<int>(mats.size())));
  const int nstages = 3 * p->steps;
  std::vector<std::pair<int, int>> act;  // (matrix, next stage)
  size_t next = 0;
  int64_t k = 0;
  while (next < mats.size() || !act.empty()) {
    while (static_cast<int>(act.size()) < window && next < mats.size()) act.emplace_back(mats[next++], 0);
    for (auto& x : act) {
      const GroupDesc& gd = p->groups[p->mats[x.first].group];
      const int kind = x.second % 3;
      for (int64_t u = 0; u < gd.tiles_per_mat[kind]; ++u)
        out[k++] = ChainTile{x.first, x.second, static_cast<int32_t>(u), 0};
      ++x.second;
    }
    act.erase(std::remove_if(act.begin(), act.end(), [&](const std::pair<int, int>& x) { return x.second == nstages; }),
              act.end());
  }
}

muon_status_t upload(muon_plan_s* p, void* ws, int dev, cudaStream_t stream) {
  if (p->chain_len > 0)
    build_chain(p, g_chain_pairs[dev], reinterpret_cast<ChainTile*>(p->blob.data() + p->off_chain));
  if (p->prec == MUON_NS_BF16) {
    char* base = static_cast<char*>(ws);
    auto* maps = reinterpret_cast<CUtensorMap*>(p->blob.data() + p->off_tmaps);
    for (size_t g = 0; g < p->groups.size(); ++g) {
      const GroupDesc& gd = p->groups[g];
      CUtensorMap* m = maps + g * kTmPerGroup;
      const auto SW128 = CU_TENSOR_MAP_SWIZZLE_128B;
      const auto SW64 = CU_TENSOR_MAP_SWIZZLE_64B;
      const bool ok =
          // operand maps (K blocks of 64 elements, 128-byte swizzle)
          encode_bf16_3d(&m[kTmXb0K], base + gd.xb_off[0], gd.c, gd.r, gd.ldc, gd.count, 64, 128, SW128) &&
          encode_bf16_3d(&m[kTmXb1K], base + gd.xb_off[1], gd.c, gd.r, gd.ldc, gd.count, 64, 128, SW128) &&
          encode_bf16_3d(&m[kTmXb0MN], base + gd.xb_off[0], gd.c, gd.r, gd.ldc, gd.count, 64, 64, SW128) &&
          encode_bf16_3d(&m[kTmXb1MN], base + gd.xb_off[1], gd.c, gd.r, gd.ldc, gd.count, 64, 64, SW128) &&
          encode_bf16_3d(&m[kTmA], base + gd.a_off, gd.r, gd.r, gd.ldr, gd.count, 64, 128, SW128) &&
          encode_bf16_3d(&m[kTmB], base + gd.b_off, gd.r, gd.r, gd.ldr, gd.count, 64, 128, SW128) &&
          // epilogue maps (32 x 32 chunks)
          encode_bf16_3d(&m[kTmXloE], base + gd.xlo_off, gd.c, gd.r, gd.ldc, gd.count, 32, 32, SW64) &&
          encode_bf16_3d(&m[kTmXb0E], base + gd.xb_off[0], gd.c, gd.r, gd.ldc, gd.count, 32, 32, SW64) &&
          encode_bf16_3d(&m[kTmXb1E], base + gd.xb_off[1], gd.c, gd.r, gd.ldc, gd.count, 32, 32, SW64) &&
          encode_bf16_3d(&m[kTmAE], base + gd.a_off, gd.r, gd.r, gd.ldr, gd.count, 32, 32, SW64) &&
          encode_bf16_3d(&m[kTmBE], base + gd.b_off, gd.r, gd.r, gd.ldr, gd.count, 32, 32, SW64) &&
          encode_bf16_3d(&m[kTmAMN], base + gd.a_off, gd.r, gd.r, gd.ldr, gd.count, 64, 64, SW128) &&
          encode_bf16_3d(&m[kTmBMN], base + gd.b_off, gd.r, gd.r, gd.ldr, gd.count, 64, 64, SW128);
      if (!ok) return MUON_ERR_CUDA;
    }
    auto* mmaps = reinterpret_cast<CUtensorMap*>(p->blob.data() + p->off_mat_tmaps);
    for (size_t k = 0; k < p->mats.size(); ++k) {
      const MatDesc& md = p->mats[k];
      CUtensorMap* m = mmaps + k * kMtPerMat;
      const auto F32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
      const auto SW128 = CU_TENSOR_MAP_SWIZZLE_128B;
      if ((md.flags & kMatWTma) &&
          !encode_3d(&m[kMtW], md.W, F32, 4, md.m, md.n, md.m, 1, 32, 32, SW128))
        return MUON_ERR_CUDA;
      if ((md.flags & kMatOTma) &&
          !encode_3d(&m[kMtO], md.O, F32, 4, md.m, md.n, md.m, 1, 32, 32, SW128))
        return MUON_ERR_CUDA;
    }
  }
  if (p->upload_by_value) {
    if (launch_blob_copy(ws, p->blob.data(), p->desc_bytes, stream) != cudaSuccess) return MUON_ERR_CUDA;
  } else if (cudaMemcpyAsync(ws, p->blob.data(), p->desc_bytes, cudaMemcpyHostToDevice, stream) !=
             cudaSuccess) {
    return MUON_ERR_CUDA;
  }
  p->uploaded_ws = ws;
  p->uploaded_dev = dev;
  return MUON_OK;
}

// Timing events around launches. Under stream capture the record must become
// an external event node of the graph, or its timestamp cannot be read after
// a replay.
std::atomic<int> g_tracing{0};

// NVTX range names of the launch kinds (host-side ranges around each launch;
// a profiler attached to the process shows them, otherwise they cost a call)
const char* kind_name(int kind) {
  static const char* names[] = {"muon:momentum+norm", "muon:gram", "muon:poly", "muon:apply",
                                "muon:apply+update", "muon:small", "muon:rms", "muon:update",
                                "muon:mid", "muon:tiny"};
  return (kind >= 0 && kind < 10) ? names[kind] : "muon:?";
}

// Slots come in pairs around launch slot / 2: timing events (when set) and
// NVTX ranges (when tracing is on).
muon_status_t record(muon_plan_s* p, int slot, cudaStream_t stream) {
  if (g_tracing.load(std::memory_order_relaxed)) {
    if ((slot & 1) == 0) {
      const int k = slot / 2;
      nvtxRangePushA(kind_name(k < static_cast<int>(p->launch_kinds.size()) ? p->launch_kinds[k] : -1));
    } else {
      nvtxRangePop();
    }
  }
  if (p->events.empty()) return MUON_OK;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return MUON_ERR_CUDA;
  const cudaEvent_t ev = static_cast<cudaEvent_t>(p->events[slot]);
  const cudaError_t e = (cap == cudaStreamCaptureStatusActive)
                            ? cudaEventRecordWithFlags(ev, stream, cudaEventRecordExternal)
                            : cudaEventRecord(ev, stream);
  return e == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

int launch_count(const muon_plan_s* p) { return static_cast<int>(p->launch_kinds.size()); }

}  // namespace

extern "C" {

muon_status_t muon_plan_create(const muon_param_t* params, int count, muon_precision_t prec,
                               const muon_ns_schedule_t* sched, muon_plan_t* plan) {
  if (!plan) return MUON_ERR_INVALID_ARG;
  *plan = nullptr;
  if (!params || count <= 0) return MUON_ERR_INVALID_ARG;
  if (prec != MUON_NS_BF16 && prec != MUON_NS_FP32) return MUON_ERR_INVALID_ARG;
  std::vector<MatDesc> caller(static_cast<size_t>(count));
  for (int k = 0; k < count; ++k) {
    const muon_param_t& q = params[k];
    if (!q.W || !q.G || !q.M || !valid_shape(q.n, q.m)) return MUON_ERR_INVALID_ARG;
    MatDesc md{};
    md.W = q.W;
    md.G = q.G;
    md.M = q.M;
    md.O = q.O;
    md.n = q.n;
    md.m = q.m;
    caller[k] = md;
  }
  auto* p = new (std::nothrow) muon_plan_s();
  if (!p) return MUON_ERR_INVALID_ARG;
  p->mode = 0;
  p->prec = prec;
  muon_status_t st = set_schedule(p, sched);
  if (st == MUON_OK) st = build_plan(p, caller);
  if (st != MUON_OK) {
    delete p;
    return st;
  }
  *plan = p;
  return MUON_OK;
}

muon_status_t muon_plan_create_ns(const muon_ns_matrix_t* mats, int count,
                                  muon_precision_t prec, const muon_ns_schedule_t* sched,
                                  muon_plan_t* plan) {
  if (!plan) return MUON_ERR_INVALID_ARG;
  *plan = nullptr;
  if (!mats || count <= 0) return MUON_ERR_INVALID_ARG;
  if (prec != MUON_NS_BF16 && prec != MUON_NS_FP32) return MUON_ERR_INVALID_ARG;
  std::vector<MatDesc> caller(static_cast<size_t>(count));
  for (int k = 0; k < count; ++k) {
    const muon_ns_matrix_t& q = mats[k];
    if (!q.X || !q.O || !valid_shape(q.n, q.m)) return MUON_ERR_INVALID_ARG;
    MatDesc md{};
    md.G = q.X;
    md.O = q.O;
    md.n = q.n;
    md.m = q.m;
    caller[k] = md;
  }
  auto* p = new (std::nothrow) muon_plan_s();
  if (!p) return MUON_ERR_INVALID_ARG;
  p->mode = 1;
  p->prec = prec;
  muon_status_t st = set_schedule(p, sched);
  if (st == MUON_OK) st = build_plan(p, caller);
  if (st != MUON_OK) {
    delete p;
    return st;
  }
  *plan = p;
  return MUON_OK;
}

muon_status_t muon_plan_workspace_size(muon_plan_t plan, size_t* bytes) {
  if (!plan || !bytes) return MUON_ERR_INVALID_ARG;
  *bytes = plan->ws_bytes;
  return MUON_OK;
}

muon_status_t muon_plan_launches(muon_plan_t plan, int* count, int* kinds, int max_kinds) {
  if (!plan || !count) return MUON_ERR_INVALID_ARG;
  const int n = launch_count(plan);
  *count = n;
  if (kinds)
    for (int k = 0; k < n && k < max_kinds; ++k) kinds[k] = plan->launch_kinds[k];
  return MUON_OK;
}

muon_status_t muon_plan_set_events(muon_plan_t plan, void* const* events, int count) {
  if (!plan) return MUON_ERR_INVALID_ARG;
  if (count == 0) {
    plan->events.clear();
    return MUON_OK;
  }
  if (!events || count != 2 * launch_count(plan)) return MUON_ERR_INVALID_ARG;
  for (int k = 0; k < count; ++k)
    if (!events[k]) return MUON_ERR_INVALID_ARG;
  plan->events.assign(events, events + count);
  return MUON_OK;
}

muon_status_t muon_plan_flops(muon_plan_t plan, double* gram, double* poly, double* apply) {
  if (!plan) return MUON_ERR_INVALID_ARG;
  if (gram) *gram = plan->flops[kGram];
  if (poly) *poly = plan->flops[kPoly];
  if (apply) *apply = plan->flops[kApply];
  return MUON_OK;
}

muon_status_t muon_plan_execute(muon_plan_t plan, const muon_hyper_t* hyper, void* workspace,
                                size_t workspace_bytes, void* stream_ptr) {
  if (!plan) return MUON_ERR_INVALID_ARG;
  if (plan->mode == 0) {
    if (!hyper) return MUON_ERR_INVALID_ARG;
    if (!std::isfinite(hyper->lr) || !std::isfinite(hyper->momentum) ||
        !std::isfinite(hyper->weight_decay) || !std::isfinite(hyper->gamma))
      return MUON_ERR_INVALID_ARG;
  }
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) != 0 ||
      workspace_bytes < plan->ws_bytes)
    return MUON_ERR_WORKSPACE;
  int dev = 0;
  muon_status_t st = device_setup(&dev);
  if (st != MUON_OK) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  if (workspace != plan->uploaded_ws || dev != plan->uploaded_dev) {
    st = upload(plan, workspace, dev, stream);
    if (st != MUON_OK) return st;
  }
  char* ws = static_cast<char*>(workspace);
  const auto* groups = reinterpret_cast<const GroupDesc*>(ws + plan->off_groups);
  const auto* mats = reinterpret_cast<const MatDesc*>(ws + plan->off_mats);
  float* scale = reinterpret_cast<float*>(ws + plan->off_scale);
  int* err = g_err_ptr[dev];
  const uint64_t limit = g_wait_limit_ns.load(std::memory_order_relaxed);

  EwArgs ew{};
  ew.groups = groups;
  ew.mats = mats;
  ew.ws = ws;
  ew.tile_mat = reinterpret_cast<const int32_t*>(ws + plan->off_tile_mat);
  ew.partial = reinterpret_cast<float*>(ws + plan->off_partial);
  ew.counter = reinterpret_cast<unsigned*>(ws + plan->off_counter);
  ew.scale = scale;
  ew.err = err;
  ew.total_tiles = plan->ew_tiles;
  ew.nmats = static_cast<int32_t>(plan->mats.size());
  ew.mode = plan->mode;
  ew.nesterov = (plan->mode == 0 && hyper->nesterov) ? 1 : 0;
  ew.split = plan->prec == MUON_NS_BF16 ? 1 : 0;
  ew.mu = plan->mode == 0 ? hyper->momentum : 0.f;
  ew.eps = plan->eps;
  ew.diag = plan->mode == 0 ? plan->diag : nullptr;
  ew.dep = chained(plan) ? reinterpret_cast<unsigned*>(ws + plan->off_dep) : nullptr;
  ew.next_tile = ew.dep ? ew.dep + plan->mats.size() : nullptr;
  if ((st = record(plan, 0, stream)) != MUON_OK) return st;
  if (launch_elementwise(ew, stream) != cudaSuccess) return MUON_ERR_CUDA;
  if ((st = record(plan, 1, stream)) != MUON_OK) return st;

  const bool tc = plan->prec == MUON_NS_BF16;
  const int sms = g_num_sms[dev];
  int slot = 2;
  if (!plan->small_mats.empty() || !plan->mid_mats.empty() || !plan->tiny_mats.empty()) {
    SmallArgs sm{};
    sm.groups = groups;
    sm.mats = mats;
    sm.tmaps = ws + plan->off_tmaps;
    sm.ws = ws;
    sm.scale = scale;
    sm.small_mats = reinterpret_cast<const int32_t*>(ws + plan->off_small);
    sm.err = err;
    sm.nsmall = static_cast<int64_t>(plan->small_mats.size());
    sm.steps = plan->steps;
    if (plan->mode == 0) {
      sm.lr = hyper->lr;
      sm.wd = hyper->weight_decay;
      sm.gamma = hyper->gamma;
    }
    sm.scale_mode = plan->scale_mode;
    sm.diag = plan->mode == 0 ? plan->diag : nullptr;
    sm.wait_limit_ns = limit;
    sm.mode = plan->mode;
    sm.nesterov = ew.nesterov;
    sm.mu = ew.mu;
    for (int k = 0; k < 3 * plan->steps; ++k) sm.abc[k] = plan->abc[k];
    if (sm.nsmall > 0) {
      const int grid = static_cast<int>(std::min<int64_t>(sm.nsmall, 2LL * sms));
      if ((st = record(plan, slot++, stream)) != MUON_OK) return st;
      if (launch_small(sm, grid, stream) != cudaSuccess) return MUON_ERR_CUDA;
      if ((st = record(plan, slot++, stream)) != MUON_OK) return st;
    }
    if (!plan->mid_mats.empty()) {
      sm.small_mats = reinterpret_cast<const int32_t*>(ws + plan->off_mid);
      sm.nsmall = static_cast<int64_t>(plan->mid_mats.size());
      const int grid = static_cast<int>(std::min<int64_t>(sm.nsmall, static_cast<int64_t>(sms)));
      if ((st = record(plan, slot++, stream)) != MUON_OK) return st;
      if (launch_mid(sm, grid, stream) != cudaSuccess) return MUON_ERR_CUDA;
      if ((st = record(plan, slot++, stream)) != MUON_OK) return st;
    }
    if (!plan->tiny_mats.empty()) {
      sm.small_mats = reinterpret_cast<const int32_t*>(ws + plan->off_tiny);
      sm.nsmall = static_cast<int64_t>(plan->tiny_mats.size());
      const int grid = static_cast<int>(std::min<int64_t>(sm.nsmall, 3LL * sms));
      if ((st = record(plan, slot++, stream)) != MUON_OK) return st;
      if (launch_tiny(sm, grid, stream) != cudaSuccess) return MUON_ERR_CUDA;
      if ((st = record(plan, slot++, stream)) != MUON_OK) return st;
    }
  }
  if (plan->stage_tiles[kApply] == 0) return MUON_OK;
  const bool unit = plan->scale_mode == MUON_SCALE_UNIT_RMS;
  const bool diag = plan->mode == 0 && plan->diag != nullptr;
  // arguments of one stage launch (step k, kind) over the tiles of batch bt
  auto stage_args = [&](int k, int kind, const std::pair<int, int>& bt) {
    StageArgs sa{};
    sa.groups = groups;
    sa.mats = mats;
    sa.tmaps = ws + plan->off_tmaps;
    sa.mat_tmaps = ws + plan->off_mat_tmaps;
    sa.ws = ws;
    sa.scale = scale;
    sa.err = err;
    sa.tile_begin = first_tile(plan, bt.first, kind);
    sa.total_tiles = first_tile(plan, bt.second, kind);
    sa.ngroups = static_cast<int32_t>(plan->groups.size());
    const bool last = k == plan->steps - 1;
    sa.first = k == 0;
    // unit-RMS scale: the last Apply keeps O' and its sums of squares; the
    // update comes after the per-matrix reduction. Diagnostics: the fused
    // last step records the sums too.
    sa.last = last && !unit;
    sa.scale_mode = plan->scale_mode;
    if ((unit || diag) && last && kind == kApply) {
      sa.sumsq_per_tile = plan->sumsq_per_tile;
      sa.sumsq = reinterpret_cast<float*>(ws + plan->off_sumsq);
    }
    sa.xsrc = k & 1;
    sa.a = plan->abc[3 * k];
    sa.b = plan->abc[3 * k + 1];
    sa.c = plan->abc[3 * k + 2];
    if (plan->mode == 0) {
      sa.lr = hyper->lr;
      sa.wd = hyper->weight_decay;
      sa.gamma = hyper->gamma;
    }
    sa.wait_limit_ns = limit;
    sa.chain_sumsq_stage = -1;
    return sa;
  };
  auto launch_one = [&](const StageArgs& sa, int kind, const std::pair<int, int>& bt) -> muon_status_t {
    const int64_t tiles = sa.total_tiles - sa.tile_begin;
    cudaError_t e;
    if (tc) {
      const int grid = 2 * static_cast<int>(std::min<int64_t>(tiles, sms / 2));
      e = launch_stage_tc(static_cast<StageKind>(kind), sa, grid, wide_epilogue(plan, bt, kind, sa.last != 0), stream);
    } else {
      const int grid = static_cast<int>(std::min<int64_t>(tiles, 8LL * sms));
      e = launch_stage_simt(static_cast<StageKind>(kind), sa, grid, stream);
    }
    return e == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
  };
  if (chained(plan)) {
    // every stage in one persistent launch (the last Apply too in the
    // unit-RMS mode), then the last Apply fused with the update
    const std::pair<int, int> all(0, static_cast<int>(plan->mats.size()));
    StageArgs sa = stage_args(0, kGram, all);
    sa.tile_begin = 0;
    sa.total_tiles = plan->chain_len;
    sa.chain = reinterpret_cast<const ChainTile*>(ws + plan->off_chain);
    sa.dep = reinterpret_cast<unsigned*>(ws + plan->off_dep);
    sa.next_tile = sa.dep + plan->mats.size();
    sa.chain_stages = unit ? 3 * plan->steps : 3 * plan->steps - 1;
    sa.last = 0;
    if (unit) {
      sa.chain_sumsq_stage = 3 * plan->steps - 1;
      sa.sumsq_per_tile = plan->sumsq_per_tile;
      sa.sumsq = reinterpret_cast<float*>(ws + plan->off_sumsq);
    }
    for (int k = 0; k < 3 * plan->steps; ++k) sa.abc[k] = plan->abc[k];
    const int pairs = std::max(1, g_chain_pairs[dev]);
    const int grid = 2 * static_cast<int>(std::min<int64_t>(plan->chain_len, pairs));
    if ((st = record(plan, slot++, stream)) != MUON_OK) return st;
    if (launch_stage_chain(sa, grid, stream) != cudaSuccess) return MUON_ERR_CUDA;
    if ((st = record(plan, slot++, stream)) != MUON_OK) return st;
    if (!unit) {
      const StageArgs la = stage_args(plan->steps - 1, kApply, all);
      if ((st = record(plan, slot++, stream)) != MUON_OK) return st;
      if ((st = launch_one(la, kApply, all)) != MUON_OK) return st;
      if ((st = record(plan, slot++, stream)) != MUON_OK) return st;
    }
  } else {
    // one pass of every step per batch: a batch's buffers stay in L2 across its
    // 3 x steps launches when the batch fits
    for (const auto& bt : plan->batches)
    for (int k = 0; k < plan->steps; ++k) {
      if (first_tile(plan, bt.first, kApply) == first_tile(plan, bt.second, kApply)) break;
      for (int kind = 0; kind < kNumKinds; ++kind) {
        const StageArgs sa = stage_args(k, kind, bt);
        if ((st = record(plan, slot++, stream)) != MUON_OK) return st;
        if ((st = launch_one(sa, kind, bt)) != MUON_OK) return st;
        if ((st = record(plan, slot++, stream)) != MUON_OK) return st;
      }
    }
  }
  if (unit || diag) {
    FinishArgs fa{};
    fa.groups = groups;
    fa.mats = mats;
    fa.tile_mat = reinterpret_cast<const int32_t*>(ws + plan->off_tile_mat);
    fa.ws = ws;
    fa.sumsq = reinterpret_cast<const float*>(ws + plan->off_sumsq);
    fa.factor = reinterpret_cast<float*>(ws + plan->off_factor);
    fa.total_tiles = plan->ew_tiles;
    fa.nmats = static_cast<int32_t>(plan->mats.size());
    // the last step (index steps - 1) wrote iterate buffer (steps & 1): the
    // fp32 iterate, or the high part of the split bf16 iterate
    fa.xf_slot = plan->steps & 1;
    fa.split = tc ? 1 : 0;
    fa.sumsq_per_tile = plan->sumsq_per_tile;
    fa.apply_kind = kApply;
    fa.lr = hyper->lr;
    fa.wd = hyper->weight_decay;
    fa.gamma = hyper->gamma;
    fa.scale_mode = plan->scale_mode;
    fa.diag = plan->diag;
    if ((st = record(plan, slot++, stream)) != MUON_OK) return st;
    if (launch_rms_reduce(fa, stream) != cudaSuccess) return MUON_ERR_CUDA;
    if ((st = record(plan, slot++, stream)) != MUON_OK) return st;
    if (unit) {
      if ((st = record(plan, slot++, stream)) != MUON_OK) return st;
      if (launch_finish(fa, stream) != cudaSuccess) return MUON_ERR_CUDA;
      if ((st = record(plan, slot++, stream)) != MUON_OK) return st;
    }
  }
  return MUON_OK;
}

muon_status_t muon_plan_set_scale_mode(muon_plan_t plan, muon_scale_mode_t mode) {
  if (!plan || plan->mode != 0) return MUON_ERR_INVALID_ARG;
  if (mode != MUON_SCALE_SHAPE && mode != MUON_SCALE_UNIT_RMS && mode != MUON_SCALE_NONE)
    return MUON_ERR_INVALID_ARG;
  plan->scale_mode = mode;
  make_launch_list(plan);
  plan->events.clear();  // the launch list may have changed: timing must be set again
  return MUON_OK;
}

void muon_set_tracing(int on) { g_tracing.store(on ? 1 : 0, std::memory_order_relaxed); }

muon_status_t muon_plan_set_l2_batching(muon_plan_t plan, size_t bytes) {
  if (!plan) return MUON_ERR_INVALID_ARG;
  plan->l2_batch_bytes = bytes;
  make_launch_list(plan);
  plan->events.clear();  // the launch list may have changed: timing must be set again
  return MUON_OK;
}

muon_status_t muon_plan_set_diagnostics(muon_plan_t plan, float* out) {
  if (!plan || plan->mode != 0) return MUON_ERR_INVALID_ARG;
  if (out && (reinterpret_cast<uintptr_t>(out) & 3) != 0) return MUON_ERR_INVALID_ARG;
  plan->diag = out;
  make_launch_list(plan);
  plan->events.clear();  // the launch list may have changed: timing must be set again
  return MUON_OK;
}

muon_status_t muon_plan_set_chaining(muon_plan_t plan, int on, int window) {
  if (!plan || window < 0) return MUON_ERR_INVALID_ARG;
  plan->chain_on = on != 0;
  plan->chain_window = window;
  make_launch_list(plan);
  plan->events.clear();    // the launch list may have changed: timing must be set again
  plan->uploaded_ws = nullptr;  // the tile list is rebuilt by the next execute
  return MUON_OK;
}

void muon_plan_destroy(muon_plan_t plan) { delete plan; }

muon_status_t muon_workspace_size(const muon_param_t* params, int count, muon_precision_t prec,
                                  size_t* bytes) {
  if (!bytes) return MUON_ERR_INVALID_ARG;
  muon_plan_t p = nullptr;
  muon_status_t st = muon_plan_create(params, count, prec, nullptr, &p);
  if (st != MUON_OK) return st;
  *bytes = p->ws_bytes;
  muon_plan_destroy(p);
  return MUON_OK;
}

muon_status_t muon_step(const muon_param_t* params, int count, float lr, float momentum,
                        float weight_decay, float gamma, int nesterov,
                        const muon_ns_schedule_t* sched, muon_precision_t prec, void* workspace,
                        size_t workspace_bytes, void* stream) {
  muon_plan_t p = nullptr;
  muon_status_t st = muon_plan_create(params, count, prec, sched, &p);
  if (st != MUON_OK) return st;
  p->upload_by_value = true;
  muon_hyper_t h{lr, momentum, weight_decay, gamma, nesterov};
  st = muon_plan_execute(p, &h, workspace, workspace_bytes, stream);
  muon_plan_destroy(p);
  return st;
}

muon_status_t ns_workspace_size(const muon_ns_matrix_t* mats, int count, muon_precision_t prec,
                                size_t* bytes) {
  if (!bytes) return MUON_ERR_INVALID_ARG;
  muon_plan_t p = nullptr;
  muon_status_t st = muon_plan_create_ns(mats, count, prec, nullptr, &p);
  if (st != MUON_OK) return st;
  *bytes = p->ws_bytes;
  muon_plan_destroy(p);
  return MUON_OK;
}

muon_status_t ns_orthogonalize(const muon_ns_matrix_t* mats, int count,
                               const muon_ns_schedule_t* sched, muon_precision_t prec,
                               void* workspace, size_t workspace_bytes, void* stream) {
  muon_plan_t p = nullptr;
  muon_status_t st = muon_plan_create_ns(mats, count, prec, sched, &p);
  if (st != MUON_OK) return st;
  p->upload_by_value = true;
  st = muon_plan_execute(p, nullptr, workspace, workspace_bytes, stream);
  muon_plan_destroy(p);
  return st;
}

muon_status_t muon_sync_status(void* stream) {
  int dev = 0;
  muon_status_t st = device_setup(&dev);
  if (st != MUON_OK) return st;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MUON_ERR_CUDA;
  int bits = 0;
  if (cudaMemcpy(&bits, g_err_ptr[dev], sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MUON_ERR_CUDA;
  if (bits) {
    const int zero = 0;
    if (cudaMemcpy(g_err_ptr[dev], &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return MUON_ERR_CUDA;
  }
  return (bits & kErrTimeout) ? MUON_ERR_TIMEOUT : MUON_OK;
}

const char* muon_status_string(muon_status_t status) {
  switch (status) {
    case MUON_OK: return "ok";
    case MUON_ERR_INVALID_ARG: return "invalid argument";
    case MUON_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MUON_ERR_CUDA: return "CUDA runtime error";
    case MUON_ERR_UNSUPPORTED: return "unsupported device or size";
    case MUON_ERR_TIMEOUT: return "device-side wait expired";
  }
  return "unknown status";
}

int muon_abi_version(void) { return MUON_ABI_VERSION; }

void muon_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns.store(ns < 1000 ? 1000 : ns, std::memory_order_relaxed);
}

muon_status_t muon_dep_wait_probe(const uint32_t* counter, uint32_t target, uint64_t limit_ns,
                                  void* stream) {
  if (!counter) return MUON_ERR_INVALID_ARG;
  int dev = 0;
  muon_status_t st = device_setup(&dev);
  if (st != MUON_OK) return st;
  return launch_dep_wait_probe(counter, target, g_err_ptr[dev], limit_ns,
                               static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MUON_OK
             : MUON_ERR_CUDA;
}

muon_status_t muon_wait_probe(const int* flag, uint64_t limit_ns, void* stream) {
  if (!flag) return MUON_ERR_INVALID_ARG;
  int dev = 0;
  muon_status_t st = device_setup(&dev);
  if (st != MUON_OK) return st;
  return launch_wait_probe(flag, g_err_ptr[dev], limit_ns, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MUON_OK
             : MUON_ERR_CUDA;
}

}  // extern "C"

namespace muon {

void plan_upload_by_value(muon_plan_t plan) {
  if (plan) plan->upload_by_value = true;
}

namespace {

// One chunk of host bytes carried in the launch's parameter space (kernel
// parameters may take up to 32764 bytes): the launch copies them to `dst`.
constexpr int kBlobChunkWords = 2040;  // 32,640 bytes of 16-byte words
struct BlobChunk {
  uint4 data[kBlobChunkWords];
  uint4* dst;
  uint32_t words;
};
static_assert(sizeof(BlobChunk) <= 32764, "kernel parameter limit");

__global__ void blob_copy_kernel(const __grid_constant__ BlobChunk c) {
  for (uint32_t i = threadIdx.x; i < c.words; i += blockDim.x) c.dst[i] = c.data[i];
}

__global__ void wait_probe_kernel(const int* flag, int* err, unsigned long long limit_ns) {
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint64_t it = 0; it < ptx::kSpinBackstop; ++it) {
    if (*reinterpret_cast<const volatile int*>(flag) != 0) return;
    if (ptx::globaltimer_ns() - t0 > limit_ns) break;
    __nanosleep(256);
  }
  atomicOr(err, kErrTimeout);
}
}  // namespace

// Copy `bytes` (a multiple of 16; `dst` 16-byte aligned) from host memory to
// the device in launches that carry the bytes as kernel arguments. Chunks of
// zeros become memsets. Nothing on the device refers to `src` afterwards.
cudaError_t launch_blob_copy(void* dst, const void* src, size_t bytes, cudaStream_t stream) {
  if ((bytes & 15) != 0 || (reinterpret_cast<uintptr_t>(dst) & 15) != 0) return cudaErrorInvalidValue;
  static thread_local BlobChunk chunk;  // 32 KB: kept off the stack
  const auto* s = static_cast<const uint8_t*>(src);
  constexpr size_t kChunkBytes = sizeof(chunk.data);
  for (size_t off = 0; off < bytes; off += kChunkBytes) {
    const size_t n = std::min(kChunkBytes, bytes - off);
    bool zero = true;
    for (size_t i = 0; i < n && zero; ++i) zero = s[off + i] == 0;
    uint8_t* d = static_cast<uint8_t*>(dst) + off;
    if (zero) {
      const cudaError_t e = cudaMemsetAsync(d, 0, n, stream);
      if (e != cudaSuccess) return e;
      continue;
    }
    std::memcpy(chunk.data, s + off, n);
    chunk.dst = reinterpret_cast<uint4*>(d);
    chunk.words = static_cast<uint32_t>(n / 16);
    blob_copy_kernel<<<1, 256, 0, stream>>>(chunk);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_wait_probe(const int* flag, int* err, unsigned long long limit_ns,
                              cudaStream_t stream) {
  wait_probe_kernel<<<1, 1, 0, stream>>>(flag, err, limit_ns);
  return cudaGetLastError();
}

namespace {
// The chained launch's dependency wait, alone: on expiry, the timeout bit.
__global__ void dep_wait_probe_kernel(const unsigned* counter, unsigned target, int* err,
                                      unsigned long long limit_ns) {
  volatile int no_abort = 0;
  if (!ptx::dep_wait(counter, target, err, limit_ns, &no_abort)) atomicOr(err, kErrTimeout);
}
}  // namespace

cudaError_t launch_dep_wait_probe(const uint32_t* counter, uint32_t target, int* err,
                                  unsigned long long limit_ns, cudaStream_t stream) {
  dep_wait_probe_kernel<<<1, 1, 0, stream>>>(counter, target, err, limit_ns);
  return cudaGetLastError();
}

// Current device, checked to be an sm_100 part; sets up the per-device state.
muon_status_t current_device_checked(int* dev) { return device_setup(dev); }

}  // namespace muon
