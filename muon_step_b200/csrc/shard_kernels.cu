// Elementwise steps of the ZeRO-sharded Muon step over lists of shards, and
// the segment copy that packs and unpacks the buffers of grouped exchanges.
//
// [V4-breakdown] "Muon 优化器完全拆解…", section "分布式工程", Algorithm 1
// "Distributed Muon": the momentum update on the local gradient shard (step 2)
// and the parameter update with the local shard of the orthogonalised matrix
// (step 6). The arithmetic repeats that of the single-GPU step exactly:
// M = fma(mu, M, G), N = fma(mu, M, G) as in the elementwise front kernel,
// W = fma(W, 1 - lr wd, -(lr gamma sqrt(c)) O) as in the last Apply epilogue.
// The segment copy moves each matrix's shards between a per-matrix layout and
// a rank-major one, so that every exchange is one collective over one buffer.
//
// Layout as in the AdamW kernel: shards cut into 4096-element chunks, one CTA
// of 256 threads per chunk, 16-byte accesses when every pointer of the shard
// is 16-byte aligned, all loads of a thread before its first store. The item
// table reaches the workspace as kernel arguments (no host memory is
// referenced after a call returns).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <vector>

#include "kernels.cuh"
#include "muon_shard.h"
#include "stage_common.cuh"

namespace muon {

muon_status_t current_device_checked(int* dev);

namespace {

constexpr int kThreads = 256;
constexpr int kGroups = 4;
constexpr int64_t kChunk = kThreads * 4 * kGroups;
constexpr int64_t kMaxNumel = int64_t(1) << 40;

enum Mode : int { kMomentum = 0, kUpdate = 1, kCopy = 2 };

struct ShardItem {
  float* a;           // M (momentum) or W (update), in place; the destination (copy)
  const float* b;     // G, O, or the source (copy)
  float* c;           // N (momentum) or unused
  int64_t numel;
  int64_t chunk_begin;
  int32_t vec;
  int32_t cdim;       // update: max(n, m) of the whole matrix
};

struct ShardArgs {
  const ShardItem* items;
  int32_t count;
  int32_t nesterov;
  float mu;
  float lr, wd, gamma;
};

template <int MODE>
__device__ __forceinline__ void elem(const ShardArgs& s, const UpdateConsts& uc, float& a, float b,
                                     float& c) {
  if (MODE == kMomentum) {
    a = fmaf(s.mu, a, b);
    c = s.nesterov ? fmaf(s.mu, a, b) : a;
  } else if (MODE == kUpdate) {
    a = fmaf(a, uc.keep, -uc.step * b);
  } else {
    a = b;
  }
}

template <int MODE>
__global__ void __launch_bounds__(kThreads) shard_kernel(const __grid_constant__ ShardArgs s) {
  __shared__ int item_s;
  const int64_t chunk = blockIdx.x;
  if (threadIdx.x == 0) {
    int lo = 0, hi = s.count - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(&s.items[mid].chunk_begin) <= chunk) lo = mid;
      else hi = mid - 1;
    }
    item_s = lo;
  }
  __syncthreads();
  const ShardItem it = s.items[item_s];
  const UpdateConsts uc = update_consts_raw(s.lr, s.wd, s.gamma, MODE == kUpdate ? it.cdim : 1);
  const int64_t base = (chunk - it.chunk_begin) * kChunk;
  const int tid = threadIdx.x;
  if (it.vec && base + kChunk <= it.numel) {
    float4 a[kGroups], b[kGroups], c[kGroups];
#pragma unroll
    for (int q = 0; q < kGroups; ++q) {
      const int64_t i = base + q * (kThreads * 4) + tid * 4;
      if (MODE != kCopy) a[q] = *reinterpret_cast<const float4*>(it.a + i);
      b[q] = __ldcs(reinterpret_cast<const float4*>(it.b + i));
    }
#pragma unroll
    for (int q = 0; q < kGroups; ++q) {
      elem<MODE>(s, uc, a[q].x, b[q].x, c[q].x);
      elem<MODE>(s, uc, a[q].y, b[q].y, c[q].y);
      elem<MODE>(s, uc, a[q].z, b[q].z, c[q].z);
      elem<MODE>(s, uc, a[q].w, b[q].w, c[q].w);
    }
#pragma unroll
    for (int q = 0; q < kGroups; ++q) {
      const int64_t i = base + q * (kThreads * 4) + tid * 4;
      *reinterpret_cast<float4*>(it.a + i) = a[q];
      if (MODE == kMomentum) *reinterpret_cast<float4*>(it.c + i) = c[q];
    }
  } else {
    for (int e = tid; e < kChunk; e += kThreads) {
      const int64_t i = base + e;
      if (i >= it.numel) break;
      float a = MODE == kCopy ? 0.f : it.a[i], c = 0.f;
      elem<MODE>(s, uc, a, it.b[i], c);
      it.a[i] = a;
      if (MODE == kMomentum) it.c[i] = c;
    }
  }
}

size_t table_bytes(int count) {
  return (static_cast<size_t>(std::max(count, 1)) * sizeof(ShardItem) + 255) / 256 * 256;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

template <int MODE>
muon_status_t launch(std::vector<ShardItem>& items, int64_t chunks, ShardArgs args, void* workspace,
                     size_t workspace_bytes, void* stream_ptr) {
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < table_bytes(static_cast<int>(items.size())))
    return MUON_ERR_WORKSPACE;
  int dev = 0;
  muon_status_t st = current_device_checked(&dev);
  if (st != MUON_OK) return st;
  if (chunks == 0) return MUON_OK;
  if (chunks > 0x7fffffffLL) return MUON_ERR_UNSUPPORTED;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  // the table goes in by value (16-byte multiple: the items are 48 bytes)
  static_assert(sizeof(ShardItem) % 16 == 0, "item size");
  if (launch_blob_copy(workspace, items.data(), items.size() * sizeof(ShardItem), stream) != cudaSuccess)
    return MUON_ERR_CUDA;
  args.items = static_cast<const ShardItem*>(workspace);
  args.count = static_cast<int32_t>(items.size());
  shard_kernel<MODE><<<static_cast<unsigned>(chunks), kThreads, 0, stream>>>(args);
  return cudaGetLastError() == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

}  // namespace
}  // namespace muon

extern "C" {

muon_status_t muon_shard_workspace_size(int count, size_t* bytes) {
  if (!bytes || count < 1) return MUON_ERR_INVALID_ARG;
  *bytes = muon::table_bytes(count);
  return MUON_OK;
}

muon_status_t muon_shard_momentum(const muon_shard_momentum_t* shards, int count, float momentum,
                                  int nesterov, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  using namespace muon;
  if (!shards || count < 1 || !std::isfinite(momentum)) return MUON_ERR_INVALID_ARG;
  std::vector<ShardItem> items;
  int64_t chunks = 0;
  for (int k = 0; k < count; ++k) {
    const muon_shard_momentum_t& q = shards[k];
    if (q.numel < 0 || q.numel > kMaxNumel) return MUON_ERR_INVALID_ARG;
    if (q.numel == 0) continue;
    if (!q.M || !q.G || !q.N || !aligned(q.M, 4) || !aligned(q.G, 4) || !aligned(q.N, 4))
      return MUON_ERR_INVALID_ARG;
    ShardItem it{};
    it.a = q.M;
    it.b = q.G;
    it.c = q.N;
    it.numel = q.numel;
    it.chunk_begin = chunks;
    it.vec = aligned(q.M, 16) && aligned(q.G, 16) && aligned(q.N, 16);
    chunks += (q.numel + kChunk - 1) / kChunk;
    items.push_back(it);
  }
  ShardArgs a{};
  a.mu = momentum;
  a.nesterov = nesterov ? 1 : 0;
  return launch<kMomentum>(items, chunks, a, workspace, workspace_bytes, stream);
}

muon_status_t muon_shard_update(const muon_shard_update_t* shards, int count, float lr,
                                float weight_decay, float gamma, void* workspace,
                                size_t workspace_bytes, void* stream) {
  using namespace muon;
  if (!shards || count < 1 || !std::isfinite(lr) || !std::isfinite(weight_decay) ||
      !std::isfinite(gamma))
    return MUON_ERR_INVALID_ARG;
  std::vector<ShardItem> items;
  int64_t chunks = 0;
  for (int k = 0; k < count; ++k) {
    const muon_shard_update_t& q = shards[k];
    if (q.numel < 0 || q.numel > kMaxNumel || q.n < 1 || q.m < 1 || q.n > 0x7fffffffLL ||
        q.m > 0x7fffffffLL)
      return MUON_ERR_INVALID_ARG;
    if (q.numel == 0) continue;
    if (!q.W || !q.O || !aligned(q.W, 4) || !aligned(q.O, 4)) return MUON_ERR_INVALID_ARG;
    ShardItem it{};
    it.a = q.W;
    it.b = q.O;
    it.numel = q.numel;
    it.chunk_begin = chunks;
    it.vec = aligned(q.W, 16) && aligned(q.O, 16);
    it.cdim = static_cast<int32_t>(std::max(q.n, q.m));
    chunks += (q.numel + kChunk - 1) / kChunk;
    items.push_back(it);
  }
  ShardArgs a{};
  a.lr = lr;
  a.wd = weight_decay;
  a.gamma = gamma;
  return launch<kUpdate>(items, chunks, a, workspace, workspace_bytes, stream);
}

muon_status_t muon_copy_segments(const muon_segment_t* segs, int count, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  using namespace muon;
  if (!segs || count < 1) return MUON_ERR_INVALID_ARG;
  std::vector<ShardItem> items;
  int64_t chunks = 0;
  for (int k = 0; k < count; ++k) {
    const muon_segment_t& q = segs[k];
    if (q.numel < 0 || q.numel > kMaxNumel) return MUON_ERR_INVALID_ARG;
    if (q.numel == 0) continue;
    if (!q.dst || !q.src || !aligned(q.dst, 4) || !aligned(q.src, 4)) return MUON_ERR_INVALID_ARG;
    ShardItem it{};
    it.a = q.dst;
    it.b = q.src;
    it.numel = q.numel;
    it.chunk_begin = chunks;
    it.vec = aligned(q.dst, 16) && aligned(q.src, 16);
    chunks += (q.numel + kChunk - 1) / kChunk;
    items.push_back(it);
  }
  ShardArgs a{};
  return launch<kCopy>(items, chunks, a, workspace, workspace_bytes, stream);
}

}  // extern "C"
