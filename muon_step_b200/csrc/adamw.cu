// AdamW companion step over a list of flattened fp32 tensors, one launch.
//
// [V4-breakdown] "Muon 优化器完全拆解…", sections "AdamW 到底哪里”不协调”"
// (bias-corrected moments, eps against division by zero) and "为什么嵌入层、
// 输出头、bias、RMSNorm 还在用 AdamW" (which parameters stay on AdamW);
// Algorithm 1 step five (decoupled decay as a factor 1 - lr wd).
//
// Layout: a host-built work list gives each CTA of 256 threads one item:
// either a 4096-element chunk of a large tensor (each thread 4 groups of 4
// consecutive elements at stride 1024, every warp access one contiguous
// 512-byte segment, all 16 of a thread's 16-byte loads issued before its
// first store), or a bundle of consecutive small tensors (up to 4096
// elements in all), one tensor per warp at a time, so that thousands of bias
// and norm vectors do not each occupy a CTA. HBM-bound: 28 bytes per element.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

#include "muon_adamw.h"

namespace muon {

muon_status_t current_device_checked(int* dev);

namespace {

constexpr int kThreads = 256;
constexpr int kGroups = 4;                             // float4 groups per thread
constexpr int64_t kChunk = kThreads * 4 * kGroups;     // 4096 elements per CTA
constexpr int64_t kMaxNumel = int64_t(1) << 40;

struct AdamwTensor {
  float* p;
  const float* g;
  float* m;
  float* v;
  int64_t numel;
  int32_t vec;          // all four pointers 16-byte aligned
  int32_t pad;
};

// One CTA's work: chunk `chunk` of tensor `first`, or (chunk < 0) every
// element of tensors first .. last - 1.
struct AdamwWork {
  int32_t first, last;
  int64_t chunk;
};

struct AdamwArgs {
  const AdamwTensor* tensors;
  const AdamwWork* work;
  int32_t count;
  int64_t total_chunks;  // work items
  float beta1, beta2, one_minus_b1, one_minus_b2, eps, keep;
  float step_size;      // lr / (1 - beta1^t)
  float inv_sqrt_bc2;   // 1 / sqrt(1 - beta2^t)
  const int32_t* step_dev;
  float lr;
  double beta1_d, beta2_d;
};

struct Consts {
  float step_size, inv_sqrt_bc2;
};

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }

__device__ __forceinline__ void adamw_elem(const AdamwArgs& a, const Consts& k, float& p, float g,
                                           float& m, float& v) {
  m = fmaf(a.beta1, m, a.one_minus_b1 * g);
  v = fmaf(a.beta2, v, a.one_minus_b2 * (g * g));
  const float denom = fmaf(sqrtf(v), k.inv_sqrt_bc2, a.eps);
  p = fmaf(p, a.keep, -k.step_size * (m / denom));
}

__global__ void __launch_bounds__(kThreads) adamw_kernel(const __grid_constant__ AdamwArgs a) {
  __shared__ Consts consts_s;
  const AdamwWork wk = a.work[blockIdx.x];
  if (threadIdx.x == 0) {
    Consts k{a.step_size, a.inv_sqrt_bc2};
    if (a.step_dev) {
      const int t = max(1, *a.step_dev);
      const double bc1 = 1.0 - pow(a.beta1_d, static_cast<double>(t));
      const double bc2 = 1.0 - pow(a.beta2_d, static_cast<double>(t));
      k.step_size = static_cast<float>(static_cast<double>(a.lr) / bc1);
      k.inv_sqrt_bc2 = static_cast<float>(1.0 / sqrt(bc2));
    }
    consts_s = k;
  }
  __syncthreads();
  const Consts k = consts_s;
  const int tid = threadIdx.x;
  if (wk.chunk < 0) {
    // bundle of small tensors: one per warp at a time
    const int warp = tid >> 5, lane = tid & 31;
    for (int t = wk.first + warp; t < wk.last; t += kThreads / 32) {
      float* tp = a.tensors[t].p;
      const float* tg = a.tensors[t].g;
      float* tm = a.tensors[t].m;
      float* tv = a.tensors[t].v;
      const int64_t numel = a.tensors[t].numel;
      // small tensors: element per lane, each warp access 128 contiguous bytes
      for (int64_t e = lane; e < numel; e += 32) {
        float p = tp[e], m = tm[e], v = tv[e];
        adamw_elem(a, k, p, tg[e], m, v);
        tp[e] = p;
        tm[e] = m;
        tv[e] = v;
      }
    }
    return;
  }
  const AdamwTensor T = a.tensors[wk.first];
  const int64_t base = wk.chunk * kChunk;
  if (T.vec && base + kChunk <= T.numel) {
    float4 p[kGroups], g[kGroups], m[kGroups], v[kGroups];
#pragma unroll
    for (int q = 0; q < kGroups; ++q) {
      const int64_t i = base + q * (kThreads * 4) + tid * 4;
      p[q] = ld4(T.p + i);
      g[q] = __ldcs(reinterpret_cast<const float4*>(T.g + i));  // read once: stream past L2
      m[q] = ld4(T.m + i);
      v[q] = ld4(T.v + i);
    }
#pragma unroll
    for (int q = 0; q < kGroups; ++q) {
      adamw_elem(a, k, p[q].x, g[q].x, m[q].x, v[q].x);
      adamw_elem(a, k, p[q].y, g[q].y, m[q].y, v[q].y);
      adamw_elem(a, k, p[q].z, g[q].z, m[q].z, v[q].z);
      adamw_elem(a, k, p[q].w, g[q].w, m[q].w, v[q].w);
    }
#pragma unroll
    for (int q = 0; q < kGroups; ++q) {
      const int64_t i = base + q * (kThreads * 4) + tid * 4;
      st4(T.p + i, p[q]);
      st4(T.m + i, m[q]);
      st4(T.v + i, v[q]);
    }
  } else {
    // ragged tail or unaligned tensor: element by element, coalesced by thread
    for (int e = tid; e < kChunk; e += kThreads) {
      const int64_t i = base + e;
      if (i >= T.numel) break;
      float p = T.p[i], m = T.m[i], v = T.v[i];
      adamw_elem(a, k, p, T.g[i], m, v);
      T.p[i] = p;
      T.m[i] = m;
      T.v[i] = v;
    }
  }
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace
}  // namespace muon

struct muon_adamw_plan_s {
  std::vector<muon::AdamwTensor> tensors;
  std::vector<muon::AdamwWork> work;
  size_t off_work = 0;
  int64_t total_chunks = 0;
  int64_t numel = 0;
  size_t ws_bytes = 0;
  void* uploaded_ws = nullptr;
  int uploaded_dev = -1;
};

extern "C" {

muon_status_t muon_adamw_plan_create(const muon_adamw_param_t* params, int count,
                                     muon_adamw_plan_t* plan) {
  using namespace muon;
  if (!plan) return MUON_ERR_INVALID_ARG;
  *plan = nullptr;
  if (!params || count < 1) return MUON_ERR_INVALID_ARG;
  auto* p = new (std::nothrow) muon_adamw_plan_s;
  if (!p) return MUON_ERR_UNSUPPORTED;
  int64_t chunks = 0;
  for (int k = 0; k < count; ++k) {
    const muon_adamw_param_t& q = params[k];
    if (q.numel < 0 || q.numel > kMaxNumel) {
      delete p;
      return MUON_ERR_INVALID_ARG;
    }
    if (q.numel == 0) continue;
    if (!q.p || !q.g || !q.m || !q.v || (reinterpret_cast<uintptr_t>(q.p) & 3) ||
        (reinterpret_cast<uintptr_t>(q.g) & 3) || (reinterpret_cast<uintptr_t>(q.m) & 3) ||
        (reinterpret_cast<uintptr_t>(q.v) & 3)) {
      delete p;
      return MUON_ERR_INVALID_ARG;
    }
    AdamwTensor t{};
    t.p = q.p;
    t.g = q.g;
    t.m = q.m;
    t.v = q.v;
    t.numel = q.numel;
    t.vec = aligned16(q.p) && aligned16(q.g) && aligned16(q.m) && aligned16(q.v);
    chunks += (q.numel + kChunk - 1) / kChunk;
    p->numel += q.numel;
    p->tensors.push_back(t);
  }
  if (chunks > 0x7fffffffLL) {
    delete p;
    return MUON_ERR_UNSUPPORTED;
  }
  // work list: chunks of tensors above half a chunk; runs of smaller ones in
  // bundles of at most kChunk elements (and 64 tensors)
  const int nt = static_cast<int>(p->tensors.size());
  int b0 = -1;
  int64_t bsum = 0;
  auto flush = [&](int end) {
    if (b0 >= 0) p->work.push_back(AdamwWork{b0, end, -1});
    b0 = -1;
    bsum = 0;
  };
  for (int t = 0; t < nt; ++t) {
    const int64_t n = p->tensors[t].numel;
    if (n > kChunk / 2) {
      flush(t);
      const int64_t nc = (n + kChunk - 1) / kChunk;
      for (int64_t ch = 0; ch < nc; ++ch) p->work.push_back(AdamwWork{t, t + 1, ch});
      continue;
    }
    if (b0 >= 0 && (bsum + n > kChunk || t - b0 >= 64)) flush(t);
    if (b0 < 0) b0 = t;
    bsum += n;
  }
  flush(nt);
  if (static_cast<int64_t>(p->work.size()) > 0x7fffffffLL) {
    delete p;
    return MUON_ERR_UNSUPPORTED;
  }
  p->total_chunks = static_cast<int64_t>(p->work.size());
  p->off_work = align_up(std::max<size_t>(p->tensors.size(), 1) * sizeof(AdamwTensor), 256);
  p->ws_bytes = p->off_work + align_up(std::max<size_t>(p->work.size(), 1) * sizeof(AdamwWork), 256);
  *plan = p;
  return MUON_OK;
}

muon_status_t muon_adamw_plan_workspace_size(muon_adamw_plan_t plan, size_t* bytes) {
  if (!plan || !bytes) return MUON_ERR_INVALID_ARG;
  *bytes = plan->ws_bytes;
  return MUON_OK;
}

muon_status_t muon_adamw_plan_numel(muon_adamw_plan_t plan, int64_t* numel) {
  if (!plan || !numel) return MUON_ERR_INVALID_ARG;
  *numel = plan->numel;
  return MUON_OK;
}

muon_status_t muon_adamw_plan_execute(muon_adamw_plan_t plan, const muon_adamw_hyper_t* h,
                                      void* workspace, size_t workspace_bytes, void* stream_ptr) {
  using namespace muon;
  if (!plan || !h) return MUON_ERR_INVALID_ARG;
  if (!std::isfinite(h->lr) || !std::isfinite(h->weight_decay) || !std::isfinite(h->eps) ||
      !(h->eps > 0.f) || !(h->beta1 >= 0.0 && h->beta1 < 1.0) ||
      !(h->beta2 >= 0.0 && h->beta2 < 1.0))
    return MUON_ERR_INVALID_ARG;
  if (!h->step_dev && h->step < 1) return MUON_ERR_INVALID_ARG;
  if (h->step_dev && (reinterpret_cast<uintptr_t>(h->step_dev) & 3)) return MUON_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) != 0 ||
      workspace_bytes < plan->ws_bytes)
    return MUON_ERR_WORKSPACE;
  int dev = 0;
  muon_status_t st = current_device_checked(&dev);
  if (st != MUON_OK) return st;
  if (plan->total_chunks == 0) return MUON_OK;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  if (workspace != plan->uploaded_ws || dev != plan->uploaded_dev) {
    if (cudaMemcpyAsync(workspace, plan->tensors.data(), plan->tensors.size() * sizeof(AdamwTensor),
                        cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaMemcpyAsync(static_cast<char*>(workspace) + plan->off_work, plan->work.data(),
                        plan->work.size() * sizeof(AdamwWork), cudaMemcpyHostToDevice,
                        stream) != cudaSuccess)
      return MUON_ERR_CUDA;
    plan->uploaded_ws = workspace;
    plan->uploaded_dev = dev;
  }
  AdamwArgs a{};
  a.tensors = static_cast<const AdamwTensor*>(workspace);
  a.work = reinterpret_cast<const AdamwWork*>(static_cast<const char*>(workspace) + plan->off_work);
  a.count = static_cast<int32_t>(plan->tensors.size());
  a.total_chunks = plan->total_chunks;
  const double b1 = h->beta1, b2 = h->beta2;
  a.beta1 = static_cast<float>(b1);
  a.beta2 = static_cast<float>(b2);
  a.beta1_d = b1;
  a.beta2_d = b2;
  a.one_minus_b1 = static_cast<float>(1.0 - b1);
  a.one_minus_b2 = static_cast<float>(1.0 - b2);
  a.eps = h->eps;
  a.lr = h->lr;
  a.keep = static_cast<float>(1.0 - static_cast<double>(h->lr) * h->weight_decay);
  a.step_dev = h->step_dev;
  if (!h->step_dev) {
    const double t = h->step;
    a.step_size = static_cast<float>(static_cast<double>(h->lr) / (1.0 - std::pow(b1, t)));
    a.inv_sqrt_bc2 = static_cast<float>(1.0 / std::sqrt(1.0 - std::pow(b2, t)));
  }
  adamw_kernel<<<static_cast<unsigned>(plan->total_chunks), kThreads, 0, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

void muon_adamw_plan_destroy(muon_adamw_plan_t plan) { delete plan; }

muon_status_t muon_adamw_workspace_size(const muon_adamw_param_t* params, int count,
                                        size_t* bytes) {
  if (!bytes) return MUON_ERR_INVALID_ARG;
  muon_adamw_plan_t p = nullptr;
  muon_status_t st = muon_adamw_plan_create(params, count, &p);
  if (st != MUON_OK) return st;
  *bytes = p->ws_bytes;
  muon_adamw_plan_destroy(p);
  return MUON_OK;
}

muon_status_t muon_adamw_step(const muon_adamw_param_t* params, int count,
                              const muon_adamw_hyper_t* hyper, void* workspace,
                              size_t workspace_bytes, void* stream) {
  muon_adamw_plan_t p = nullptr;
  muon_status_t st = muon_adamw_plan_create(params, count, &p);
  if (st != MUON_OK) return st;
  st = muon_adamw_plan_execute(p, hyper, workspace, workspace_bytes, stream);
  muon_adamw_plan_destroy(p);
  return st;
}

}  // extern "C"
