// Muon step whose scratch memory is a fixed array inside this library.
//
// Who needs it: callers that must not allocate device memory during a step.
// Examples are runtimes that reserve (nearly) all of HBM up front for their
// own pool; real-time or multi-stream code that cannot afford the device-wide
// synchronisation cudaMalloc / cudaFree may cause; plugins that are handed
// data pointers but no allocator. Such callers pass their matrices and get
// the update in place, and the library uses a file-scope device array as the
// workspace instead of asking for one.
//
// The array is MUON_STATIC_SCRATCH_BYTES (64 MiB). The CUDA module holds it on
// every device where this library is loaded, until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "muon_step.h"

namespace {

static __device__ __align__(256) unsigned char g_static_scratch[MUON_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// The device address of g_static_scratch on the current device. In host code
// the array's name is only a host-side stand-in, so the address must come
// from cudaGetSymbolAddress, once per device, with that device current.
muon_status_t scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MUON_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return MUON_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MUON_OK;
}

}  // namespace

namespace muon {
// The plan's descriptor tables go to the device as kernel arguments (the plan
// ends when this call returns). Defined with the planner.
void plan_upload_by_value(muon_plan_t plan);
}  // namespace muon

extern "C" muon_status_t muon_step_static_scratch(const muon_param_t* params, int count, float lr,
                                                  float momentum, float weight_decay, float gamma,
                                                  int nesterov, const muon_ns_schedule_t* sched,
                                                  muon_precision_t prec, void* stream) {
  muon_plan_t plan = nullptr;
  muon_status_t st = muon_plan_create(params, count, prec, sched, &plan);
  if (st != MUON_OK) return st;
  muon::plan_upload_by_value(plan);
  size_t need = 0;
  st = muon_plan_workspace_size(plan, &need);
  if (st == MUON_OK && need > static_cast<size_t>(MUON_STATIC_SCRATCH_BYTES)) st = MUON_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (st == MUON_OK) st = scratch_address(&scratch);
  // A new plan copies its descriptor tables (with the per-matrix counters
  // that must start at zero) into the scratch before its kernels run; every
  // other scratch byte is written before it is read.
  if (st == MUON_OK) {
    muon_hyper_t h{lr, momentum, weight_decay, gamma, nesterov};
    st = muon_plan_execute(plan, &h, scratch, MUON_STATIC_SCRATCH_BYTES, stream);
  }
  muon_plan_destroy(plan);
  return st;
}
