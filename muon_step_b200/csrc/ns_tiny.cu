// Newton-Schulz for tiny matrices with fp32 operands, one CTA per matrix.
//
// A matrix of at most kTinyMaxElems elements (so min(n, m) <= 64) has too
// few elements for the rounding of bf16 operands to average out over the
// Frobenius norm of O': a bf16-operand iteration can land above the 2e-2
// bound on matrices of a few dozen elements. In the bf16 precision these
// matrices therefore run here, with fp32 operands and fp32 accumulation on
// the CUDA cores; the cost is a few hundred kFLOP per matrix.
//
// One CTA of 256 threads takes one matrix at a time and keeps everything in
// shared memory: the iterate X and its successor (r x c each), A and B
// (r x r each), all fp32, rows padded to an odd stride so that lanes reading
// different rows at the same column hit different banks.
//
//   N        formed again from the caller's M (already advanced to M_t by the
//            elementwise kernel) and G with the elementwise kernel's own fp32
//            operations, N = mu M_t + G (Nesterov), so the iterate starts
//            from the exact fp32 N rather than its bf16 high + low parts
//   steps    A = alpha^2 X X^T, B = b A + c A A, X' = alpha (a X + B X)
//            ("Ch 06 · Muon" §3 and §5 Algorithm 1, regrouped; alpha = s
//            on step one, the elementwise kernel's 1 / (||N||_F + eps))
//   update   W <- W (1 - lr wd) - lr gamma sqrt(max(n, m)) O' in the caller's
//            orientation ("Muon 优化器完全拆解…", Algorithm 1 steps four and
//            five), or one of the other scale rules, as the small kernel does
//
// Every dot product runs over its index in increasing order with fmaf, and
// the sums of squares are reduced in a fixed order: results are
// deterministic. There are no spin-waits.
#include "kernels.cuh"
#include "stage_common.cuh"

namespace muon {

namespace {

constexpr int kTinyThreads = 256;
constexpr int kTinyWarps = kTinyThreads / 32;
// r * (c | 1) <= kTinyMaxElems + r and r * (r | 1) <= 64 * 65: four such buffers
constexpr int kTinyMaxR = 64;
constexpr int kTinyBufFloats = kTinyMaxElems + kTinyMaxR;
constexpr size_t kTinySmem = 4 * kTinyBufFloats * sizeof(float);
static_assert(kTinyMaxR * kTinyMaxR <= kTinyMaxElems, "r <= 64 follows from r * c <= kTinyMaxElems");
static_assert(kTinyMaxR * (kTinyMaxR + 1) <= kTinyBufFloats, "A and B fit their buffers");

}  // namespace

__global__ void __launch_bounds__(kTinyThreads) ns_tiny_kernel(const __grid_constant__ SmallArgs a) {
  extern __shared__ float tiny_smem[];
  __shared__ float red[kTinyWarps];
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;

  for (int64_t idx = blockIdx.x; idx < a.nsmall; idx += gridDim.x) {
    const int mat = a.small_mats[idx];
    const MatDesc& md = a.mats[mat];
    const GroupDesc& gd = a.groups[md.group];
    const int r = gd.r, c = gd.c;
    const int ldx = c | 1;
    const int ldr = r | 1;
    const int cols = static_cast<int>(md.m);  // caller columns
    const bool tr = md.transposed != 0;
    float* X = tiny_smem;
    float* Xn = tiny_smem + kTinyBufFloats;
    float* A = tiny_smem + 2 * kTinyBufFloats;
    float* B = tiny_smem + 3 * kTinyBufFloats;

    // N in the iterate's orientation (rows <= cols), read in caller order
    for (int e = tid; e < r * c; e += kTinyThreads) {
      const int crow = e / cols, ccol = e - crow * cols;
      const float g = md.G[e];
      float v = g;
      if (a.mode == 0) {
        const float mt = md.M[e];
        v = a.nesterov ? fmaf(a.mu, mt, g) : mt;
      }
      const int i = tr ? ccol : crow, j = tr ? crow : ccol;
      X[i * ldx + j] = v;
    }
    __syncthreads();
    const float s = a.scale[mat];

    for (int k = 0; k < a.steps; ++k) {
      const float alpha = (k == 0) ? s : 1.f;
      const float ca = a.abc[3 * k], cb = a.abc[3 * k + 1], cc = a.abc[3 * k + 2];
      // Gram: A = alpha^2 X X^T (A[i][j] and A[j][i] take the same products
      // in the same order, so A is exactly symmetric)
      for (int e = tid; e < r * r; e += kTinyThreads) {
        const int i = e / r, j = e - i * r;
        const float* xi = X + i * ldx;
        const float* xj = X + j * ldx;
        float acc = 0.f;
        for (int l = 0; l < c; ++l) acc = fmaf(xi[l], xj[l], acc);
        A[i * ldr + j] = alpha * alpha * acc;
      }
      __syncthreads();
      // Poly: B = b A + c A A
      for (int e = tid; e < r * r; e += kTinyThreads) {
        const int i = e / r, j = e - i * r;
        const float* ai = A + i * ldr;
        float acc = 0.f;
        for (int l = 0; l < r; ++l) acc = fmaf(ai[l], A[l * ldr + j], acc);
        B[i * ldr + j] = fmaf(cb, ai[j], cc * acc);
      }
      __syncthreads();
      // Apply: X' = alpha (a X + B X)
      for (int e = tid; e < r * c; e += kTinyThreads) {
        const int i = e / c, j = e - i * c;
        const float* bi = B + i * ldr;
        float acc = 0.f;
        for (int l = 0; l < r; ++l) acc = fmaf(bi[l], X[l * ldx + j], acc);
        Xn[i * ldx + j] = alpha * fmaf(ca, X[i * ldx + j], acc);
      }
      __syncthreads();
      float* t = X;
      X = Xn;
      Xn = t;
    }

    // O' = X. Sum of squares (unit-RMS scale, diagnostics) in a fixed order.
    const bool need_rms = a.scale_mode == kScaleUnitRms || a.diag != nullptr;
    float rms = 0.f;
    if (need_rms) {
      float ssq = 0.f;
      for (int e = tid; e < r * c; e += kTinyThreads) {
        const int i = e / c, j = e - i * c;
        const float x = X[i * ldx + j];
        ssq = fmaf(x, x, ssq);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
      if (lane == 0) red[warp] = ssq;
      __syncthreads();
      float tot = 0.f;
      for (int w = 0; w < kTinyWarps; ++w) tot += red[w];
      rms = sqrtf(tot / (static_cast<float>(r) * c));
    }
    float gam = a.gamma;
    int mode = a.scale_mode;
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
    for (int e = tid; e < r * c; e += kTinyThreads) {
      const int crow = e / cols, ccol = e - crow * cols;
      const int i = tr ? ccol : crow, j = tr ? crow : ccol;
      const float o = X[i * ldx + j];
      if (md.O) md.O[e] = o;
      if (md.W) md.W[e] = fmaf(md.W[e], uc.keep, -uc.step * o);
    }
    __syncthreads();  // the next matrix overwrites the buffers and red[]
  }
}

size_t tiny_smem_bytes() { return kTinySmem; }

cudaError_t launch_tiny(const SmallArgs& args, int grid, cudaStream_t stream) {
  if (args.nsmall <= 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(ns_tiny_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kTinySmem));
  if (e != cudaSuccess) return e;
  ns_tiny_kernel<<<grid, kTinyThreads, kTinySmem, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace muon
