// Low-rank compensation of the dropped entries (sm_100a): the small kernels
// around the factor GEMVs of larosa_sparse_lowrank_linear for several tokens
// (the row-streaming GEMV, or for bf16 the tensor-core product fed with
// coefficient rows).
//
// R-Sparse report, 研究流程与方法 / R-Sparse框架设计 (hybrid computation): the
// entries a selection drops are not discarded but sent through rank-r
// factors of the weight, y = y_s + (x - sigma(x)) . A_r . B_r.  The dropped
// part is x with the kept entries set to zero; the two products with the
// factors and the sparse product are GEMVs of the library; the sum is the
// last step.
#include <algorithm>

#include "coef.cuh"
#include "common.cuh"
#include "internal.h"

namespace larosa {
namespace {

constexpr int kThreads = 1024;

// x_drop[m] = x[m] with x_drop[m][idx[m][k]] = 0 for the token's K kept
// entries.  One CTA per token.  An index outside [0, d) sets LAROSA_DEV_INDEX.
__global__ void __launch_bounds__(kThreads) dropped_kernel(const float* __restrict__ x,
                                                           const int32_t* __restrict__ idx, int K,
                                                           int d, float* __restrict__ x_drop,
                                                           int* dev_status) {
  const int m = blockIdx.x;
  pdl_wait();
  pdl_launch_dependents();
  const float* xr = x + (size_t)m * d;
  float* out = x_drop + (size_t)m * d;
  for (int i = threadIdx.x; i < d; i += kThreads) out[i] = xr[i];
  __syncthreads();
  bool bad = false;
  for (int k = threadIdx.x; k < K; k += kThreads) {
    const int i = idx[(size_t)m * K + k];
    if (static_cast<unsigned>(i) < static_cast<unsigned>(d))
      out[i] = 0.f;
    else
      bad = true;
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) report(dev_status, LAROSA_DEV_INDEX);
}

// For the tensor-core factor products of several bf16 tokens: the head and
// tail coefficient rows (hl[m][0, d), hl[M + m][0, d)) of x[m] with the K
// kept entries idx[m] set to zero -- the dropped part -- or of x[m] itself
// when K = 0.  One CTA per token; the row is staged in shared memory.  An
// index outside [0, d) sets LAROSA_DEV_INDEX.
__global__ void __launch_bounds__(kThreads) dropped_rows_kernel(const float* __restrict__ x,
                                                                const int32_t* __restrict__ idx, int K,
                                                                int d, __nv_bfloat16* hl, int* dev_status) {
  extern __shared__ float row[];
  const int m = blockIdx.x;
  pdl_wait();
  pdl_launch_dependents();
  const float* xr = x + (size_t)m * d;
  for (int i = threadIdx.x; i < d; i += kThreads) row[i] = xr[i];
  __syncthreads();
  bool bad = false;
  for (int k = threadIdx.x; k < K; k += kThreads) {
    const int i = idx[(size_t)m * K + k];
    if (static_cast<unsigned>(i) < static_cast<unsigned>(d))
      row[i] = 0.f;
    else
      bad = true;
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) report(dev_status, LAROSA_DEV_INDEX);
  const size_t M = gridDim.x;
  write_head_tail_rows<kThreads>(d, [&](int i) { return row[i]; }, hl + (size_t)m * d, hl + (M + m) * d);
}

// y[i] += add[i], n elements.
__global__ void __launch_bounds__(kThreads) add_kernel(float* __restrict__ y,
                                                       const float* __restrict__ add, int n) {
  pdl_wait();
  pdl_launch_dependents();
  for (int i = blockIdx.x * kThreads + threadIdx.x; i < n; i += gridDim.x * kThreads) y[i] += add[i];
}

cudaError_t launch_pdl(const void* fn, int grid, void** args, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace

cudaError_t launch_dropped(const float* x, const int32_t* idx, int M, int K, int d, float* x_drop,
                           int* dev_status, cudaStream_t stream) {
  void* args[] = {&x, &idx, &K, &d, &x_drop, &dev_status};
  return launch_pdl(reinterpret_cast<const void*>(&dropped_kernel), M, args, stream);
}

cudaError_t launch_dropped_rows(const float* x, const int32_t* idx, int M, int K, int d, __nv_bfloat16* hl,
                                int* dev_status, cudaStream_t stream) {
  if (d % 8 != 0 || d > LAROSA_MAX_D) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool configured[64] = {};  // per device: the shared-memory ceiling for a row of LAROSA_MAX_D
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(dropped_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(LAROSA_MAX_D * sizeof(float)));
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(M, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)d * sizeof(float);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, dropped_rows_kernel, x, idx, K, d, hl, dev_status);
}

cudaError_t launch_add(float* y, const float* add, int n, cudaStream_t stream) {
  const int grid = std::max(1, std::min((n + kThreads - 1) / kThreads, 296));
  void* args[] = {&y, &add, &n};
  return launch_pdl(reinterpret_cast<const void*>(&add_kernel), grid, args, stream);
}

}  // namespace larosa
