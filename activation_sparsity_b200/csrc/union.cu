// Multi-token support for the sparse linear (sm_100a).
//
// Each token keeps its own K rows.  Streaming every token's rows separately
// would read a row once per token that keeps it; instead the rows kept by any
// token are streamed once and every token multiplies them by its own
// coefficient, which is zero where the token did not keep the row:
//
//   scatter: coef[m][i] = kept value of token m at row i, else 0, and a bitmap
//            of the rows kept by any token;
//   union:   the bitmap compacted into an ascending row list and its length.
//
// The row-streaming GEMV then runs in "coefficient by row id" mode over that
// list, with the list length read on the device.
#include "common.cuh"
#include "internal.h"

namespace larosa {
namespace {

constexpr int kThreads = 1024;

__global__ void __launch_bounds__(kThreads) scatter_kernel(const int32_t* __restrict__ idx,
                                                           const float* __restrict__ val, int K,
                                                           int d_in, float* __restrict__ coef,
                                                           unsigned* bitmap, int* dev_status) {
  const int m = blockIdx.x;
  float* row = coef + (size_t)m * d_in;
  pdl_wait();
  pdl_launch_dependents();
  for (int i = threadIdx.x; i < d_in; i += kThreads) row[i] = 0.f;
  __syncthreads();
  bool bad = false;
  for (int k = threadIdx.x; k < K; k += kThreads) {
    const int i = idx[(size_t)m * K + k];
    if (static_cast<unsigned>(i) < static_cast<unsigned>(d_in)) {
      row[i] = val[(size_t)m * K + k];
      atomicOr(&bitmap[i >> 5], 1u << (i & 31));
    } else {
      bad = true;
    }
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) report(dev_status, LAROSA_DEV_INDEX);
}

// One thread per 32-row bitmap word (d_in <= 32768 = 1024 words).
__global__ void __launch_bounds__(kThreads) union_kernel(unsigned* bitmap, int d_in,
                                                         int32_t* __restrict__ rows,
                                                         int* __restrict__ count) {
  __shared__ uint32_t warp_sums[32];
  const int t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5;
  const int n_words = (d_in + 31) >> 5;
  pdl_wait();
  pdl_launch_dependents();
  const uint32_t w = t < n_words ? bitmap[t] : 0u;
  uint32_t v = __popc(w);
  // inclusive scan of the per-word counts
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_sums[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t s = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += n;
    }
    warp_sums[lane] = s;
  }
  __syncthreads();
  if (warp > 0) v += warp_sums[warp - 1];
  uint32_t pos = v - __popc(w);
  uint32_t bitsleft = w;
  while (bitsleft) {
    const int b = __ffs(bitsleft) - 1;
    rows[pos++] = t * 32 + b;
    bitsleft &= bitsleft - 1;
  }
  if (t < n_words) bitmap[t] = 0u;  // leave the bitmap clear for the next call
  if (t == kThreads - 1) *count = static_cast<int>(v);
}

}  // namespace

cudaError_t launch_scatter(const int32_t* idx, const float* val, int M, int K, int d_in,
                           float* coef, unsigned* bitmap, int* dev_status, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(M, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, scatter_kernel, idx, val, K, d_in, coef, bitmap, dev_status);
}

cudaError_t launch_union(unsigned* bitmap, int d_in, int32_t* rows, int* count,
                         cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, union_kernel, bitmap, d_in, rows, count);
}

}  // namespace larosa
