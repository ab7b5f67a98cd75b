// Exact per-token Top-K by magnitude (sm_100a), one 1024-thread CTA per token.
//
// LaRoSA keeps, for every rotated activation vector, the K entries of largest
// magnitude and zeroes the rest ("La RoSA" summary, 方法详解 / 技术框架;
// abstract: Top-K gives the same sparsity on every token).  Ties are broken
// towards the lower index, +0 and -0 are equal, and the kept entries are
// emitted in ascending index order.
//
// The selection itself (select.cuh) is a radix select over the fp32 bit
// patterns with the sign cleared; one packed block scan then gives every kept
// entry its position, ascending in the index.  The whole vector (d <= 32768
// fp32) stays in shared memory; nothing but the input row and the K outputs
// touches global memory.
#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace larosa {
namespace {

constexpr int kTopkThreads = 1024;
constexpr int kTopkCand = 2048;

__global__ void __launch_bounds__(kTopkThreads, 1)
    topk_kernel(const float* __restrict__ x_rot, int d, int K, int32_t* __restrict__ idx,
                float* __restrict__ val, int* dev_status) {
  extern __shared__ __align__(16) uint32_t bits[];  // raw fp32 bits of the row
  __shared__ SelectScratch sel;
  __shared__ uint32_t cand[2 * kTopkCand];  // keys, then indices

  const int tid = threadIdx.x;
  const int m = blockIdx.x;
  const float* x = x_rot + (size_t)m * d;
  int32_t* out_i = idx + (size_t)m * K;
  float* out_v = val + (size_t)m * K;

  for (int b = tid; b < 2 * kSelBins; b += kTopkThreads) sel.hist[b] = 0u;
  pdl_wait();
  pdl_launch_dependents();

  bool nonfinite = false;
  if ((d & 3) == 0 && (reinterpret_cast<uintptr_t>(x) & 15u) == 0) {
    const uint4* x4 = reinterpret_cast<const uint4*>(x);
    uint4* b4 = reinterpret_cast<uint4*>(bits);
    for (int i = tid; i < (d >> 2); i += kTopkThreads) {
      const uint4 u = __ldcg(x4 + i);
      b4[i] = u;
      nonfinite |= ((u.x & kKeyMask) >= 0x7f800000u) | ((u.y & kKeyMask) >= 0x7f800000u) |
                   ((u.z & kKeyMask) >= 0x7f800000u) | ((u.w & kKeyMask) >= 0x7f800000u);
    }
  } else {
    for (int i = tid; i < d; i += kTopkThreads) {
      const uint32_t u = __float_as_uint(__ldcg(x + i));
      bits[i] = u;
      nonfinite |= (u & kKeyMask) >= 0x7f800000u;
    }
  }
  if (__syncthreads_or(nonfinite) && tid == 0) report(dev_status, LAROSA_DEV_NONFINITE);

  if (K == 0) return;
  if (K == d) {
    for (int i = tid; i < d; i += kTopkThreads) {
      out_i[i] = i;
      out_v[i] = __uint_as_float(bits[i]);
    }
    return;
  }

  uint32_t T = 0, krem = 0;
  select_threshold_fast<kTopkThreads>(bits, d, K, &sel, cand, cand + kTopkCand, kTopkCand, &T,
                                      &krem);

  // ---- stable compaction over contiguous chunks
  const int chunk = (d + kTopkThreads - 1) / kTopkThreads;
  const int i0 = min(d, tid * chunk);
  const int i1 = min(d, i0 + chunk);
  uint32_t gt_before = 0, eq_before = 0;
  kept_chunk_base_1s<kTopkThreads>(bits, i0, i1, T, &sel, &gt_before, &eq_before);
  for (int i = i0; i < i1; ++i) {
    const uint32_t u = bits[i];
    const uint32_t k = u & kKeyMask;
    if (k > T) {
      const uint32_t pos = gt_before + min(eq_before, krem);
      if (pos < static_cast<uint32_t>(K)) {
        out_i[pos] = i;
        out_v[pos] = __uint_as_float(u);
      }
      ++gt_before;
    } else if (k == T) {
      if (eq_before < krem && gt_before + eq_before < static_cast<uint32_t>(K)) {
        const uint32_t pos = gt_before + eq_before;
        out_i[pos] = i;
        out_v[pos] = __uint_as_float(u);
      }
      ++eq_before;
    }
  }
}

}  // namespace

cudaError_t launch_topk(const float* x_rot, int M, int d, int K, int32_t* idx, float* val,
                        int* dev_status, cudaStream_t stream) {
  const size_t smem = (size_t)d * sizeof(uint32_t);
  static int configured[64] = {0};  // per device: dynamic shared memory limit raised
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(LAROSA_MAX_D * sizeof(uint32_t)));
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = 1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(M, 1, 1);
  cfg.blockDim = dim3(kTopkThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, topk_kernel, x_rot, d, K, idx, val, dev_status);
}

}  // namespace larosa
