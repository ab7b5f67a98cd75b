// Exact per-token Top-K by magnitude (sm_100a), one 1024-thread CTA per token.
//
// LaRoSA keeps, for every rotated activation vector, the K entries of largest
// magnitude and zeroes the rest ("La RoSA" summary, 方法详解 / 技术框架;
// abstract: Top-K gives the same sparsity on every token).  Ties are broken
// towards the lower index, +0 and -0 are equal, and the kept entries are
// emitted in ascending index order.
//
// Method: the magnitude of an fp32 value orders exactly like its bit pattern
// with the sign bit cleared, read as an unsigned integer.  A three-pass MSB
// radix select over those 31-bit keys (digits of 11, 11 and 9 bits, shared
// memory histograms) finds the K-th largest key T and how many keys equal to
// T must be kept.  One block-wide scan of packed (#greater, #equal) counts
// over contiguous per-thread chunks then gives every kept entry its output
// position, which is ascending in the index by construction.  The whole
// vector (d <= 32768 fp32) stays in shared memory; nothing but the input row
// and the K outputs touches global memory.
#include "common.cuh"
#include "internal.h"

namespace larosa {
namespace {

constexpr int kTopkThreads = 1024;
constexpr int kMaxBins = 2048;

// Inclusive prefix sum over the 1024 threads of the block.
__device__ __forceinline__ uint32_t block_inclusive_scan(uint32_t v, uint32_t* warp_sums) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_sums[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    warp_sums[lane] = w;
  }
  __syncthreads();
  if (warp > 0) v += warp_sums[warp - 1];
  __syncthreads();
  return v;
}

__global__ void __launch_bounds__(kTopkThreads, 1)
    topk_kernel(const float* __restrict__ x_rot, int d, int K, int32_t* __restrict__ idx,
                float* __restrict__ val, int* dev_status) {
  extern __shared__ __align__(16) uint32_t bits[];  // raw fp32 bits of the row
  __shared__ uint32_t hist[kMaxBins];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t pick[2];

  const int tid = threadIdx.x;
  const int m = blockIdx.x;
  const float* x = x_rot + (size_t)m * d;
  int32_t* out_i = idx + (size_t)m * K;
  float* out_v = val + (size_t)m * K;

  pdl_wait();
  pdl_launch_dependents();

  bool nonfinite = false;
  if ((d & 3) == 0 && (reinterpret_cast<uintptr_t>(x) & 15u) == 0) {
    const uint4* x4 = reinterpret_cast<const uint4*>(x);
    uint4* b4 = reinterpret_cast<uint4*>(bits);
    for (int i = tid; i < (d >> 2); i += kTopkThreads) {
      const uint4 u = __ldcg(x4 + i);
      b4[i] = u;
      nonfinite |= ((u.x & 0x7fffffffu) >= 0x7f800000u) | ((u.y & 0x7fffffffu) >= 0x7f800000u) |
                   ((u.z & 0x7fffffffu) >= 0x7f800000u) | ((u.w & 0x7fffffffu) >= 0x7f800000u);
    }
  } else {
    for (int i = tid; i < d; i += kTopkThreads) {
      const uint32_t u = __float_as_uint(__ldcg(x + i));
      bits[i] = u;
      nonfinite |= (u & 0x7fffffffu) >= 0x7f800000u;
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

  // ---- radix select of the K-th largest key, most significant digit first
  uint32_t prefix = 0, mask = 0;
  uint32_t krem = static_cast<uint32_t>(K);  // keys still to take at/below the prefix
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 20 : (pass == 1 ? 9 : 0);
    const int nb = pass == 2 ? 512 : 2048;
    for (int b = tid; b < nb; b += kTopkThreads) hist[b] = 0;
    __syncthreads();
    for (int i = tid; i < d; i += kTopkThreads) {
      const uint32_t k = bits[i] & 0x7fffffffu;
      if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & (nb - 1)], 1u);
    }
    __syncthreads();
    // thread t owns bins nb-1-2t and nb-2-2t: counts from the top
    uint32_t h_hi = 0, h_lo = 0;
    if (2 * tid < nb) {
      h_hi = hist[nb - 1 - 2 * tid];
      h_lo = hist[nb - 2 - 2 * tid];
    }
    const uint32_t own = h_hi + h_lo;
    const uint32_t incl = block_inclusive_scan(own, warp_sums);
    const uint32_t before = incl - own;
    if (2 * tid < nb && before < krem && krem <= incl) {
      if (before + h_hi >= krem) {
        pick[0] = static_cast<uint32_t>(nb - 1 - 2 * tid);
        pick[1] = before;
      } else {
        pick[0] = static_cast<uint32_t>(nb - 2 - 2 * tid);
        pick[1] = before + h_hi;
      }
    }
    __syncthreads();
    prefix |= pick[0] << shift;
    mask |= static_cast<uint32_t>(nb - 1) << shift;
    krem -= pick[1];
    __syncthreads();
  }
  const uint32_t T = prefix;  // the K-th largest key; krem keys equal to T are kept

  // ---- stable compaction: contiguous chunks, one packed scan of (#eq, #gt)
  const int chunk = (d + kTopkThreads - 1) / kTopkThreads;
  const int i0 = min(d, tid * chunk);
  const int i1 = min(d, i0 + chunk);
  uint32_t gt = 0, eq = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t k = bits[i] & 0x7fffffffu;
    gt += k > T;
    eq += k == T;
  }
  const uint32_t packed = (eq << 16) | gt;  // d < 65536: no carry between halves
  const uint32_t excl = block_inclusive_scan(packed, warp_sums) - packed;
  uint32_t gt_before = excl & 0xffffu;
  uint32_t eq_before = excl >> 16;
  for (int i = i0; i < i1; ++i) {
    const uint32_t u = bits[i];
    const uint32_t k = u & 0x7fffffffu;
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
