// Offline weight counter-rotation W_rot = Q^T . W (sm_100a).
//
// The pages do not print this step: it is what keeps the layer's output
// unchanged when the input is rotated, since x . W = (x . Q) . (Q^T . W) for
// an orthogonal Q.  The rotation is stored as Qt = Q^T (row-major), so this is
// the plain product Qt . W.  It runs once per projection group, off the
// per-token path.  A 128 x 64 output tile per 256-thread CTA, k-steps of 16
// staged in shared memory, 8 x 4 fp32 register accumulators per thread; bf16
// results are rounded to nearest even.
#include "common.cuh"
#include "internal.h"

namespace larosa {
namespace {

constexpr int BM = 128;  // rows of W_rot (columns of Q) per CTA
constexpr int BN = 64;   // columns of W_rot per CTA
constexpr int BK = 16;
constexpr int kPrepThreads = 256;

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// W_rot[i][j] = sum_k Qt[i][k] * W[k][j]; Qt is [d x d], W and W_rot [d x n].
template <typename T>
__global__ void __launch_bounds__(kPrepThreads) prepare_kernel(const T* __restrict__ Qt,
                                                               const T* __restrict__ W,
                                                               T* __restrict__ W_rot, int d,
                                                               int n) {
  __shared__ float As[BK][BM + 4];  // As[k][i] = Qt[i0 + i][k0 + k]
  __shared__ float Bs[BK][BN + 4];  // Bs[k][j] = W[k0 + k][j0 + j]
  const int tid = threadIdx.x;
  const int i0 = blockIdx.y * BM;
  const int j0 = blockIdx.x * BN;
  const int tx = tid % 16;  // 4 columns each
  const int ty = tid / 16;  // 8 rows each

  // No early trigger: the kernels of the decode path may read their weights
  // as soon as the previous kernel lets them launch, so the kernel that
  // writes a weight lets them launch only when it ends.
  pdl_wait();

  float acc[8][4];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;

  for (int k0 = 0; k0 < d; k0 += BK) {
#pragma unroll
    for (int q = 0; q < (BK * BM) / kPrepThreads; ++q) {
      const int e = tid + q * kPrepThreads;
      const int ii = e / BK, kk = e % BK;  // consecutive threads read along k
      const int k = k0 + kk, i = i0 + ii;
      As[kk][ii] = (k < d && i < d) ? to_f32(Qt[(size_t)i * d + k]) : 0.f;
    }
#pragma unroll
    for (int q = 0; q < (BK * BN) / kPrepThreads; ++q) {
      const int e = tid + q * kPrepThreads;
      const int kk = e / BN, jj = e % BN;
      const int k = k0 + kk, j = j0 + jj;
      Bs[kk][jj] = (k < d && j < n) ? to_f32(W[(size_t)k * n + j]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[8], b[4];
#pragma unroll
      for (int r = 0; r < 8; ++r) a[r] = As[kk][ty * 8 + r];
#pragma unroll
      for (int c = 0; c < 4; ++c) b[c] = Bs[kk][tx * 4 + c];
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int i = i0 + ty * 8 + r;
    if (i >= d) continue;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = j0 + tx * 4 + c;
      if (j < n) W_rot[(size_t)i * n + j] = from_f32<T>(acc[r][c]);
    }
  }
}

}  // namespace

cudaError_t launch_prepare(const void* Q, const void* W, void* W_rot, int d_in, int d_out,
                           Elem elem, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((d_out + BN - 1) / BN, (d_in + BM - 1) / BM, 1);
  cfg.blockDim = dim3(kPrepThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (elem == Elem::BF16)
    return cudaLaunchKernelEx(&cfg, prepare_kernel<__nv_bfloat16>,
                              static_cast<const __nv_bfloat16*>(Q),
                              static_cast<const __nv_bfloat16*>(W),
                              static_cast<__nv_bfloat16*>(W_rot), d_in, d_out);
  return cudaLaunchKernelEx(&cfg, prepare_kernel<float>, static_cast<const float*>(Q),
                            static_cast<const float*>(W), static_cast<float*>(W_rot), d_in,
                            d_out);
}

}  // namespace larosa
