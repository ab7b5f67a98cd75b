// Offline weight counter-rotation W_rot = Q^T . W (sm_100a).
//
// The pages do not print this step: it is what keeps the layer's output
// unchanged when the input is rotated, since x . W = (x . Q) . (Q^T . W) for
// an orthogonal Q.  The rotation is stored as Qt = Q^T (row-major), so this is
// the plain product Qt . W.  It runs once per projection group, off the
// per-token path, and is a dense GEMM: bf16 weights go to the fifth-
// generation tensor cores (prep_umma_kernel: 128 x 128 output tiles, Qt
// K-major and W MN-major in 128-byte swizzled TMA tiles, accumulated in TMEM
// a segment at a time and in fp32 registers across segments, bf16 rounded to
// nearest even on the way out); fp32 weights, and
// bf16 ones whose rows are not 16-byte multiples, take the CUDA-core kernel
// (prepare_kernel: a 128 x 64 output tile per 256-thread CTA, k-steps of 16
// staged in shared memory, 8 x 4 fp32 register accumulators per thread).
#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

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

// ---------------------------------------------------------------- tcgen05 GEMM
//
// W_rot[i][j] = sum_k Qt[i][k] W[k][j], bf16: one 128 x 128 output tile per
// CTA over the whole reduction, six warps.  Warp 0 streams 64-deep chunks of
// Qt (128 rows x 64 k, K-major) and of W (64 k x 128 columns as two
// 64-column boxes, MN-major) into a six-stage ring; warp 1 issues M = 128,
// N = 128, K = 16 MMAs and returns each stage with tcgen05.commit.  The
// MMAs accumulate one segment of kPSeg chunks at a time, alternately into
// two TMEM buffers; warps 2-5 (one TMEM lane quarter each) add every
// finished segment into fp32 registers, round to nearest, while the next
// segment fills the other buffer, and at the end round to bf16 and store.
// The accumulation inside the tensor cores behaves like a truncating sum
// (its error grows with the number of MMAs that add into one accumulator):
// with one accumulator over the whole reduction 99.76 % (d = 4096) and
// 99.78 % (d = 11008) of the bf16 outputs equalled the rounding of the
// exact product, against more than 99.9 % for a sequential fp32 sum;
// short segments added with round-to-nearest restore that.  Every mbarrier
// wait is bounded.
constexpr int kPM = 128, kPN = 128, kPStages = 6;
constexpr int kPSeg = 2;  // chunks (64 k each) per segment: 8 MMAs into one accumulator
constexpr uint32_t kPABytes = kPM * tc::kBox * 2;  // 16 KB
constexpr uint32_t kPBBytes = kPN * tc::kBox * 2;  // 16 KB
constexpr uint32_t kPStage = kPABytes + kPBBytes;
constexpr size_t kPSmem = (size_t)kPStages * kPStage + 1024;
constexpr int kPTmemCols = 2 * kPN;  // two segment buffers
constexpr int kPThreads = 192;       // producer, MMA issuer, four epilogue warps
// Tile order: groups of kPGroup row tiles, row tile fastest inside a group,
// so that a wave of CTAs shares a few column blocks of W (and row blocks of
// Qt) through L2 instead of each wave reading all of W once more.
constexpr int kPGroup = 8;

struct PParams {
  __nv_bfloat16* W_rot;
  int d;
  int n;
  int* dev_status;
  unsigned long long wait_ns;
};

__global__ void __launch_bounds__(kPThreads, 1)
    prep_umma_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_w,
                     const PParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* stages = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[kPStages], empty[kPStages], seg_full[2], seg_empty[2];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tiles_m = (p.d + kPM - 1) / kPM, tiles_n = (p.n + kPN - 1) / kPN;
  const int group = static_cast<int>(blockIdx.x) / (kPGroup * tiles_n);
  const int first_m = group * kPGroup;
  const int gm = min(tiles_m - first_m, kPGroup);
  const int in_group = static_cast<int>(blockIdx.x) - group * kPGroup * tiles_n;
  const int j0 = (in_group / gm) * kPN, i0 = (first_m + in_group % gm) * kPM;
  const int n_it = (p.d + tc::kBox - 1) / tc::kBox;
  const int n_seg = (n_it + kPSeg - 1) / kPSeg;
  constexpr uint32_t kId = tc::idesc(kPN, false, true);
  if (tid == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&seg_full[b], 1);   // tcgen05.commit after a segment's last MMA
      mbar_init(&seg_empty[b], 4);  // one arrival per epilogue warp
    }
    s_abort = 0;
    mbar_init_fence();
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(kPTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc::tmem_fence_before();
  __syncthreads();
  tc::tmem_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;
  pdl_wait();  // Qt and W may come from the previous kernel; no early trigger (W_rot is a weight)

  int issued = 0;
  if (warp == 0) {
    if (lane == 0) {
      for (int it = 0; it < n_it; ++it) {
        const int s = it % kPStages;
        if (it >= kPStages && !mbar_wait_bounded(&empty[s], ((it / kPStages) - 1) & 1, abort_flag, p.wait_ns)) {
          *abort_flag = 1;
          break;
        }
        unsigned char* dst = stages + (size_t)s * kPStage;
        const int k = it * tc::kBox;
        mbar_arrive_expect_tx(&full[s], kPStage);
        tc::tma_load_2d(dst, &map_q, k, i0, &full[s]);  // Qt rows i0.., inputs k..k+63
#pragma unroll
        for (int jb = 0; jb < kPN / tc::kBox; ++jb)  // W rows k..k+63, columns j0 + 64 jb..
          tc::tma_load_2d(dst + kPABytes + jb * 8192, &map_w, j0 + tc::kBox * jb, k, &full[s]);
        ++issued;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      for (int it = 0; it < n_it; ++it) {
        const int seg = it / kPSeg, buf = seg & 1;
        const bool first = it % kPSeg == 0, last = it % kPSeg == kPSeg - 1 || it == n_it - 1;
        // a buffer is reused once the epilogue has added the segment before last
        if (first && seg >= 2 &&
            !mbar_wait_bounded(&seg_empty[buf], ((seg >> 1) - 1) & 1, abort_flag, p.wait_ns)) {
          *abort_flag = 1;
          break;
        }
        const int s = it % kPStages;
        if (!mbar_wait_bounded(&full[s], (it / kPStages) & 1, abort_flag, p.wait_ns)) {
          *abort_flag = 1;
          break;
        }
        tc::tmem_fence_after();
        const uint32_t a = smem_u32(stages + (size_t)s * kPStage);
        const uint32_t b = a + kPABytes;
#pragma unroll
        for (int kk = 0; kk < tc::kBox / 16; ++kk)
          tc::umma_bf16(tmem + buf * kPN, tc::sw128_desc(a + kk * 32), tc::sw128_mn_desc(b + kk * 2048, 8192, 1024),
                        (!first || kk > 0) ? 1u : 0u, kId);
        tc::umma_commit(&empty[s]);
        if (last) tc::umma_commit(&seg_full[buf]);
      }
    }
  } else {
    // ---- epilogue warps: warp w reads TMEM lanes 32 (w % 4) ... (its rows of the tile)
    const int quarter = warp & 3;
    float acc[kPN];
#pragma unroll
    for (int c = 0; c < kPN; ++c) acc[c] = 0.f;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    for (int seg = 0; seg < n_seg; ++seg) {
      const int buf = seg & 1;
      // warp-uniform: the whole warp reads TMEM or none of it does
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&seg_full[buf], (seg >> 1) & 1, abort_flag, p.wait_ns))) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      tc::tmem_fence_after();
      __syncwarp();  // tcgen05.ld is .aligned
#pragma unroll
      for (int c0 = 0; c0 < kPN; c0 += 32) {
        float t[32];
        tc::tmem_ld32(lane_base + buf * kPN + c0, t);
#pragma unroll
        for (int e = 0; e < 32; ++e) acc[c0 + e] += t[e];
      }
      tc::tmem_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&seg_empty[buf]);
    }
    if (!*abort_flag) {
      const int i = i0 + quarter * 32 + lane;
      if (i < p.d) {
        __nv_bfloat16* row = p.W_rot + (size_t)i * p.n + j0;
#pragma unroll
        for (int q = 0; q < kPN / 8; ++q) {
          if (j0 + 8 * q < p.n) {  // n is a multiple of 8
            __align__(16) __nv_bfloat16 h[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) h[e] = __float2bfloat16_rn(acc[8 * q + e]);
            *reinterpret_cast<uint4*>(row + 8 * q) = *reinterpret_cast<const uint4*>(h);
          }
        }
      }
    }
  }
  __syncthreads();
  if (*abort_flag && warp == 0 && lane == 0) {
    // let every copy this CTA armed land before its shared memory goes away
    for (int it = max(0, issued - kPStages); it < issued; ++it)
      mbar_wait_bounded(&full[it % kPStages], (it / kPStages) & 1, nullptr, p.wait_ns);
    report(p.dev_status, LAROSA_DEV_TIMEOUT);
  }
  tc::tmem_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc::tmem_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kPTmemCols) : "memory");
  }
}

cudaError_t launch_prep_umma(const void* Qt, const void* W, void* W_rot, int d, int n, cudaStream_t stream) {
  CUtensorMap map_q, map_w;
  if (!tc::make_map(&map_q, Qt, d, d, kPM) || !tc::make_map(&map_w, W, d, n, tc::kBox))
    return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  static bool configured[64] = {};  // per device: the attribute belongs to a device's context
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(prep_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPSmem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  PParams p{static_cast<__nv_bfloat16*>(W_rot), d, n, nullptr, wait_limit_ns()};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(((n + kPN - 1) / kPN) * ((d + kPM - 1) / kPM), 1, 1);
  cfg.blockDim = dim3(kPThreads, 1, 1);
  cfg.dynamicSmemBytes = kPSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, prep_umma_kernel, map_q, map_w, p);
}

}  // namespace

cudaError_t launch_prepare(const void* Q, const void* W, void* W_rot, int d_in, int d_out,
                           Elem elem, cudaStream_t stream) {
  // bf16 with 16-byte rows and 16-byte aligned bases (the tensor maps and the
  // epilogue's vector stores): the tensor cores
  const bool aligned = ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(W) |
                         reinterpret_cast<uintptr_t>(W_rot)) & 15u) == 0;
  if (elem == Elem::BF16 && aligned && d_in % 8 == 0 && d_out % 8 == 0)
    return launch_prep_umma(Q, W, W_rot, d_in, d_out, stream);
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
