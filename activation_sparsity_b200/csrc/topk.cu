// Exact per-token Top-K by magnitude (sm_100a), one 1024-thread CTA per token.
//
// LaRoSA keeps, for every rotated activation vector, the K entries of largest
// magnitude and zeroes the rest ("La RoSA" summary, 方法详解 / 技术框架;
// abstract: Top-K gives the same sparsity on every token).  Ties are broken
// towards the lower index, +0 and -0 are equal, and the kept entries are
// emitted in ascending index order.
//
// The selection itself is kept_list() (select.cuh): a 4096-bin histogram of
// the top 12 bits of every magnitude, counted while the row is loaded, one
// scan for the boundary bin, the boundary bin's keys ranked directly, and one
// scan that places every kept entry, ascending in the index.  The whole
// vector (d <= 32768 fp32) stays in shared memory; nothing but the input row
// and the K outputs touches global memory.
#include "coef.cuh"
#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace larosa {
namespace {

constexpr int kTopkThreads = 1024;
constexpr int kTopkCand = 2048;
constexpr int kTopkU = 8;  // 16-byte loads in flight per thread

// Writes the token's dense coefficient rows hi[0, d), lo[0, d): the head and
// tail of x where kept(key, i), zero elsewhere.  d a multiple of 8, hi and lo
// 16-byte aligned.
template <typename Kept>
__device__ __forceinline__ void write_head_tail(const uint32_t* bits, int d, Kept kept,
                                                __nv_bfloat16* hi, __nv_bfloat16* lo) {
  write_head_tail_rows<kTopkThreads>(
      d,
      [&](int i) {
        const uint32_t u = bits[i];
        return kept(u & kKeyMask, i) ? __uint_as_float(u) : 0.f;
      },
      hi, lo);
}

// With hl != nullptr the kernel also writes each token's dense coefficient
// rows for the tensor-core product: hl[m][0, d) the heads, hl[M + m][0, d)
// the tails (d a multiple of 8).
__global__ void __launch_bounds__(kTopkThreads, 1)
    topk_kernel(const float* __restrict__ x_rot, int d, int K, int32_t* __restrict__ idx,
                float* __restrict__ val, int* dev_status, __nv_bfloat16* hl) {
  // raw fp32 bits of the row, padded with zero keys to a multiple of 4: a
  // zero key at an index >= d loses every tie, so padding is never kept
  extern __shared__ __align__(16) uint32_t bits[];
  __shared__ SelectScratch sel;
  __shared__ __align__(16) uint32_t cand[kTopkCand];
  __shared__ uint32_t cand_idx[kTopkCand];

  const int tid = threadIdx.x;
  const int m = blockIdx.x;
  const int d4 = (d + 3) & ~3;
  const float* x = x_rot + (size_t)m * d;
  int32_t* out_i = idx + (size_t)m * K;
  float* out_v = val + (size_t)m * K;

  for (int b = tid; b < kFineBins; b += kTopkThreads) sel.hist[b] = 0u;
  for (int i = d + tid; i < d4; i += kTopkThreads) bits[i] = 0u;
  __syncthreads();
  pdl_wait();
  pdl_launch_dependents();

  bool nonfinite = false;
  if ((d & 3) == 0 && (reinterpret_cast<uintptr_t>(x) & 15u) == 0) {
    const uint4* x4 = reinterpret_cast<const uint4*>(x);
    uint4* b4 = reinterpret_cast<uint4*>(bits);
    const int nv = d >> 2;
    for (int v0 = tid; v0 < nv; v0 += kTopkThreads * kTopkU) {
      uint4 u[kTopkU];
#pragma unroll
      for (int k = 0; k < kTopkU; ++k) {
        const int v = v0 + k * kTopkThreads;
        u[k] = v < nv ? __ldcg(x4 + v) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int k = 0; k < kTopkU; ++k) {
        if (v0 + k * kTopkThreads < nv) {
          b4[v0 + k * kTopkThreads] = u[k];
          const uint32_t w[4] = {u[k].x & kKeyMask, u[k].y & kKeyMask, u[k].z & kKeyMask,
                                 u[k].w & kKeyMask};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            nonfinite |= w[e] >= 0x7f800000u;
            atomicAdd(&sel.hist[w[e] >> kFineShift], 1u);
          }
        }
      }
    }
  } else {
    for (int i = tid; i < d; i += kTopkThreads) {
      const uint32_t u = __float_as_uint(__ldcg(x + i));
      bits[i] = u;
      nonfinite |= (u & kKeyMask) >= 0x7f800000u;
      atomicAdd(&sel.hist[(u & kKeyMask) >> kFineShift], 1u);
    }
  }
  if (tid == 0 && d4 > d) atomicAdd(&sel.hist[0], static_cast<uint32_t>(d4 - d));
  if (__syncthreads_or(nonfinite) && tid == 0) report(dev_status, LAROSA_DEV_NONFINITE);

  // the K-th entry (T, I): K = 0 keeps nothing, K = d everything
  KthEntry e{0xffffffffu, -1};
  if (K == d) {
    e = KthEntry{0u, d};
    for (int i = tid; i < d; i += kTopkThreads) {
      out_i[i] = i;
      out_v[i] = __uint_as_float(bits[i]);
    }
  } else if (K > 0) {
    uint32_t B, above, nB;
    fine_boundary<kTopkThreads>(&sel, K, &B, &above, &nB);
    e = kth_entry<kTopkThreads>(bits, d4, K, B, static_cast<uint32_t>(K) - above, nB, &sel, cand, cand_idx,
                                kTopkCand);
    write_kept<kTopkThreads>(bits, d4, e, 0, K, out_i, out_v, &sel);
  }
  if (hl != nullptr) {
    const size_t M = gridDim.x;
    write_head_tail(bits, d, [&](uint32_t key, int i) { return is_kept(key, i, e); }, hl + (size_t)m * d,
                    hl + (M + m) * d);
  }
}

// The tokens' dense coefficient rows for the tensor-core sparse linear, from
// given kept lists: hl[m][i] / hl[M + m][i] = head / tail of val[m][k] where
// idx[m][k] = i, zero at rows no entry names.  One CTA per token builds the
// row in shared memory (indices within a row are distinct, so no two threads
// write one word) and stores it with 16-byte stores.  An index outside
// [0, d) sets LAROSA_DEV_INDEX and is skipped.
__global__ void __launch_bounds__(kTopkThreads, 1)
    coef_rows_kernel(const int32_t* __restrict__ idx, const float* __restrict__ val, int K, int d,
                     __nv_bfloat16* hl, int* dev_status) {
  extern __shared__ __align__(16) uint32_t row[];  // [d] fp32 coefficients
  const int m = blockIdx.x;
  for (int i = threadIdx.x; i < d; i += kTopkThreads) row[i] = 0u;
  __syncthreads();
  pdl_wait();
  pdl_launch_dependents();
  bool bad = false;
  for (int k = threadIdx.x; k < K; k += kTopkThreads) {
    const int i = __ldg(idx + (size_t)m * K + k);
    if (static_cast<unsigned>(i) < static_cast<unsigned>(d))
      row[i] = __float_as_uint(__ldg(val + (size_t)m * K + k));
    else
      bad = true;
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) report(dev_status, LAROSA_DEV_INDEX);
  const size_t M = gridDim.x;
  // every word of the row is the coefficient itself (0 where not named)
  write_head_tail(row, d, [](uint32_t, int) { return true; }, hl + (size_t)m * d, hl + (M + m) * d);
}

// ---------------------------------------------------------------- threshold
//
// Threshold selection (R-Sparse report, 研究流程与方法 / R-Sparse框架设计: the
// inputs with |x_j| >= t are kept, the rest masked), one 1024-thread CTA per
// token.  t_key is the bit pattern of t >= 0 (0 for t <= 0); magnitudes
// compare as their sign-cleared bit patterns.  The kept entries are written
// in ascending index order to idx/val [M x d] (positions beyond nnz[m] are
// left as they were) and their count to nnz[m].  With coef != nullptr the
// token's row of coef [M x d] also receives x where kept and 0 elsewhere,
// and the kept rows are marked in `bitmap` (the multi-token sparse linear's
// input, as the scatter kernel makes it); with hl != nullptr the token's
// dense bf16 head and tail coefficient rows for the tensor-core product, as
// the Top-K kernel writes them.  Each warp walks its own segment
// of the row twice: once to count, once to place its kept entries after the
// earlier warps' ones.
__global__ void __launch_bounds__(kTopkThreads, 1)
    threshold_kernel(const float* __restrict__ x_rot, int d, uint32_t t_key, int32_t* __restrict__ idx,
                     float* __restrict__ val, int32_t* __restrict__ nnz, float* __restrict__ coef,
                     unsigned* bitmap, int* dev_status, __nv_bfloat16* hl) {
  __shared__ uint32_t warp_sums[32];
  const int m = blockIdx.x;
  const int lane = threadIdx.x & 31;
  const uint32_t below = (1u << lane) - 1u;
  const uint32_t* bits = reinterpret_cast<const uint32_t*>(x_rot + (size_t)m * d);
  pdl_wait();
  pdl_launch_dependents();
  int s0, s1;
  warp_segment<kTopkThreads>(d, &s0, &s1);
  uint32_t n = 0;
  bool bad = false;
  for (int i = s0 + lane; i < s1; i += 32) {
    const uint32_t key = bits[i] & kKeyMask;
    n += key >= t_key;
    bad |= key >= 0x7f800000u;
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) report(dev_status, LAROSA_DEV_NONFINITE);
  n = __reduce_add_sync(0xffffffffu, n);
  uint32_t total = 0;
  uint32_t pos = warp_base<kTopkThreads>(n, warp_sums, &total);
  int32_t* out_i = idx + (size_t)m * d;
  float* out_v = val + (size_t)m * d;
  float* crow = coef != nullptr ? coef + (size_t)m * d : nullptr;
  for (int i0 = s0; i0 < s1; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t u = i < s1 ? bits[i] : 0u;
    const bool kept = i < s1 && (u & kKeyMask) >= t_key;
    const uint32_t mk = __ballot_sync(0xffffffffu, kept);
    if (kept) {
      out_i[pos + __popc(mk & below)] = i;
      out_v[pos + __popc(mk & below)] = __uint_as_float(u);
    }
    if (crow != nullptr && i < s1) {
      crow[i] = kept ? __uint_as_float(u) : 0.f;
      if (kept) atomicOr(&bitmap[i >> 5], 1u << (i & 31));
    }
    pos += __popc(mk);
  }
  if (threadIdx.x == 0) nnz[m] = static_cast<int32_t>(total);
  if (hl != nullptr) {
    const size_t M = gridDim.x;
    write_head_tail(bits, d, [&](uint32_t key, int) { return key >= t_key; }, hl + (size_t)m * d,
                    hl + (M + m) * d);
  }
}

}  // namespace

cudaError_t launch_threshold(const float* x_rot, int M, int d, uint32_t t_key, int32_t* idx,
                             float* val, int32_t* nnz, float* coef, unsigned* bitmap,
                             int* dev_status, cudaStream_t stream, __nv_bfloat16* hl) {
  if (hl != nullptr && d % 8 != 0) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(M, 1, 1);
  cfg.blockDim = dim3(kTopkThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, threshold_kernel, x_rot, d, t_key, idx, val, nnz, coef, bitmap,
                            dev_status, hl);
}

cudaError_t launch_coef_rows(const int32_t* idx, const float* val, int M, int K, int d, __nv_bfloat16* hl,
                             int* dev_status, cudaStream_t stream) {
  if (d % 8 != 0) return cudaErrorInvalidValue;
  const size_t smem = (size_t)d * sizeof(uint32_t);
  static int configured[64] = {0};  // per device: dynamic shared memory limit raised
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    e = cudaFuncSetAttribute(coef_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
  return cudaLaunchKernelEx(&cfg, coef_rows_kernel, idx, val, K, d, hl, dev_status);
}

cudaError_t launch_topk(const float* x_rot, int M, int d, int K, int32_t* idx, float* val,
                        int* dev_status, cudaStream_t stream, __nv_bfloat16* hl) {
  if (hl != nullptr && d % 8 != 0) return cudaErrorInvalidValue;
  const size_t smem = (size_t)((d + 3) & ~3) * sizeof(uint32_t);
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
  return cudaLaunchKernelEx(&cfg, topk_kernel, x_rot, d, K, idx, val, dev_status, hl);
}

}  // namespace larosa
