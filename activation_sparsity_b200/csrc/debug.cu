// Debug checks of kept lists (enabled with larosa_set_debug or LAROSA_DEBUG).
//
// The sparse linear sums val[m][k] * W[idx[m][k]] over a token's kept list,
// which the La RoSA summary (方法详解 / 技术框架) defines as a set of rows of
// the rotated weight: each index at most once.  The paths for several tokens
// turn a list into a dense coefficient row (a repeated index would be
// counted once there and twice in the one-token gather), so a repeated index
// is reported rather than given a meaning.  The lists the library writes are
// also in ascending index order, which the check confirms for them.
#include "common.cuh"
#include "internal.h"

namespace larosa {
namespace {

constexpr int kCheckThreads = 1024;

// One CTA per token: a bitmap of the indices seen so far (d bits of shared
// memory), set with atomicOr so that a second visit of an index is seen.
__global__ void __launch_bounds__(kCheckThreads) check_lists_kernel(const int32_t* __restrict__ idx,
                                                                    const float* __restrict__ val, int K,
                                                                    int d, int ascending, int* dev_status) {
  extern __shared__ uint32_t seen[];
  const int m = blockIdx.x;
  const int words = (d + 31) / 32;
  for (int w = threadIdx.x; w < words; w += kCheckThreads) seen[w] = 0u;
  __syncthreads();
  const int32_t* row = idx + (size_t)m * K;
  const float* vrow = val + (size_t)m * K;
  int bits = 0;
  for (int k = threadIdx.x; k < K; k += kCheckThreads) {
    const int i = row[k];
    if (static_cast<unsigned>(i) >= static_cast<unsigned>(d)) {
      bits |= LAROSA_DEV_INDEX;
      continue;
    }
    const uint32_t b = 1u << (i & 31);
    if (atomicOr(&seen[i >> 5], b) & b) bits |= LAROSA_DEV_LIST;
    if (ascending && k > 0 && row[k - 1] >= i) bits |= LAROSA_DEV_LIST;
    if (!isfinite(vrow[k])) bits |= LAROSA_DEV_NONFINITE;
  }
  bits = __reduce_or_sync(0xffffffffu, bits);
  if ((threadIdx.x & 31) == 0 && bits != 0) report(dev_status, bits);
}

}  // namespace

cudaError_t launch_check_lists(const int32_t* idx, const float* val, int M, int K, int d, bool ascending,
                               int* dev_status, cudaStream_t stream) {
  if (dev_status == nullptr || M < 1 || K < 1) return cudaSuccess;  // nothing to report or to check
  const size_t smem = (size_t)((d + 31) / 32) * 4;
  check_lists_kernel<<<M, kCheckThreads, smem, stream>>>(idx, val, K, d, ascending ? 1 : 0, dev_status);
  return cudaGetLastError();
}

}  // namespace larosa
