// Row-dot products of 8 to 16 bf16 tokens on the fifth-generation tensor
// cores (sm_100a): y[m][j] = sum_i x[m][i] * A[j][i], A row-major
// [n_out x n_in].  The rotation x_rot = x . Q reads Q through A = Q^T ("La
// RoSA" summary, 方法详解 / 技术框架: each layer's input activation is
// multiplied by that layer's orthogonal matrix); the dense baseline reads W
// in torch.nn.Linear layout.
//
// One MMA tile is 128 output rows (M) by the 16 token slots (N), over 16
// inputs (K) per instruction.  A CTA owns 128 output rows and one split of
// the inputs:
//   * one thread streams 64-input chunks of A (128 rows x 128 bytes) and of
//     x (16 rows x 128 bytes) into a 4-stage shared-memory ring with 2-D TMA
//     copies in the 128-byte swizzled layout the MMA reads (rows past n_out
//     and tokens past M arrive as zeros);
//   * one thread issues tcgen05.mma (bf16 in, fp32 accumulate into 16 TMEM
//     columns) and returns each stage to the producer with tcgen05.commit;
//   * all four warps read the 128 x 16 accumulator out of TMEM (warp w owns
//     TMEM lanes 32w..32w+31) into shared memory.
// The splits of one row tile form a thread-block cluster and add their
// partial tiles through distributed shared memory in rank order, so the
// result does not depend on timing.  Every mbarrier wait gives up after
// the wait limit; the CTA then lets its copies and MMAs land, frees its TMEM
// and writes nothing.
#include <cooperative_groups.h>
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace larosa {
namespace {

constexpr int kUThreads = 128;                       // 4 warps: TMEM lanes 0..127
constexpr int kURows = 128;                          // MMA M: output rows per CTA
constexpr int kUTokens = 16;                         // MMA N: token slots
constexpr int kUChunk = 64;                          // inputs per stage (128 bytes of bf16)
constexpr int kUStages = 4;
constexpr uint32_t kUABytes = kURows * kUChunk * 2;    // 16 KB
constexpr uint32_t kUBBytes = kUTokens * kUChunk * 2;  // 2 KB
// rotation: A, x; GEMV: A (two 64-column boxes), coefficient head, tail
template <bool kGemv>
constexpr uint32_t stage_bytes() { return kUABytes + (kGemv ? 2 : 1) * kUBBytes; }
constexpr int kUTmemCols = 32;                       // smallest allocation; 16 used

struct UParams {
  float* y;
  int n_out;
  int M;
  int k_per_split;  // inputs per split, a multiple of kUChunk
  int n_in;
  int* dev_status;
  unsigned long long wait_ns;  // limit of every mbarrier wait
};

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// Shared-memory matrix descriptor of a K-major tile in the 128-byte swizzled
// layout: 8-row groups 1024 bytes apart (stride byte offset), leading byte
// offset 1 (unused by swizzled K-major layouts), descriptor version 1,
// layout type 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor: fp32 accumulator, bf16 A and B, both K-major,
// N = 16, M = 128.
constexpr uint32_t kUIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kUTokens >> 3) << 17) |
                             ((uint32_t)(kURows >> 4) << 24);

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate,
                                          uint32_t idesc = kUIdesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u),
      "r"(0u));
}

// Shared-memory descriptor of an MN-major tile in the 128-byte swizzled
// layout: atoms of 64 MN-elements x 8 K-rows (1024 bytes), K-atoms `sbo`
// bytes apart, MN-atoms `lbo` bytes apart.
__device__ __forceinline__ uint64_t sw128_mn_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// As kUIdesc, with A MN-major (bit 15).
constexpr uint32_t kUIdescMN = kUIdesc | (1u << 15);

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// kGemv = false: y[m][j] = sum_i x[m][i] A[j][i] (A = map_a, K-major rows;
// x = map_b0).  kGemv = true: y[m][c] = sum_r coef[m][r] W[r][c] (W = map_a,
// read MN-major: its rows are the reduction; the fp32 coefficients as a bf16
// head map_b0 and tail map_b1, two MMAs per step).
template <bool kGemv>
__global__ void __launch_bounds__(kUThreads, 1)
    umma_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b0,
                const __grid_constant__ CUtensorMap map_b1, const UParams p) {
  constexpr uint32_t kStage = stage_bytes<kGemv>();
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // the swizzled stages need 1024-byte alignment
  unsigned char* stages = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[kUStages], empty[kUStages], done;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x;            // = rank in the cluster
  const int j0 = blockIdx.y * kURows;
  const int k0 = split * p.k_per_split;
  const int k1 = min(p.n_in, k0 + p.k_per_split);
  const int n_it = k1 > k0 ? (k1 - k0 + kUChunk - 1) / kUChunk : 0;

  if (tid == 0) {
    for (int s = 0; s < kUStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&done, 1);
    s_abort = 0;
    mbar_init_fence();
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(kUTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;

  pdl_wait();  // x and A may come from the previous kernel on the stream
  pdl_launch_dependents();

  int issued = 0;
  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      for (int it = 0; it < n_it; ++it) {
        const int s = it % kUStages;
        if (it >= kUStages && !mbar_wait_bounded(&empty[s], ((it / kUStages) - 1) & 1, abort_flag, p.wait_ns)) {
          *abort_flag = 1;
          break;
        }
        unsigned char* a_dst = stages + (size_t)s * kStage;
        const int k = k0 + it * kUChunk;
        mbar_arrive_expect_tx(&full[s], kStage);
        if constexpr (kGemv) {
          // 64 rows of W (the reduction) x 128 columns, as two 64-column boxes
          tma_load_2d(a_dst, &map_a, j0, k, &full[s]);
          tma_load_2d(a_dst + kUABytes / 2, &map_a, j0 + 64, k, &full[s]);
          tma_load_2d(a_dst + kUABytes, &map_b0, k, 0, &full[s]);
          tma_load_2d(a_dst + kUABytes + kUBBytes, &map_b1, k, 0, &full[s]);
        } else {
          tma_load_2d(a_dst, &map_a, k, j0, &full[s]);
          tma_load_2d(a_dst + kUABytes, &map_b0, k, 0, &full[s]);
        }
        ++issued;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      for (int it = 0; it < n_it; ++it) {
        const int s = it % kUStages;
        if (!mbar_wait_bounded(&full[s], (it / kUStages) & 1, abort_flag, p.wait_ns)) {
          *abort_flag = 1;
          break;
        }
        tmem_fence_after();
        const uint32_t a_addr = smem_u32(stages + (size_t)s * kStage);
        const uint32_t b_addr = a_addr + kUABytes;
#pragma unroll
        for (int kk = 0; kk < kUChunk / 16; ++kk) {  // 16 inputs per instruction
          if constexpr (kGemv) {
            // 16 rows of W = two 8-row atoms (2 KB); the two column boxes 8 KB apart
            const uint64_t ad = sw128_mn_desc(a_addr + kk * 2048, kUABytes / 2, 1024);
            umma_bf16(tmem, ad, sw128_desc(b_addr + kk * 32), (it > 0 || kk > 0) ? 1u : 0u, kUIdescMN);
            umma_bf16(tmem, ad, sw128_desc(b_addr + kUBBytes + kk * 32), 1u, kUIdescMN);
          } else {
            umma_bf16(tmem, sw128_desc(a_addr + kk * 32), sw128_desc(b_addr + kk * 32),
                      (it > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&empty[s]);  // the stage is free once these MMAs have read it
      }
      umma_commit(&done);  // every MMA issued above has completed
    }
  }
  __syncwarp();

  // ------------------------------------------------------------------ epilogue
  // all MMAs (and so all their smem reads) are complete once `done` fires
  bool ok = mbar_wait_bounded(&done, 0, nullptr, p.wait_ns);
  tmem_fence_after();
  __syncwarp();  // tcgen05.ld is .aligned: the whole warp issues it together
  float v[kUTokens];
  {
    uint32_t r[kUTokens];
    const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int c = 0; c < kUTokens; ++c) v[c] = n_it > 0 ? __uint_as_float(r[c]) : 0.f;
  }
  if (!ok) *abort_flag = 1;
  __syncthreads();
  if (*abort_flag && warp == 0 && lane == 0) {
    // let every copy this CTA armed land before its shared memory goes away
    for (int it = max(0, issued - kUStages); it < issued; ++it)
      mbar_wait_bounded(&full[it % kUStages], (it / kUStages) & 1, nullptr, p.wait_ns);
    report(p.dev_status, LAROSA_DEV_TIMEOUT);
  }
  const bool abort = *abort_flag != 0;

  // this CTA's partial tile, [token][row], in the (now idle) first stage
  float* part = reinterpret_cast<float*>(stages);
#pragma unroll
  for (int c = 0; c < kUTokens; ++c) part[c * kURows + tid] = v[c];
  tmem_fence_before();
  __syncthreads();
  if (warp == 2) {
    tmem_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kUTmemCols)
                 : "memory");
  }
  cluster.sync();
  if (!abort) {
    // rank q of the S splits adds rows [q * 128 / S, (q + 1) * 128 / S) over
    // the splits in rank order
    const int S = static_cast<int>(cluster.num_blocks());
    const int q = static_cast<int>(cluster.block_rank());
    const int r0 = q * kURows / S, r1 = (q + 1) * kURows / S;
    const int n = (r1 - r0) * p.M;
    for (int e = tid; e < n; e += kUThreads) {
      const int m = e / (r1 - r0);
      const int row = r0 + (e - m * (r1 - r0));
      float s = 0.f;
      for (int qq = 0; qq < S; ++qq) s += cluster.map_shared_rank(part, qq)[m * kURows + row];
      if (j0 + row < p.n_out) p.y[(size_t)m * p.n_out + j0 + row] = s;
    }
  }
  cluster.sync();  // no CTA leaves while another may still read its partial tile
}

// The driver's tensor-map encoder, looked up through the runtime so that the
// library does not link against the driver library itself.
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encoder() {
  static EncodeTiled fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  }
  return fn;
}

// A 2-D bf16 tensor map of a row-major [rows x cols] matrix, box
// [box_rows x 64 columns], 128-byte swizzle; rows past `rows` read as zero.
bool make_map(CUtensorMap* map, const void* base, int rows, int cols, int box_rows) {
  const EncodeTiled enc = encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kUChunk, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


template <bool kGemv>
cudaError_t launch_umma(const CUtensorMap& map_a, const CUtensorMap& map_b0, const CUtensorMap& map_b1,
                        float* y, int M, int n_in, int n_out, int sms, int* dev_status, cudaStream_t stream) {
  const int tiles = (n_out + kURows - 1) / kURows;
  const int chunks = (n_in + kUChunk - 1) / kUChunk;
  // splits of the reduction: about two CTAs per SM in all, each at least
  // kUStages chunks long, at most a portable cluster of 8
  int S = 1;
  while (S < 8 && tiles * S * 2 <= 2 * sms && chunks / (S * 2) >= kUStages) S *= 2;
  const int k_per_split = ((chunks + S - 1) / S) * kUChunk;
  UParams p{y, n_out, M, k_per_split, n_in, dev_status, wait_limit_ns()};
  const size_t smem = (size_t)kUStages * stage_bytes<kGemv>() + 1024;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  static bool configured[64] = {};  // per device: the attribute belongs to a device's context
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(umma_kernel<kGemv>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(S, tiles, 1);
  cfg.blockDim = dim3(kUThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, umma_kernel<kGemv>, map_a, map_b0, map_b1, p);
}

// hi[m][i] = bf16(c), lo[m][i] = bf16(c - hi) for c = coef[m][i]: the head
// and tail that the tensor cores multiply as two bf16 operands (about 16
// significant bits of each fp32 coefficient kept).  Also returns the row
// bitmap the scatter kernel set to zero, as every call leaves it.
__global__ void __launch_bounds__(256) split_coef_kernel(const float* __restrict__ coef, int n,
                                                         __nv_bfloat16* __restrict__ hi,
                                                         __nv_bfloat16* __restrict__ lo, unsigned* bitmap,
                                                         int n_words) {
  pdl_wait();
  pdl_launch_dependents();
  for (int i = blockIdx.x * 256 + threadIdx.x; i < n_words; i += gridDim.x * 256) bitmap[i] = 0u;
  for (int i = blockIdx.x * 256 + threadIdx.x; i < n; i += gridDim.x * 256) {
    const float c = coef[i];
    const __nv_bfloat16 h = __float2bfloat16_rn(c);
    hi[i] = h;
    lo[i] = __float2bfloat16_rn(c - __bfloat162float(h));
  }
}

}  // namespace

bool rot_umma_applies(int M, int n_in, int n_out) {
  return M >= 8 && M <= kUTokens && n_in % kUChunk == 0 && n_out % 8 == 0 && n_in >= kUChunk;
}

cudaError_t launch_rot_umma(const void* A, const void* x, float* y, int M, int n_in, int n_out, int sms,
                            int* dev_status, cudaStream_t stream) {
  CUtensorMap map_a, map_x;
  if (!make_map(&map_a, A, n_out, n_in, kURows) || !make_map(&map_x, x, M, n_in, kUTokens))
    return cudaErrorInvalidValue;
  return launch_umma<false>(map_a, map_x, map_x, y, M, n_in, n_out, sms, dev_status, stream);
}

bool umma_gemv_applies(int M, int d_in, int d_out) {
  return M >= 8 && M <= kUTokens && d_in % 8 == 0 && d_out % 8 == 0 && d_in >= kUChunk;
}

cudaError_t launch_umma_gemv(const void* W, const float* coef, __nv_bfloat16* coef_hi, __nv_bfloat16* coef_lo,
                             unsigned* bitmap, float* y, int M, int d_in, int d_out, int sms, int* dev_status,
                             cudaStream_t stream) {
  {
    const int n = M * d_in;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(std::max(1, std::min((n + 255) / 256, 2 * sms)), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int n_words = (d_in + 31) / 32;
    cudaError_t e = cudaLaunchKernelEx(&cfg, split_coef_kernel, coef, n, coef_hi, coef_lo, bitmap, n_words);
    if (e != cudaSuccess) return e;
  }
  CUtensorMap map_w, map_hi, map_lo;
  // W: d_in rows (the reduction) of d_out columns, boxes of 64 rows x 64 columns
  if (!make_map(&map_w, W, d_in, d_out, kUChunk) || !make_map(&map_hi, coef_hi, M, d_in, kUTokens) ||
      !make_map(&map_lo, coef_lo, M, d_in, kUTokens))
    return cudaErrorInvalidValue;
  return launch_umma<true>(map_w, map_hi, map_lo, y, M, d_in, d_out, sms, dev_status, stream);
}

}  // namespace larosa
