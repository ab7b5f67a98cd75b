// Products of 2 to 16 bf16 tokens on the fifth-generation tensor cores
// (sm_100a), both HBM-bound streams of a bf16 matrix:
//
//   row-dot  y[m][j] = sum_i x[m][i] * A[j][i], A row-major [n_out x n_in]:
//            the rotation x_rot = x . Q reads Q through A = Q^T ("La RoSA"
//            summary, 方法详解 / 技术框架: each layer's input activation is
//            multiplied by that layer's orthogonal matrix); the dense
//            baseline reads W in torch.nn.Linear layout;
//   GEMV     y[m][c] = sum_r coef[m][r] * W[r][c], W row-major [d_in x d_out]:
//            the sparse linear of several tokens over every row of the
//            counter-rotated weight (abstract: activation sparsity reduces
//            memory transfers; from a few tokens on, the rows some token
//            keeps are nearly all of them), each token's coefficient row
//            zero where it did not keep the row.
//
// One MMA tile is 128 output elements (M) by the token slots (N), over 16
// inputs (K) per instruction; the accumulators live in TMEM.  A CTA owns
// kCols output elements and one split of the reduction:
//   * one thread streams chunks of the matrix and of the token operand into
//     a ring of shared-memory stages with 2-D TMA copies in the 128-byte
//     swizzled layout the MMA reads (elements past the matrix arrive as
//     zeros);
//   * one thread issues tcgen05.mma (bf16 in, fp32 accumulate) and returns
//     each stage to the producer with tcgen05.commit;
//   * all four warps read the accumulators out of TMEM (warp w owns TMEM
//     lanes 32w..32w+31) into shared memory.
// The row-dot's A tile is K-major (rows of A are the reduction's inputs); a
// stage takes kKB 64-input boxes of 128 rows, so each row is read kKB x 128
// contiguous bytes at a time.  The GEMV's W tile is MN-major (W's rows are
// the reduction); a stage takes 64 rows of kNB x 128 columns, i.e. kNB x 256
// contiguous bytes per row, one M = 128 accumulator per 128 columns.  Its
// fp32 coefficients enter as a bf16 head and tail (about 16 significant bits
// kept): one N = 32 MMA multiplies both, heads in accumulator columns 0..15
// and tails in 16..31, added in the epilogue.
// The splits of one tile form a thread-block cluster and add their partial
// tiles through distributed shared memory in rank order, so the result does
// not depend on timing.  Every mbarrier wait gives up after the wait limit;
// the CTA then lets its copies and MMAs land, frees its TMEM and writes
// nothing.
#include <cooperative_groups.h>
#include <cuda.h>

#include <algorithm>
#include <cmath>

#include "coef.cuh"
#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace cg = cooperative_groups;

namespace larosa {
namespace {

constexpr int kUThreads = 128;  // 4 warps: TMEM lanes 0..127
constexpr int kUTokens = 16;    // token slots
constexpr int kUBox = 64;       // elements of a 128-byte swizzle row (bf16)

// Compile-time shape of one kernel: the row-dot (kGemv false) or the GEMV
// with kNB 128-column accumulators per CTA.
template <bool kGemv, int kNB>
struct UCfg;
template <>
struct UCfg<false, 1> {
  static constexpr int kNB = 1;      // one 128-row accumulator per CTA
  static constexpr int kKB = 2;      // 64-input boxes per stage: 256 contiguous bytes per row
  static constexpr int kStages = 3;  // 3 x 36 KB: two CTAs per SM
  static constexpr int kN = kUTokens;
};
template <int NB>
struct UCfg<true, NB> {
  static constexpr int kNB = NB;     // 128-column accumulators per CTA: 256 NB contiguous bytes per row
  static constexpr int kKB = 1;      // one 64-row box per stage
  // 2 x 20 KB: four CTAs per SM, or 3 x 36 KB: two.  More CTAs issuing
  // copies beat deeper rings: at 16 tokens on the LLaMA2-7B groups, 128
  // columns with two stages (4 CTAs per SM) were 5 % faster than 256 columns
  // with three (2 per SM), 128 with three (3 per SM) 1.5 %, 256 with two
  // (3 per SM) 1.5 % slower.
  static constexpr int kStages = NB == 1 ? 2 : 3;
  static constexpr int kN = 2 * kUTokens;          // heads, then tails
};

template <bool kGemv, int kNB>
struct UShape {
  using C = UCfg<kGemv, kNB>;
  static constexpr int kCols = 128 * C::kNB;        // output elements per CTA
  static constexpr int kChunk = kUBox * C::kKB;     // reduction inputs per stage
  static constexpr uint32_t kABytes = (uint32_t)kCols * kChunk * 2;
  static constexpr uint32_t kBBytes = (uint32_t)C::kN * kChunk * 2;
  static constexpr uint32_t kStage = kABytes + kBBytes;
  static constexpr int kTmemCols = C::kNB * C::kN <= 32 ? 32 : C::kNB * C::kN <= 64 ? 64 : 128;
  static constexpr size_t kSmem = (size_t)C::kStages * kStage + 1024;  // + alignment slack
  static_assert(kStage % 1024 == 0, "swizzled stages stay 1024-byte aligned");
  static_assert((size_t)kUTokens * kCols * 4 <= (size_t)C::kStages * kStage, "partials fit the ring");
};

struct UParams {
  float* y;
  __nv_bfloat16* hl_out;  // not null: the result as bf16 head/tail rows [2 x M x n_out] instead of y
  int accumulate;         // 1: y += result
  int n_out;
  int M;
  int k_per_split;  // inputs per split, a multiple of the stage's chunk
  int n_in;
  int* dev_status;
  unsigned long long wait_ns;  // limit of every mbarrier wait
};

// kGemv = false: y[m][j] = sum_i x[m][i] A[j][i] (A = map_a, K-major rows;
// x = map_b0).  kGemv = true: y[m][c] = sum_r coef[m][r] W[r][c] (W = map_a,
// read MN-major; the coefficients' bf16 heads map_b0 and tails map_b1).
template <bool kGemv, int kNB>
__global__ void __launch_bounds__(kUThreads, 1)
    umma_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b0,
                const __grid_constant__ CUtensorMap map_b1, const UParams p) {
  using C = UCfg<kGemv, kNB>;
  using S = UShape<kGemv, kNB>;
  constexpr int kStages = C::kStages;
  constexpr uint32_t kId = tc::idesc(C::kN, kGemv);
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // the swizzled stages need 1024-byte alignment
  unsigned char* stages = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[kStages], empty[kStages], done;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x;  // = rank in the cluster
  const int j0 = blockIdx.y * S::kCols;
  const int k0 = split * p.k_per_split;
  const int k1 = min(p.n_in, k0 + p.k_per_split);
  const int n_it = k1 > k0 ? (k1 - k0 + S::kChunk - 1) / S::kChunk : 0;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&done, 1);
    s_abort = 0;
    mbar_init_fence();
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(S::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc::tmem_fence_before();
  __syncthreads();
  tc::tmem_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;

  // The matrix tiles of one stage (Q^T or W: weights, never written by a
  // kernel that lets this one launch before it ends) and its token operand
  // (x or the coefficient rows, which the previous kernel on the stream may
  // still be writing), both completing on full[s].
  auto load_a = [&](int it) {
    const int s = it % kStages;
    unsigned char* a_dst = stages + (size_t)s * S::kStage;
    const int k = k0 + it * S::kChunk;
    mbar_arrive_expect_tx(&full[s], S::kStage);  // A and B bytes together
    if constexpr (kGemv) {
      // 64 rows of W (the reduction) x kCols columns, as 64-column boxes
#pragma unroll
      for (int j = 0; j < 2 * C::kNB; ++j) tc::tma_load_2d(a_dst + j * 8192, &map_a, j0 + 64 * j, k, &full[s]);
    } else {
      // kKB boxes of 128 rows of A x 64 inputs
#pragma unroll
      for (int kb = 0; kb < C::kKB; ++kb) tc::tma_load_2d(a_dst + kb * 16384, &map_a, k + kUBox * kb, j0, &full[s]);
    }
  };
  auto load_b = [&](int it) {
    const int s = it % kStages;
    unsigned char* b_dst = stages + (size_t)s * S::kStage + S::kABytes;
    const int k = k0 + it * S::kChunk;
    if constexpr (kGemv) {
      tc::tma_load_2d(b_dst, &map_b0, k, 0, &full[s]);
      tc::tma_load_2d(b_dst + kUTokens * kUBox * 2, &map_b1, k, 0, &full[s]);
    } else {
#pragma unroll
      for (int kb = 0; kb < C::kKB; ++kb)
        tc::tma_load_2d(b_dst + kb * (kUTokens * kUBox * 2), &map_b0, k + kUBox * kb, 0, &full[s]);
    }
  };

  int issued = 0;
  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- producer
    // the first stages' matrix tiles stream while the previous kernel on the
    // stream finishes; the token operand only after it has completed
    const int pre = min(n_it, kStages);
    for (int it = 0; it < pre; ++it) load_a(it);
    pdl_wait();
    pdl_launch_dependents();
    for (int it = 0; it < pre; ++it) load_b(it);
    issued = pre;
    for (int it = pre; it < n_it; ++it) {
      const int s = it % kStages;
      if (!mbar_wait_bounded(&empty[s], ((it / kStages) - 1) & 1, abort_flag, p.wait_ns)) {
        *abort_flag = 1;
        break;
      }
      load_a(it);
      load_b(it);
      ++issued;
    }
  } else {
    pdl_wait();  // the epilogue writes y, which the previous kernel may still read
    pdl_launch_dependents();
  }
  if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      for (int it = 0; it < n_it; ++it) {
        const int s = it % kStages;
        if (!mbar_wait_bounded(&full[s], (it / kStages) & 1, abort_flag, p.wait_ns)) {
          *abort_flag = 1;
          break;
        }
        tc::tmem_fence_after();
        const uint32_t a_addr = smem_u32(stages + (size_t)s * S::kStage);
        const uint32_t b_addr = a_addr + S::kABytes;
        if constexpr (kGemv) {
#pragma unroll
          for (int kk = 0; kk < kUBox / 16; ++kk) {  // 16 rows of W per instruction: two 8-row atoms
            const uint64_t bd = tc::sw128_desc(b_addr + kk * 32);
#pragma unroll
            for (int nb = 0; nb < C::kNB; ++nb) {
              // columns 128 nb .. 128 nb + 127: two 64-column boxes 8 KB apart
              const uint64_t ad = tc::sw128_mn_desc(a_addr + nb * 16384 + kk * 2048, 8192, 1024);
              tc::umma_bf16(tmem + nb * C::kN, ad, bd, (it > 0 || kk > 0) ? 1u : 0u, kId);
            }
          }
        } else {
#pragma unroll
          for (int kb = 0; kb < C::kKB; ++kb)
#pragma unroll
            for (int kk = 0; kk < kUBox / 16; ++kk)  // 16 inputs per instruction
              tc::umma_bf16(tmem, tc::sw128_desc(a_addr + kb * 16384 + kk * 32),
                        tc::sw128_desc(b_addr + kb * (kUTokens * kUBox * 2) + kk * 32),
                        (it > 0 || kb > 0 || kk > 0) ? 1u : 0u, kId);
        }
        tc::umma_commit(&empty[s]);  // the stage is free once these MMAs have read it
      }
      tc::umma_commit(&done);  // every MMA issued above has completed
    }
  }
  __syncwarp();

  // ------------------------------------------------------------------ epilogue
  // all MMAs (and so all their shared-memory reads) are complete once `done` fires
  const bool ok = mbar_wait_bounded(&done, 0, nullptr, p.wait_ns);
  tc::tmem_fence_after();
  __syncwarp();  // tcgen05.ld is .aligned: the whole warp issues it together
  if (!ok) *abort_flag = 1;
  __syncthreads();
  if (*abort_flag && warp == 0 && lane == 0) {
    // let every copy this CTA armed land before its shared memory goes away
    for (int it = max(0, issued - kStages); it < issued; ++it)
      mbar_wait_bounded(&full[it % kStages], (it / kStages) & 1, nullptr, p.wait_ns);
    report(p.dev_status, LAROSA_DEV_TIMEOUT);
  }
  __syncthreads();
  const bool abort = *abort_flag != 0;

  // this CTA's partial tile, [token][element], in the (now idle) ring
  float* part = reinterpret_cast<float*>(stages);
  const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll
  for (int nb = 0; nb < C::kNB; ++nb) {
    float v[16];
    tc::tmem_ld16(lane_base + nb * C::kN, v);
    if constexpr (kGemv) {
      float t[16];
      tc::tmem_ld16(lane_base + nb * C::kN + kUTokens, t);  // the tails' products
#pragma unroll
      for (int c = 0; c < 16; ++c) v[c] += t[c];
    }
#pragma unroll
    for (int c = 0; c < kUTokens; ++c) part[c * S::kCols + nb * 128 + tid] = n_it > 0 ? v[c] : 0.f;
  }
  tc::tmem_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc::tmem_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(S::kTmemCols)
                 : "memory");
  }
  cluster.sync();
  if (!abort) {
    // rank q of the R splits adds elements [q * kCols / R, (q + 1) * kCols / R)
    // over the splits in rank order
    const int R = static_cast<int>(cluster.num_blocks());
    const int q = static_cast<int>(cluster.block_rank());
    const int r0 = q * S::kCols / R, r1 = (q + 1) * S::kCols / R;
    const int n = (r1 - r0) * p.M;
    for (int e = tid; e < n; e += kUThreads) {
      const int m = e / (r1 - r0);
      const int row = r0 + (e - m * (r1 - r0));
      float s = 0.f;
      for (int qq = 0; qq < R; ++qq) s += cluster.map_shared_rank(part, qq)[m * S::kCols + row];
      const int j = j0 + row;
      if (j < p.n_out) {
        if (p.hl_out != nullptr) {
          // the next product's coefficients: heads in rows 0 .. M-1, tails in M .. 2M-1
          __nv_bfloat16 h, t;
          split_head_tail(s, &h, &t);
          p.hl_out[(size_t)m * p.n_out + j] = h;
          p.hl_out[(size_t)(p.M + m) * p.n_out + j] = t;
        } else if (p.accumulate) {
          p.y[(size_t)m * p.n_out + j] += s;
        } else {
          p.y[(size_t)m * p.n_out + j] = s;
        }
      }
    }
  }
  cluster.sync();  // no CTA leaves while another may still read its partial tile
}

// Splits of the reduction per tile, for `slots` co-resident CTAs: the S in
// 1..8 (at most one split per chunk) that minimises the number of full
// waves times the chunks one CTA streams, i.e. the time of the slowest CTA
// when every wave runs at the same speed; ties go to the smaller S (fewer
// partial tiles to add).
int pick_splits(int tiles, int chunks, int slots) {
  int best_S = 1;
  long long best = -1;
  for (int S = 1; S <= 8 && S <= chunks; ++S) {
    const long long ctas = (long long)tiles * S;
    const long long waves = (ctas + slots - 1) / slots;
    const long long t = waves * ((chunks + S - 1) / S);
    if (best < 0 || t < best) {
      best = t;
      best_S = S;
    }
  }
  return best_S;
}

// Per device (a function attribute belongs to a device's context): SMs and
// CTAs per SM of one kernel.  The CTAs an SM holds are set by shared memory
// (the occupancy query reports one for these kernels, while two run side by
// side).
struct UDev {
  int sms = 0;
  int per_sm = 0;
};

template <bool kGemv, int kNB>
cudaError_t umma_dev(int dev, UDev* out) {
  using S = UShape<kGemv, kNB>;
  static UDev st[64];
  UDev& d = st[dev];
  if (d.per_sm == 0) {
    int smem_sm = 0, reserved = 0, sms = 0;
    cudaError_t e = cudaFuncSetAttribute(umma_kernel<kGemv, kNB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)S::kSmem);
    // all of the unified L1/shared storage as shared memory, so that two CTAs fit
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(umma_kernel<kGemv, kNB>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    if (e != cudaSuccess) return e;
    d.sms = sms;
    // + the static shared memory (barriers, flags: under 1 KB)
    d.per_sm = std::max(1, std::min(4, smem_sm / (int)(S::kSmem + 1024 + reserved)));
  }
  *out = d;
  return cudaSuccess;
}

template <bool kGemv, int kNB>
cudaError_t launch_umma(const CUtensorMap& map_a, const CUtensorMap& map_b0, const CUtensorMap& map_b1,
                        float* y, int M, int n_in, int n_out, int R, int* dev_status, cudaStream_t stream,
                        bool accumulate = false, __nv_bfloat16* hl_out = nullptr) {
  using S = UShape<kGemv, kNB>;
  const int tiles = (n_out + S::kCols - 1) / S::kCols;
  const int chunks = (n_in + S::kChunk - 1) / S::kChunk;
  const int k_per_split = ((chunks + R - 1) / R) * S::kChunk;
  UParams p{y, hl_out, accumulate ? 1 : 0, n_out, M, k_per_split, n_in, dev_status, wait_limit_ns()};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(R, tiles, 1);
  cfg.blockDim = dim3(kUThreads, 1, 1);
  cfg.dynamicSmemBytes = S::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = R;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, umma_kernel<kGemv, kNB>, map_a, map_b0, map_b1, p);
}

// Splits and the modelled time of one shape for a kernel (see pick_splits).
template <bool kGemv, int kNB>
cudaError_t plan_umma(int n_in, int n_out, int* R, long long* t) {
  using S = UShape<kGemv, kNB>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  UDev d;
  e = umma_dev<kGemv, kNB>(dev, &d);
  if (e != cudaSuccess) return e;
  const int tiles = (n_out + S::kCols - 1) / S::kCols;
  const int chunks = (n_in + S::kChunk - 1) / S::kChunk;
  const int slots = d.sms * d.per_sm;
  const int forced = split_k_override();  // larosa_set_split_k
  *R = forced > 0 ? std::min(forced, chunks) : pick_splits(tiles, chunks, slots);
  // bytes of the slowest wave's CTAs, in 64 x 128 bf16 units
  const long long ctas = (long long)tiles * *R;
  *t = (ctas + slots - 1) / slots * ((chunks + *R - 1) / *R) * S::kChunk / kUBox * kNB;
  return cudaSuccess;
}

}  // namespace

// From two tokens on the tensor-core kernels take the batch path: their cost
// does not depend on the token count (16 slots, the unused ones zero), and
// they stream faster than the CUDA-core kernels (the row-dot of 2 tokens,
// mma.sync for 3-7, the row-streaming GEMV over the union of kept rows) even
// where the union of two tokens' kept rows is only 84 % of the weight.
constexpr int kUMinTokens = 2;

bool rot_umma_applies(int M, int n_in, int n_out) {
  return M >= kUMinTokens && M <= kUTokens && n_in % kUBox == 0 && n_out % 8 == 0 && n_in >= kUBox;
}

cudaError_t launch_rot_umma(const void* A, const void* x, float* y, int M, int n_in, int n_out,
                            int* dev_status, cudaStream_t stream) {
  CUtensorMap map_a, map_x;
  if (!tc::make_map(&map_a, A, n_out, n_in, 128) || !tc::make_map(&map_x, x, M, n_in, kUTokens))
    return cudaErrorInvalidValue;
  int R = 1;
  long long t = 0;
  cudaError_t e = plan_umma<false, 1>(n_in, n_out, &R, &t);
  if (e != cudaSuccess) return e;
  return launch_umma<false, 1>(map_a, map_x, map_x, y, M, n_in, n_out, R, dev_status, stream);
}

bool umma_gemv_applies(int M, int d_in, int d_out) {
  return M >= kUMinTokens && M <= kUTokens && d_in % 8 == 0 && d_out % 8 == 0 && d_in >= kUBox;
}

// The dense product streams every row of W; the row-streaming GEMV only the
// union of the kept rows, but with a fixed cost of about 20 us (coefficient
// scatter, union, its own ramp) and a lower rate per byte, worse still with
// the mma.sync consumers it uses from 8 tokens.  Measured on a 4096 x 22016
// weight (us per call, dense / union): 2 tokens keeping 15 % 31.8 / 24.6,
// 30 % 32.6 / 32.6 (the union then covers 51 %); 4 tokens keeping 5 %
// 32.5 / 29.9, 10 % 32.5 / 35.4; 8 tokens keeping 3 % 33.0 / 39.8; 16 tokens
// keeping 5 % 34.8 / 128.  So the union is streamed only where few tokens
// keep few rows.
bool umma_gemv_pays(int M, int d_in, int d_out, int K) {
  if (!umma_gemv_applies(M, d_in, d_out) || K <= 0) return false;
  const double kept = 1.0 - std::pow(1.0 - static_cast<double>(K) / d_in, M);
  const double union_below = M <= 2 ? 0.3 : M <= 4 ? 0.2 : 0.0;
  return kept >= union_below;
}

// Column tiles of 128 (one accumulator) with the two-stage ring above, four
// CTAs per SM: measured on the LLaMA2-7B groups at 2 to 16 tokens they beat
// tiles of 256 at two CTAs per SM on every batch size; 0 would choose per
// shape by the wave model.
constexpr int kGemvNB = 1;

cudaError_t launch_umma_gemv(const void* W, const __nv_bfloat16* hl, float* y, int M, int d_in, int d_out,
                             int* dev_status, cudaStream_t stream, bool accumulate, __nv_bfloat16* hl_out) {
  CUtensorMap map_w, map_hi, map_lo;
  // W: d_in rows (the reduction) of d_out columns, boxes of 64 rows x 64 columns
  if (!tc::make_map(&map_w, W, d_in, d_out, kUBox) || !tc::make_map(&map_hi, hl, M, d_in, kUTokens) ||
      !tc::make_map(&map_lo, hl + (size_t)M * d_in, M, d_in, kUTokens))
    return cudaErrorInvalidValue;
  int R1 = 1, R2 = 1;
  long long t1 = 0, t2 = 0;
  cudaError_t e = plan_umma<true, 1>(d_in, d_out, &R1, &t1);
  if (e == cudaSuccess) e = plan_umma<true, 2>(d_in, d_out, &R2, &t2);
  if (e != cudaSuccess) return e;
  const bool wide = kGemvNB == 2 || (kGemvNB == 0 && t2 <= t1);
  if (wide)
    return launch_umma<true, 2>(map_w, map_hi, map_lo, y, M, d_in, d_out, R2, dev_status, stream, accumulate,
                                hl_out);
  return launch_umma<true, 1>(map_w, map_hi, map_lo, y, M, d_in, d_out, R1, dev_status, stream, accumulate,
                              hl_out);
}

}  // namespace larosa
