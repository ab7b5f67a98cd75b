// Row-streaming GEMV for sm_100a: the sparse linear of several tokens where
// the tcgen05 product does not apply (fp32 weights, d_in < 64) and after a
// threshold selection of several tokens (over the union of their kept
// rows), the factor GEMVs of the sparse + low-rank mode for several tokens,
// and the one-token fallbacks (a kept list longer than the cluster gather
// holds, the no-allocation entry point when its gather plan does not fit).
//
//   y[m][c] = sum_r coef(m, r) * W[row(r)][c]
//
// The LaRoSA saving comes from reading only the K kept rows of the
// counter-rotated weight (La RoSA abstract: activation sparsity reduces memory
// transfers).  With the weight row-major [d_in x d_out], every kept row is
// one contiguous run, so the kernel is a row gather that is bound by HBM
// bandwidth.  Design:
//
//  * grid = (splits, column tiles).  A CTA owns Wc output columns and a
//    contiguous range of the row list; clusters of C CTAs along the splits
//    reduce their partial sums through distributed shared memory.
//  * One producer warp streams the CTA's row segments (Wc elements each) into
//    a 6-stage shared-memory ring with 1-D bulk copies (cp.async.bulk, the
//    TMA engine) completing on per-stage mbarriers; 8 consumer warps hold
//    fp32 accumulators for CPT columns x MT tokens per thread and release
//    each stage through an "empty" mbarrier.
//  * From 8 tokens on (bf16 weights, fp32 coefficients) the consumers use
//    the tensor cores instead (mma.sync m16n8k16): tokens are the MMA's
//    rows, 8 output columns its columns, 16 weight rows its reduction.  A
//    16 x 8 weight tile is read from the ring with ldmatrix.trans (ring rows
//    padded by 16 bytes so that its 8-row reads do not share banks); each
//    fp32 coefficient is split into a bf16 head and a bf16 tail, two MMAs
//    per tile, so the products keep about 16 bits of the coefficient.
//    Consumer warp w owns the 8-column blocks w, w + 8, ... of the tile.
//  * Reduction order is fixed (rows in list order per thread, row groups in
//    order, cluster ranks in order, cluster partials in order), so results
//    are bitwise reproducible for a given launch geometry.
//  * Across clusters of one column tile: partials go to the workspace and the
//    last-arriving CTA of each column slice (an atomic ticket, no waiting)
//    sums them and resets the ticket to zero.
#include <cooperative_groups.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace larosa {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;  // + one producer warp
constexpr int kStages = 6;
constexpr int kStageBytes = 16384;
constexpr int kHeaderBytes = 256;  // mbarriers + flags

struct Params {
  const void* W;
  int d_out;
  int row_bound;
  const int32_t* rows;
  int n_rows;
  const int* n_rows_dev;
  const void* coef;
  int coef_ld;
  int coef_by_row;
  int M;
  float* y;
  int y_ld;
  float* partials;
  unsigned* tickets;
  int col_tile;
  int tpr;
  int rows_per_stage;
  int pitch;  // bytes between two rows of a stage
  int max_rpc;
  int* dev_status;
  unsigned long long wait_ns;  // limit of every mbarrier wait
};

template <int MT, int CPT>
struct Acc {
  float v[MT][CPT];
};

constexpr int kMmaBlocks = 8;                           // 8-column blocks per consumer warp
constexpr int kMmaTile = 8 * kMmaBlocks * kConsumerWarps;  // columns of a tensor-core tile

// bf16 pair {lo, hi} of two floats, round to nearest even
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// head (bf16 of c) and tail (bf16 of c - head) of two coefficients
__device__ __forceinline__ void split_pair(float c0, float c1, uint32_t* head, uint32_t* tail) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(c0, c1);
  const float2 hf = __bfloat1622float2(h);
  *head = *reinterpret_cast<const uint32_t*>(&h);
  *tail = pack_bf16x2(c0 - hf.x, c1 - hf.y);
}

__device__ __forceinline__ void ldmatrix_x2_trans(uint32_t* b0, uint32_t* b1, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(*b0), "=r"(*b1)
               : "r"(addr));
}

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <typename Tw, typename Tc, int MT, int CPT, bool kMma>
__global__ void __launch_bounds__(kThreads, (MT <= 2 ? 2 : 1)) rowstream_gemv_kernel(const Params p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kStages;
  int* flags = reinterpret_cast<int*>(empty + kStages);  // [0] abort, [1] ticket
  int32_t* row_ids = reinterpret_cast<int32_t*>(smem + kHeaderBytes);
  float* coef_s = reinterpret_cast<float*>(row_ids + p.max_rpc);
  unsigned char* stages = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(coef_s + MT * p.max_rpc) + 1023) & ~uintptr_t(1023));

  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int split = blockIdx.x;
  const int splits = gridDim.x;
  const int tile = blockIdx.y;
  const int c0 = tile * p.col_tile;
  const int wc = min(p.col_tile, p.d_out - c0);
  volatile int* abort_flag = flags;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    flags[0] = 0;
    flags[1] = 0;
    mbar_init_fence();
  }
  __syncthreads();

  // Everything below may read what the previous kernel on the stream wrote.
  pdl_wait();
  pdl_launch_dependents();

  int n = p.n_rows;
  if (p.n_rows_dev != nullptr) n = max(0, min(n, *p.n_rows_dev));
  const int rps = (n + splits - 1) / splits;
  const int r0 = min(n, split * rps);
  const int nr = max(0, min(n, r0 + rps) - r0);

  // Row ids and coefficients of this CTA's rows, validated once.
  {
    bool bad = false;
    for (int r = tid; r < nr; r += kThreads) {
      int row = p.rows != nullptr ? p.rows[r0 + r] : r0 + r;
      const bool ok = static_cast<unsigned>(row) < static_cast<unsigned>(p.row_bound);
      bad |= !ok;
      row_ids[r] = ok ? row : 0;
      const int ci = p.coef_by_row ? row : r0 + r;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        float c = 0.f;
        if (ok && m < p.M) c = to_f32(static_cast<const Tc*>(p.coef)[(size_t)m * p.coef_ld + ci]);
        coef_s[m * p.max_rpc + r] = c;
      }
    }
    if (__syncthreads_or(bad) && tid == 0) report(p.dev_status, LAROSA_DEV_INDEX);
  }

  const int rstage = p.rows_per_stage;
  const int n_it = (nr + rstage - 1) / rstage;
  const uint32_t row_bytes = static_cast<uint32_t>(wc) * sizeof(Tw);
  const int pitch = p.pitch;

  Acc<MT, (kMma ? 1 : CPT)> acc;
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int v = 0; v < (kMma ? 1 : CPT); ++v) acc.v[m][v] = 0.f;
  float dacc[kMmaBlocks][4];  // tensor-core variant: D tiles of this warp's column blocks
#pragma unroll
  for (int bi = 0; bi < kMmaBlocks; ++bi)
#pragma unroll
    for (int e = 0; e < 4; ++e) dacc[bi][e] = 0.f;

  const int g = tid / p.tpr;                 // row group of a consumer thread
  const int n_groups = kConsumers / p.tpr;   // row groups
  const int col = (tid % p.tpr) * CPT;       // first column (within the tile)
  int issued = 0;                            // producer: stages armed

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    const uint64_t pol = l2_evict_first_policy();
    for (int it = 0; it < n_it; ++it) {
      const int s = it % kStages;
      if (it >= kStages) {
        int ok = 1;
        if (lane == 0) ok = mbar_wait_bounded(&empty[s], ((it / kStages) - 1) & 1, abort_flag, p.wait_ns);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) *abort_flag = 1;
          break;
        }
      }
      const int rows_here = min(rstage, nr - it * rstage);
      if (lane == 0) mbar_arrive_expect_tx(&full[s], rows_here * row_bytes);
      __syncwarp();
      unsigned char* dst = stages + s * kStageBytes;
      for (int j = lane; j < rows_here; j += 32) {
        const int row = row_ids[it * rstage + j];
        const unsigned char* src = static_cast<const unsigned char*>(p.W) +
                                   ((size_t)row * p.d_out + c0) * sizeof(Tw);
        bulk_copy_g2s(dst + j * pitch, src, row_bytes, &full[s], pol);
      }
      ++issued;
    }
  } else {
    // ------------------------------------------------------------ consumers
    const bool active = col < wc;
    for (int it = 0; it < n_it; ++it) {
      const int s = it % kStages;
      // every lane polls the barrier (acquiring the copied bytes); the warp
      // leaves together if any lane gave up
      const bool ok = mbar_wait_bounded(&full[s], (it / kStages) & 1, abort_flag, p.wait_ns);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      const int rows_here = min(rstage, nr - it * rstage);
      if constexpr (kMma) {
        const unsigned char* base = stages + s * kStageBytes;
        const float* cs = coef_s + it * rstage;
        const int gq = lane >> 2, q = lane & 3;
        const int nb8 = wc / 8;
        for (int kb = 0; kb < rows_here; kb += 16) {
          // A: coefficients of tokens gq, gq + 8 for rows kb + 2q + {0, 1}
          // and kb + 2q + {8, 9}, as bf16 head + tail (zero past the rows)
          auto cf = [&](int m, int r) {
            return (m < MT && kb + r < rows_here) ? cs[m * p.max_rpc + kb + r] : 0.f;
          };
          uint32_t h0, t0, h1, t1, h2, t2, h3, t3;
          split_pair(cf(gq, 2 * q), cf(gq, 2 * q + 1), &h0, &t0);
          split_pair(cf(gq + 8, 2 * q), cf(gq + 8, 2 * q + 1), &h1, &t1);
          split_pair(cf(gq, 2 * q + 8), cf(gq, 2 * q + 9), &h2, &t2);
          split_pair(cf(gq + 8, 2 * q + 8), cf(gq + 8, 2 * q + 9), &h3, &t3);
          // lanes 0..15 address the 16 weight rows of the tile (a row past
          // the stage's last repeats it: its coefficient is zero)
          const int rr = min(kb + (lane & 15), rows_here - 1);
#pragma unroll
          for (int bi = 0; bi < kMmaBlocks; ++bi) {
            const int blk = warp + bi * kConsumerWarps;
            if (blk < nb8) {  // warp-uniform
              uint32_t b0, b1;
              ldmatrix_x2_trans(&b0, &b1, smem_u32(base + rr * pitch + blk * 16));
              mma_16816(dacc[bi], h0, h1, h2, h3, b0, b1);
              mma_16816(dacc[bi], t0, t1, t2, t3, b0, b1);
            }
          }
        }
      } else if (active) {
        const unsigned char* base = stages + s * kStageBytes + col * sizeof(Tw);
        const float* cs = coef_s + it * rstage;
        for (int j = g; j < rows_here; j += n_groups) {
          float w[CPT];
          VecLoad<Tw, CPT>::load(base + j * pitch, w);
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const float c = cs[m * p.max_rpc + j];
#pragma unroll
            for (int v = 0; v < CPT; ++v) acc.v[m][v] = fmaf(c, w[v], acc.v[m][v]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }

  __syncthreads();
  if (*abort_flag) {
    // A wait gave up.  Let every bulk copy this CTA armed land before the
    // CTA's shared memory is released, then leave without writing outputs.
    if (warp == kConsumerWarps && lane == 0) {
      for (int it = max(0, issued - kStages); it < issued; ++it)
        mbar_wait_bounded(&full[it % kStages], (it / kStages) & 1, nullptr, p.wait_ns);
      report(p.dev_status, LAROSA_DEV_TIMEOUT);
    }
    __syncthreads();
    cluster.sync();
    cluster.sync();
    return;
  }

  // ---------------------------------------------------------------- epilogue
  // 1) row groups -> CTA partial, in shared memory (reusing the ring).
  float* red = reinterpret_cast<float*>(stages);
  // the CTA partial; the start of the ring later holds this rank's reduced
  // slice (outs), which must not overlap a partial a peer may still read
  float* part = red + (kMma ? 1 : n_groups) * MT * p.col_tile;
  if constexpr (kMma) {
    // D[token][column]: (gq, 2q), (gq, 2q + 1), (gq + 8, 2q), (gq + 8, 2q + 1)
    const int gq = lane >> 2, q = lane & 3;
    if (warp < kConsumerWarps) {
#pragma unroll
      for (int bi = 0; bi < kMmaBlocks; ++bi) {
        const int c = (warp + bi * kConsumerWarps) * 8 + 2 * q;
        if (c < wc) {
          if (gq < MT) {
            part[gq * p.col_tile + c] = dacc[bi][0];
            part[gq * p.col_tile + c + 1] = dacc[bi][1];
          }
          if (gq + 8 < MT) {
            part[(gq + 8) * p.col_tile + c] = dacc[bi][2];
            part[(gq + 8) * p.col_tile + c + 1] = dacc[bi][3];
          }
        }
      }
    }
  } else {
    if (warp < kConsumerWarps && col < wc) {
#pragma unroll
      for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int v = 0; v < CPT; ++v) red[(g * MT + m) * p.col_tile + col + v] = acc.v[m][v];
    }
    __syncthreads();
    for (int e = tid; e < MT * wc; e += kThreads) {
      const int m = e / wc;
      const int c = e - m * wc;
      float s = 0.f;
      for (int gg = 0; gg < n_groups; ++gg) s += red[(gg * MT + m) * p.col_tile + c];
      part[m * p.col_tile + c] = s;
    }
  }

  // 2) cluster ranks -> cluster partial: rank q owns columns [q*sl, q*sl+sl).
  cluster.sync();
  const int C = static_cast<int>(cluster.num_blocks());
  const int q = static_cast<int>(cluster.block_rank());
  const int sl = (p.col_tile + C - 1) / C;
  const int cs0 = min(wc, q * sl);
  const int cs1 = min(wc, cs0 + sl);
  const int ns = cs1 - cs0;
  const int n_clusters = splits / C;
  const int cl = split / C;
  const int Mw = min(p.M, MT);
  float* outs = red;  // this rank's reduced slice, [Mw][ns], reusing the ring
  for (int e = tid; e < Mw * ns; e += kThreads) {
    const int m = e / ns;
    const int c = cs0 + (e - m * ns);
    float s = 0.f;
    for (int qq = 0; qq < C; ++qq) s += cluster.map_shared_rank(part, qq)[m * p.col_tile + c];
    outs[e] = s;
  }
  cluster.sync();  // no rank leaves while another may still read its `part`

  if (n_clusters == 1) {
    for (int e = tid; e < Mw * ns; e += kThreads) {
      const int m = e / ns;
      const int c = cs0 + (e - m * ns);
      p.y[(size_t)m * p.y_ld + c0 + c] = outs[e];
    }
    return;
  }

  // 3) clusters of one column tile -> y, by the last CTA of each slice.
  // partials layout: [tile][cluster][m][col_tile]
  float* mine = p.partials + (((size_t)tile * n_clusters + cl) * Mw) * p.col_tile;
  for (int e = tid; e < Mw * ns; e += kThreads) {
    const int m = e / ns;
    const int c = cs0 + (e - m * ns);
    mine[(size_t)m * p.col_tile + c] = outs[e];
  }
  __threadfence();
  __syncthreads();
  unsigned* ticket = p.tickets + tile * C + q;
  if (tid == 0) flags[1] = static_cast<int>(atomicAdd(ticket, 1u));
  __syncthreads();
  if (flags[1] != n_clusters - 1) return;
  __threadfence();
  const float* all = p.partials + ((size_t)tile * n_clusters * Mw) * p.col_tile;
  for (int e = tid; e < Mw * ns; e += kThreads) {
    const int m = e / ns;
    const int c = cs0 + (e - m * ns);
    float s = 0.f;
    for (int k = 0; k < n_clusters; ++k) s += __ldcg(all + ((size_t)k * Mw + m) * p.col_tile + c);
    p.y[(size_t)m * p.y_ld + c0 + c] = s;
  }
  if (tid == 0) atomicExch(ticket, 0u);
}

// ------------------------------------------------------------------ host side

template <typename Tw, typename Tc, int MT, int CPT, bool kMma = false>
struct Inst {
  static void* fn() { return reinterpret_cast<void*>(&rowstream_gemv_kernel<Tw, Tc, MT, CPT, kMma>); }
};

// bf16 weights and fp32 coefficients from 8 tokens on: the tensor-core
// consumers (at 4 tokens the FMA consumers with their wider tiles measured
// faster)
bool uses_mma(Elem w, Elem c, int MT) { return w == Elem::BF16 && c == Elem::F32 && MT >= 8; }

constexpr int cols_per_thread(Elem w, int MT) {
  // 16-byte shared-memory reads per row for MT <= 4; fewer columns per thread
  // for wider token batches to bound the accumulator count (MT * CPT <= 32).
  return w == Elem::BF16 ? (MT <= 4 ? 8 : (MT == 8 ? 4 : 2)) : (MT <= 4 ? 4 : (MT == 8 ? 2 : 1));
}

int round_mt(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16; }

void* kernel_for(Elem w, Elem c, int MT) {
#define LAROSA_PICK(TW, TC)                                                    \
  switch (MT) {                                                                \
    case 1: return Inst<TW, TC, 1, (sizeof(TW) == 2 ? 8 : 4)>::fn();           \
    case 2: return Inst<TW, TC, 2, (sizeof(TW) == 2 ? 8 : 4)>::fn();           \
    case 4: return Inst<TW, TC, 4, (sizeof(TW) == 2 ? 8 : 4)>::fn();           \
    case 8: return Inst<TW, TC, 8, (sizeof(TW) == 2 ? 4 : 2)>::fn();           \
    case 16: return Inst<TW, TC, 16, (sizeof(TW) == 2 ? 2 : 1)>::fn();         \
    default: return nullptr;                                                   \
  }
  if (w == Elem::BF16 && c == Elem::BF16) { LAROSA_PICK(__nv_bfloat16, __nv_bfloat16) }
  if (uses_mma(w, c, MT)) {
    switch (MT) {
      case 8: return Inst<__nv_bfloat16, float, 8, 8, true>::fn();
      case 16: return Inst<__nv_bfloat16, float, 16, 8, true>::fn();
      default: return nullptr;
    }
  }
  if (w == Elem::BF16 && c == Elem::F32) { LAROSA_PICK(__nv_bfloat16, float) }
  if (w == Elem::F32 && c == Elem::F32) { LAROSA_PICK(float, float) }
#undef LAROSA_PICK
  return nullptr;
}

// Rows (and their coefficients) a CTA keeps in shared memory; sized so that
// MT <= 2 fits two CTAs per SM next to the 96 KB ring.
int max_rows_per_cta(int MT) { return MT <= 2 ? 1024 : (MT <= 8 ? 512 : 256); }

size_t smem_bytes_for(int MT) {
  const size_t pre = kHeaderBytes + (size_t)max_rows_per_cta(MT) * 4 * (1 + MT);
  // + 1 KB: the ring is aligned to 1 KB inside the dynamic window
  return ((pre + 1023) & ~size_t(1023)) + 1024 + (size_t)kStages * kStageBytes;
}

// Co-resident CTAs for each cluster size, per kernel instantiation, cached.
struct OccKey {
  int dev;
  void* fn;
};
struct OccEntry {
  OccKey key;
  int target[4];  // cluster 1, 2, 4, 8
  int sms;
};
std::mutex g_occ_mu;
OccEntry g_occ[64];
int g_occ_n = 0;

cudaError_t occupancy(void* fn, int MT, OccEntry* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_occ_mu);
  for (int i = 0; i < g_occ_n; ++i)
    if (g_occ[i].key.dev == dev && g_occ[i].key.fn == fn) {
      *out = g_occ[i];
      return cudaSuccess;
    }
  OccEntry ent{};
  ent.key = {dev, fn};
  e = cudaDeviceGetAttribute(&ent.sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const size_t smem = smem_bytes_for(MT);
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  for (int ci = 0; ci < 4; ++ci) {
    const int C = 1 << ci;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C * 64, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, fn, &cfg);
    if (e != cudaSuccess) {
      (void)cudaGetLastError();
      clusters = 0;
    }
    ent.target[ci] = clusters * C;
  }
  if (ent.target[0] == 0) {
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, smem);
    if (e != cudaSuccess) return e;
    ent.target[0] = per_sm * ent.sms;
  }
  if (g_occ_n < 64) g_occ[g_occ_n++] = ent;
  *out = ent;
  return cudaSuccess;
}

}  // namespace

cudaError_t plan_gemv(Elem w_elem, Elem coef_elem, int M, int d_out, int n_rows_max,
                      GemvPlan* plan) {
  const int MT = round_mt(M);
  void* fn = kernel_for(w_elem, coef_elem, MT);
  if (fn == nullptr) return cudaErrorInvalidValue;
  OccEntry occ;
  cudaError_t e = occupancy(fn, MT, &occ);
  if (e != cudaSuccess) return e;
  const int cpt = cols_per_thread(w_elem, MT);
  const int elem = w_elem == Elem::BF16 ? 2 : 4;
  const int max_rpc = max_rows_per_cta(MT);
  const int n_rows = std::max(0, n_rows_max);

  // Widest column tile that is not mostly idle threads.
  const bool mma = uses_mma(w_elem, coef_elem, MT);
  int tpr = 256;
  while (tpr > 32 && (tpr / 2) * cpt >= d_out) tpr /= 2;
  // the tensor-core tile: kMmaTile columns, fewer when d_out is smaller
  const int wc = mma ? std::min(kMmaTile, (d_out + 7) / 8 * 8) : tpr * cpt;
  const int n_ct = (d_out + wc - 1) / wc;

  const int min_s = (n_rows + max_rpc - 1) / max_rpc;  // coefficient capacity
  int best_c = 1, best_s = std::max(1, min_s);
  for (int ci = 3; ci >= 0; --ci) {
    const int C = 1 << ci;
    const int target = occ.target[ci];
    if (target < C * n_ct) continue;
    int s = target / n_ct;                         // CTAs per column tile, one wave
    s = std::min(s, std::max(1, n_rows / 8));      // at least 8 rows per CTA
    s = std::max(s, min_s);
    s = std::max(C, (s / C) * C);                  // whole clusters
    while ((long long)s * max_rpc < n_rows) s += C;
    if (C > 1 && n_rows < 4 * s) continue;          // too thin to split C ways
    best_c = C;
    best_s = s;
    break;
  }
  GemvPlan pl;
  pl.col_tile = wc;
  pl.tpr = tpr;
  pl.pitch = mma ? wc * elem + 16 : wc * elem;
  pl.rows_per_stage = kStageBytes / pl.pitch;
  pl.n_col_tiles = n_ct;
  pl.splits = best_s;
  pl.cluster = best_c;
  pl.max_rows_per_cta = max_rpc;
  pl.smem_bytes = smem_bytes_for(MT);
  const int n_clusters = best_s / best_c;
  const int Mw = std::min(M, MT);
  pl.partial_floats = n_clusters > 1 ? (size_t)n_ct * n_clusters * Mw * wc : 0;
  pl.ticket_words = n_clusters > 1 ? (size_t)n_ct * best_c : 0;
  *plan = pl;
  return cudaSuccess;
}

cudaError_t launch_gemv(const GemvArgs& a, const GemvPlan& pl, cudaStream_t stream) {
  const int MT = round_mt(a.M);
  void* fn = kernel_for(a.w_elem, a.coef_elem, MT);
  if (fn == nullptr) return cudaErrorInvalidValue;
  Params p;
  p.W = a.W;
  p.d_out = a.d_out;
  p.row_bound = a.row_bound;
  p.rows = a.rows;
  p.n_rows = a.n_rows;
  p.n_rows_dev = a.n_rows_dev;
  p.coef = a.coef;
  p.coef_ld = a.coef_ld;
  p.coef_by_row = a.coef_by_row;
  p.M = a.M;
  p.y = a.y;
  p.y_ld = a.y_ld;
  p.partials = a.partials;
  p.tickets = a.tickets;
  p.col_tile = pl.col_tile;
  p.tpr = pl.tpr;
  p.rows_per_stage = pl.rows_per_stage;
  p.pitch = pl.pitch;
  p.max_rpc = pl.max_rows_per_cta;
  p.dev_status = a.dev_status;
  p.wait_ns = wait_limit_ns();

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.splits, pl.n_col_tiles, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = pl.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = pl.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  void* args[] = {&p};
  return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace larosa
