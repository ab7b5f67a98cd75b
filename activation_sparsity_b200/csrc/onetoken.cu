// Decode-path kernels (sm_100a): the GEMVs of one token, and of up to 16
// tokens for the row-dot form.  All are bound by HBM bandwidth (about one
// flop per byte), so the design goal is bytes in flight and one read of every
// weight byte:
//
//   * CTAs of 512 threads, two per SM where registers and shared memory
//     allow; every lane keeps eight independent 16-byte loads in flight
//     (ld.global.cs: streamed, evict-first).  Streaming probes on B200 put
//     this at 5.7 (one CTA per SM) to 6.4 TB/s (two), the copy peak, even
//     for row segments of 128-256 bytes; TMA bulk copies into a shared ring
//     reached only about 4.2 TB/s with one CTA per SM and were left out;
//   * a fixed reduction order everywhere, so results are bit-reproducible.
//
// rowdot  y[m][j] = sum_i x[m][i] * A[j][i], A row-major [n_out x n_in].
//         The rotation x_rot = x . Q reads Q through A = Q^T ("La RoSA"
//         summary, 方法详解 / 技术框架: each layer's input activation is
//         multiplied by that layer's orthogonal matrix); the dense baseline
//         reads W in torch.nn.Linear layout.  Each warp owns whole output rows:
//         no cross-CTA reduction at all.
//
// gather  y[c] = sum_{p < K} val[p] * W[idx[p]][c], W row-major
//         [d_in x d_out]: the sparse linear over the kept rows of the
//         counter-rotated weight (abstract: activation sparsity reduces memory
//         transfers).  One thread-block cluster per column tile; the cluster's
//         CTAs take equal consecutive parts of the kept list and add their
//         partial sums through distributed shared memory in rank order, so
//         nothing leaves the cluster but y.  The tile width is chosen so the
//         clusters that fit on the GPU at once cover d_out.
//
// rotsel  the rotation with the Top-K by the last CTA to arrive, and fused
//         the whole one-token path in one cooperative launch (rotation,
//         selection by one CTA, gather of the kept rows by the others); each
//         is described at its kernel below.
#include <cooperative_groups.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace cg = cooperative_groups;

namespace larosa {
namespace {

constexpr int kT = 512;        // threads per CTA
constexpr int kWarps = kT / 32;
constexpr int kU = 8;          // 16-byte loads in flight per lane

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  return __ldcs(static_cast<const uint4*>(p));
}

// 8 bf16 (or 4 fp32, twice) -> fp32
template <typename T>
struct Vec8;
template <>
struct Vec8<__nv_bfloat16> {
  static constexpr int kLoads = 1;
  static __device__ __forceinline__ void cvt(const uint4* u, float (&v)[8]) {
    const uint32_t w[4] = {u[0].x, u[0].y, u[0].z, u[0].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};
template <>
struct Vec8<float> {
  static constexpr int kLoads = 2;
  static __device__ __forceinline__ void cvt(const uint4* u, float (&v)[8]) {
    v[0] = __uint_as_float(u[0].x); v[1] = __uint_as_float(u[0].y);
    v[2] = __uint_as_float(u[0].z); v[3] = __uint_as_float(u[0].w);
    v[4] = __uint_as_float(u[1].x); v[5] = __uint_as_float(u[1].y);
    v[6] = __uint_as_float(u[1].z); v[7] = __uint_as_float(u[1].w);
  }
};

// ================================================================ rowdot

constexpr int kXSmemBytes = 96 * 1024;  // x staged in shared memory when it fits

struct RParams {
  const void* A;   // [n_out x n_in]
  const void* x;   // [M x n_in]
  float* y;        // [M x n_out]
  int n_in;
  int n_out;
  int M;
  int x_in_smem;
};

// One warp, one output row, MT tokens.  Lane l handles the 8-element vectors
// l, l+32, l+64, ... of the row; kU of them are loaded before any is used.
template <typename T, int MT>
__global__ void __launch_bounds__(kT, (MT <= 2 && sizeof(T) == 2 ? 2 : 1)) rowdot_kernel(const RParams p) {
  extern __shared__ __align__(16) unsigned char xs_raw[];
  const T* xs = reinterpret_cast<const T*>(xs_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_wait();
  const T* xg = static_cast<const T*>(p.x);
  if (p.x_in_smem) {
    const int nv = p.M * p.n_in * (int)sizeof(T) / 16;
    for (int i = tid; i < nv; i += kT)
      reinterpret_cast<uint4*>(xs_raw)[i] = __ldg(reinterpret_cast<const uint4*>(xg) + i);
    __syncthreads();
  }
  const T* xsrc = p.x_in_smem ? xs : xg;
  const int G = gridDim.x, cta = blockIdx.x;
  const int r0 = (int)((long long)p.n_out * cta / G);
  const int r1 = (int)((long long)p.n_out * (cta + 1) / G);
  const int nv = p.n_in / 8;  // 8-element vectors per row
  constexpr int L = Vec8<T>::kLoads;
  for (int row = r0 + warp; row < r1; row += kWarps) {
    const unsigned char* arow = static_cast<const unsigned char*>(p.A) + (size_t)row * p.n_in * sizeof(T);
    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.f;
    for (int v0 = lane; v0 < nv; v0 += 32 * kU) {
      uint4 u[kU][L];
#pragma unroll
      for (int k = 0; k < kU; ++k) {
        const int v = v0 + 32 * k;
#pragma unroll
        for (int l = 0; l < L; ++l)
          u[k][l] = v < nv ? ld_stream(arow + (size_t)v * 8 * sizeof(T) + l * 16) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int k = 0; k < kU; ++k) {
        const int v = v0 + 32 * k;
        if (v < nv) {
          float w[8];
          Vec8<T>::cvt(u[k], w);
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            if (m < p.M) {
              uint4 xu[L];
              const unsigned char* xp = reinterpret_cast<const unsigned char*>(
                  xsrc + (size_t)m * p.n_in + (size_t)v * 8);
#pragma unroll
              for (int l = 0; l < L; ++l) xu[l] = *reinterpret_cast<const uint4*>(xp + l * 16);
              float xv[8];
              Vec8<T>::cvt(xu, xv);
#pragma unroll
              for (int e = 0; e < 8; ++e) acc[m] = fmaf(w[e], xv[e], acc[m]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float s = acc[m];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0 && m < p.M) p.y[(size_t)m * p.n_out + row] = s;
    }
  }
  // No early trigger: the next kernel is often a cluster launch that needs
  // whole GPCs, and placing its clusters around this grid's retiring CTAs
  // left some of them for a second wave.  It launches when this grid ends.
}

// ================================================================ rowmma
//
// y[m][j] = sum_k x[m][k] * A[j][k] for 3 to 16 bf16 tokens on the legacy
// tensor-core path (mma.sync m16n8k16, bf16 inputs, fp32 accumulation), for
// the shapes the tcgen05 kernel (rot_umma.cu) does not take: n_in a
// multiple of 32 but not of 64.  From about eight tokens on, the products
// per weight byte exceed what the FMA pipes deliver at HBM speed, and the
// FMA kernel also reads every token's inputs from shared memory once per
// weight vector.  The tokens are the MMA's 16
// rows (zero beyond M), 8 consecutive output rows j its 8 columns, 16 inputs
// k its reduction.  Lane (g, q) = (lane / 4, lane % 4) loads 16 bytes of
// output row j0 + g of A and the same 8 inputs of tokens g and g + 8 per
// block of 32 inputs; the order of the 32 inputs inside a block is permuted
// the same way for x and for A (a sum does not depend on its order), so that
// these loads are the fragments of two MMAs as they stand.  A CTA of
// kMmaWarps warps owns 8 output rows; warp w adds up the input blocks
// [nb*w/kMmaWarps, nb*(w+1)/kMmaWarps) and the warps' partial tiles are added
// in warp order.  Needs n_in % 32 == 0 and n_out % 8 == 0.
constexpr int kMmaWarps = 8;
constexpr int kMmaU = 4;          // 32-input blocks in flight per lane
constexpr int kMmaMinTokens = 3;  // from this many tokens on (bf16) the tensor-core kernel is used

struct MParams {
  const void* A;  // [n_out x n_in] bf16
  const void* x;  // [M x n_in] bf16
  float* y;       // [M x n_out]
  int n_in;
  int n_out;
  int M;
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <bool kTwoRows>  // tokens 8..15 present
__global__ void __launch_bounds__(kMmaWarps * 32) rowmma_kernel(const MParams p) {
  __shared__ float4 s_part[kMmaWarps][32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  const int j0 = blockIdx.x * 8;
  pdl_wait();
  const int nb = p.n_in / 32;
  const int b0 = nb * warp / kMmaWarps, b1 = nb * (warp + 1) / kMmaWarps;
  const unsigned char* arow =
      static_cast<const unsigned char*>(p.A) + ((size_t)(j0 + g) * p.n_in + 8 * q) * 2;
  const unsigned char* xr0 = static_cast<const unsigned char*>(p.x) + ((size_t)g * p.n_in + 8 * q) * 2;
  const unsigned char* xr8 = xr0 + (size_t)8 * p.n_in * 2;
  const bool has0 = g < p.M, has8 = kTwoRows && g + 8 < p.M;
  const uint4 zero = make_uint4(0, 0, 0, 0);
  float d[4] = {0.f, 0.f, 0.f, 0.f};
  for (int b = b0; b < b1; b += kMmaU) {
    uint4 w[kMmaU], u0[kMmaU], u8[kMmaU];
#pragma unroll
    for (int k = 0; k < kMmaU; ++k) {
      const bool in = b + k < b1;
      w[k] = in ? ld_stream(arow + (size_t)(b + k) * 64) : zero;
      u0[k] = in && has0 ? __ldg(reinterpret_cast<const uint4*>(xr0 + (size_t)(b + k) * 64)) : zero;
      u8[k] = kTwoRows && in && has8 ? __ldg(reinterpret_cast<const uint4*>(xr8 + (size_t)(b + k) * 64))
                                     : zero;
    }
#pragma unroll
    for (int k = 0; k < kMmaU; ++k) {
      // step 0 takes the block's inputs 8q + 0..3, step 1 the inputs 8q + 4..7
      mma_bf16_16816(d, u0[k].x, u8[k].x, u0[k].y, u8[k].y, w[k].x, w[k].y);
      mma_bf16_16816(d, u0[k].z, u8[k].z, u0[k].w, u8[k].w, w[k].z, w[k].w);
    }
  }
  s_part[warp][lane] = make_float4(d[0], d[1], d[2], d[3]);
  __syncthreads();
  if (warp == 0) {
    float4 t = s_part[0][lane];
#pragma unroll
    for (int v = 1; v < kMmaWarps; ++v) {
      const float4 o = s_part[v][lane];
      t.x += o.x;
      t.y += o.y;
      t.z += o.z;
      t.w += o.w;
    }
    // D[g][2q], D[g][2q + 1], D[g + 8][2q], D[g + 8][2q + 1]: tokens by rows
    const int j = j0 + 2 * q;
    if (g < p.M) {
      p.y[(size_t)g * p.n_out + j] = t.x;
      p.y[(size_t)g * p.n_out + j + 1] = t.y;
    }
    if (g + 8 < p.M) {
      p.y[(size_t)(g + 8) * p.n_out + j] = t.z;
      p.y[(size_t)(g + 8) * p.n_out + j + 1] = t.w;
    }
  }
}

// ================================================================ gather

constexpr int kGatherSmemCeiling = 227 * 1024;
constexpr int kCandCap = 1024;  // boundary-bin keys ranked directly

struct GParams {
  const void* W;         // [d_in x d_out] row-major
  int d_out;
  int d_in;              // row bound; also the length of x_rot
  int K;                 // kept entries
  const void* coef;      // val[K]
  const int32_t* rows;   // idx[K]
  float* y;
  int col_tile;
  int tpr;
  int list_cap;          // list entries a CTA holds: ceil(K / cluster)
  int* dev_status;
};

// Shared memory of one CTA, laid out from sizes known at launch.
struct GLayout {
  size_t red, rows, vals, part, total;
};

__host__ __device__ inline size_t al16(size_t v) { return (v + 15) & ~size_t(15); }

__host__ __device__ inline GLayout glayout(int list_cap, int col_tile, int cpt) {
  GLayout L{};
  size_t o = 0;
  L.red = o;   o = al16(o + (size_t)(kT / (col_tile / cpt)) * col_tile * 4);
  L.rows = o;  o = al16(o + (size_t)list_cap * 4);
  L.vals = o;  o = al16(o + (size_t)list_cap * 4);
  L.part = o;  o = al16(o + (size_t)col_tile * 4);
  L.total = o;
  return L;
}

// Streams rows lrows[lo, hi) of one column tile (columns [c0, c0 + wc) of a
// row-major [* x d_out] weight), scaled by lvals, into this thread's acc.
// Thread (g, col) reads 16 bytes of rows lo + g, lo + g + ng, ... with NU
// loads in flight.
// Weight rows a thread of the list-mode gather has in flight (6 measured
// faster than 8 and 4 on the LLaMA2-7B groups).
constexpr int kGatherU = 6;

template <typename Tw, int NU = kU>
__device__ __forceinline__ void accumulate_rows(const void* W, int d_out, int c0, int wc, int tpr,
                                                const int32_t* lrows, const float* lvals, int lo,
                                                int hi, float (&acc)[16 / sizeof(Tw)]) {
  constexpr int CPT = 16 / sizeof(Tw);
  const int tid = threadIdx.x;
  const int ng = kT / tpr;
  const int g = tid / tpr;
  const int col = (tid - g * tpr) * CPT;
  if (g >= ng || col >= wc) return;
  const unsigned char* wbase = static_cast<const unsigned char*>(W) + ((size_t)c0 + col) * sizeof(Tw);
  const size_t pitch = (size_t)d_out * sizeof(Tw);
  for (int r0 = lo + g; r0 < hi; r0 += ng * NU) {
    uint4 u[NU];
#pragma unroll
    for (int k = 0; k < NU; ++k) {
      const int r = r0 + k * ng;
      u[k] = r < hi ? ld_stream(wbase + (size_t)lrows[r] * pitch) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int k = 0; k < NU; ++k) {
      const int r = r0 + k * ng;
      const float cf = r < hi ? lvals[r] : 0.f;
      if constexpr (CPT == 8) {
        float w[8];
        Vec8<__nv_bfloat16>::cvt(&u[k], w);
#pragma unroll
        for (int v = 0; v < 8; ++v) acc[v] = fmaf(cf, w[v], acc[v]);
      } else {
        acc[0] = fmaf(cf, __uint_as_float(u[k].x), acc[0]);
        acc[1] = fmaf(cf, __uint_as_float(u[k].y), acc[1]);
        acc[2] = fmaf(cf, __uint_as_float(u[k].z), acc[2]);
        acc[3] = fmaf(cf, __uint_as_float(u[k].w), acc[3]);
      }
    }
  }
}

// Adds the threads' acc of one column tile into y[c0, c0 + wc): the row
// groups meet in `red`, the CTA's partial in `part`, and rank r of the
// cluster adds its slice of the tile over the C partials in rank order.
// Every CTA of the cluster calls it (it holds two cluster barriers).
template <typename Tw, int C>
__device__ __forceinline__ void reduce_tile(cg::cluster_group& cl, int rank, int c0, int wc,
                                            int col_tile, int tpr, const float (&acc)[16 / sizeof(Tw)],
                                            float* red, float* part, float* y) {
  constexpr int CPT = 16 / sizeof(Tw);
  const int tid = threadIdx.x;
  const int ng = kT / tpr;
  const int g = tid / tpr;
  const int col = (tid - g * tpr) * CPT;
  if (g < ng && col < wc) {
#pragma unroll
    for (int v = 0; v < CPT; ++v) red[g * col_tile + col + v] = acc[v];
  }
  __syncthreads();
  for (int e = tid; e < wc; e += kT) {
    float sum = 0.f;
    for (int gg = 0; gg < ng; ++gg) sum += red[gg * col_tile + e];
    part[e] = sum;
  }
  cl.sync();
  const int sl = (wc + C - 1) / C;
  const int e0 = rank * sl, e1 = min(wc, e0 + sl);
  for (int e = e0 + tid; e < e1; e += kT) {
    float v[C];
#pragma unroll
    for (int q = 0; q < C; ++q) v[q] = cl.map_shared_rank(part, q)[e];  // all in flight
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < C; ++q) sum += v[q];
    y[c0 + e] = sum;
  }
  cl.sync();  // no CTA leaves while another may still read its partial
}

// Adds the C CTAs' partial sums of one column tile without any CTA waiting
// for another: each CTA writes its partial of the tile (row groups added in
// shared memory) to gpart[rank * col_tile, ...) and arrives on the tile's
// counter; the CTA that arrives last adds the C partials in rank order and
// writes y[c0, c0 + wc).  The counter must be zero beforehand and is left at
// C.  All kT threads of the CTA call it.
template <typename Tw, int C>
__device__ __forceinline__ void reduce_tile_last(int rank, int c0, int wc, int col_tile, int tpr,
                                                 const float (&acc)[16 / sizeof(Tw)], float* red,
                                                 float* gpart, unsigned* counter, float* y) {
  constexpr int CPT = 16 / sizeof(Tw);
  __shared__ unsigned s_last_of_tile;
  const int tid = threadIdx.x;
  const int ng = kT / tpr;
  const int g = tid / tpr;
  const int col = (tid - g * tpr) * CPT;
  if (g < ng && col < wc) {
#pragma unroll
    for (int v = 0; v < CPT; ++v) red[g * col_tile + col + v] = acc[v];
  }
  __syncthreads();
  for (int e = tid; e < wc; e += kT) {
    float sum = 0.f;
    for (int gg = 0; gg < ng; ++gg) sum += red[gg * col_tile + e];
    __stcg(gpart + (size_t)rank * col_tile + e, sum);
  }
  __syncthreads();  // the CTA's partial is written
  if (tid == 0) {
    // release this CTA's partial; the last to arrive also acquires the others'
    s_last_of_tile = atomic_add_acq_rel_gpu(counter, 1u) == static_cast<unsigned>(C - 1);
  }
  __syncthreads();
  if (!s_last_of_tile) return;
  for (int e = tid; e < wc; e += kT) {
    float v[C];
#pragma unroll
    for (int q = 0; q < C; ++q) v[q] = __ldcg(gpart + (size_t)q * col_tile + e);  // all in flight
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < C; ++q) sum += v[q];
    y[c0 + e] = sum;
  }
}

// Streams rows lrows[0, len) of one column tile and adds the cluster's
// partial sums into y (accumulate_rows, then reduce_tile).
template <typename Tw, int C>
__device__ __forceinline__ void gather_tile(cg::cluster_group& cl, int rank, const void* W, int d_out,
                                            int c0, int wc, int col_tile, int tpr,
                                            const int32_t* lrows, const float* lvals, int len,
                                            float* red, float* part, float* y) {
  float acc[16 / sizeof(Tw)];
#pragma unroll
  for (int v = 0; v < 16 / (int)sizeof(Tw); ++v) acc[v] = 0.f;
  accumulate_rows<Tw, kGatherU>(W, d_out, c0, wc, tpr, lrows, lvals, 0, len, acc);
  reduce_tile<Tw, C>(cl, rank, c0, wc, col_tile, tpr, acc, red, part, y);
}

// One cluster of C CTAs per column tile.  The cluster's CTAs take equal
// consecutive parts of the kept list (in ascending row order), stream those
// rows of the tile, and add their partial sums through distributed shared
// memory in rank order.  An index outside [0, d_in) sets LAROSA_DEV_INDEX
// and is read as row 0 with coefficient 0.
template <typename Tw, int C>
__global__ void __launch_bounds__(kT, 2) gather_kernel(const GParams p) {
  constexpr int CPT = 16 / sizeof(Tw);  // columns per thread per row
  extern __shared__ __align__(16) unsigned char smem_raw[];
  cg::cluster_group cl = cg::this_cluster();
  const int rank = static_cast<int>(cl.block_rank());
  const GLayout L = glayout(p.list_cap, p.col_tile, CPT);
  int32_t* lrows = reinterpret_cast<int32_t*>(smem_raw + L.rows);
  float* lvals = reinterpret_cast<float*>(smem_raw + L.vals);
  float* part = reinterpret_cast<float*>(smem_raw + L.part);
  float* red = reinterpret_cast<float*>(smem_raw + L.red);

  const int tid = threadIdx.x;
  const int tile = blockIdx.y;
  const int c0 = tile * p.col_tile;
  const int wc = min(p.col_tile, p.d_out - c0);
  const int K = p.K;
  // this CTA's part of the kept list: positions [p0, p1)
  const int p0 = (int)((long long)K * rank / C);
  const int p1 = (int)((long long)K * (rank + 1) / C);
  const int len = p1 - p0;

  pdl_wait();
  pdl_launch_dependents();

  {
    bool bad = false;
    for (int j = tid; j < len; j += kT) {
      const int row = p.rows[p0 + j];
      const bool ok = static_cast<unsigned>(row) < static_cast<unsigned>(p.d_in);
      bad |= !ok;
      lrows[j] = ok ? row : 0;
      lvals[j] = ok ? static_cast<const float*>(p.coef)[p0 + j] : 0.f;
    }
    if (__syncthreads_or(bad) && tid == 0) report(p.dev_status, LAROSA_DEV_INDEX);
  }
  __syncthreads();  // the list is complete

  gather_tile<Tw, C>(cl, rank, p.W, p.d_out, c0, wc, p.col_tile, p.tpr, lrows, lvals, len, red,
                     part, p.y);
}

// ================================================================ rotate + select
//
// First kernel of the one-token fused path.  Every CTA computes an equal
// share of the rotated rows x_rot[j] = x . Q^T[j] (as rowdot does) and then
// arrives on a ticket; the last CTA to arrive reads the whole x_rot, selects
// the K largest magnitudes (kept_list: exact, ties to the lower index) and
// writes the kept list, in ascending index order, for the list-mode gather
// that follows.  No CTA waits for another: the ticket only decides which CTA
// does the selection.  The kernel lets its dependent launch at once, so the
// gather's clusters are placed on the SMs that retiring CTAs free and wait
// there (griddepcontrol.wait) until the selection is done.

struct RSParams {
  const void* x;     // [d] activation
  const void* Qt;    // [d x d] rotation, stored transposed (row j = column j of Q)
  float* x_rot;      // [d]
  int32_t* idx;      // [K] kept list
  float* val;        // [K]
  unsigned* ticket;  // zero between calls
  int d;
  int K;
  int* dev_status;
};

// Shared memory: the staged activation, later the last CTA's selection.
struct RSLayout {
  size_t sel, keys, cand, cand_idx, total;
};

__host__ __device__ inline RSLayout rslayout(int d, int elem_bytes) {
  RSLayout L{};
  size_t o = 0;
  L.sel = o;   o = al16(o + sizeof(SelectScratch));
  L.keys = o;  o = al16(o + (size_t)d * 4);
  L.cand = o;  o = al16(o + (size_t)kCandCap * 4);
  L.cand_idx = o; o = al16(o + (size_t)kCandCap * 4);
  const size_t x_bytes = al16((size_t)d * elem_bytes);
  L.total = o > x_bytes ? o : x_bytes;
  return L;
}

template <typename T>
__global__ void __launch_bounds__(kT, 2) rotsel_kernel(const RSParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ unsigned s_last;
  const RSLayout L = rslayout(p.d, sizeof(T));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int d = p.d, K = p.K;

  pdl_wait();
  pdl_launch_dependents();

  // ---- rotation rows [r0, r1) of this CTA
  {
    const int nvx = d * (int)sizeof(T) / 16;
    const uint4* xg = static_cast<const uint4*>(p.x);
    for (int i = tid; i < nvx; i += kT) reinterpret_cast<uint4*>(smem_raw)[i] = __ldg(xg + i);
    __syncthreads();
    const T* xs = reinterpret_cast<const T*>(smem_raw);
    const int r0 = (int)((long long)d * cta / G);
    const int r1 = (int)((long long)d * (cta + 1) / G);
    const int nv = d / 8;  // 8-element vectors per row
    constexpr int LD = Vec8<T>::kLoads;
    constexpr int KU = kU / LD;  // the same bytes in flight for both element sizes
    for (int row = r0 + warp; row < r1; row += kWarps) {
      const unsigned char* arow = static_cast<const unsigned char*>(p.Qt) + (size_t)row * d * sizeof(T);
      float acc = 0.f;
      for (int v0 = lane; v0 < nv; v0 += 32 * KU) {
        uint4 u[KU][LD];
#pragma unroll
        for (int k = 0; k < KU; ++k) {
          const int v = v0 + 32 * k;
#pragma unroll
          for (int l = 0; l < LD; ++l)
            u[k][l] = v < nv ? ld_stream(arow + (size_t)v * 8 * sizeof(T) + l * 16) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int k = 0; k < KU; ++k) {
          const int v = v0 + 32 * k;
          if (v < nv) {
            float w[8], xv[8];
            Vec8<T>::cvt(u[k], w);
            uint4 xu[LD];
#pragma unroll
            for (int l = 0; l < LD; ++l)
              xu[l] = *reinterpret_cast<const uint4*>(reinterpret_cast<const unsigned char*>(xs + (size_t)v * 8) + l * 16);
            Vec8<T>::cvt(xu, xv);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc = fmaf(w[e], xv[e], acc);
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) __stcg(p.x_rot + row, acc);
    }
  }
  SelectScratch* sel = reinterpret_cast<SelectScratch*>(smem_raw + L.sel);
  __syncthreads();  // the staged x is dead; this CTA's rows are written
  for (int b = tid; b < kFineBins; b += kT) sel->hist[b] = 0u;  // for the selection, if last
  if (tid == 0) {
    // release this CTA's rows; the last to arrive also acquires every CTA's
    s_last = atomic_add_acq_rel_gpu(p.ticket, 1u) == static_cast<unsigned>(G - 1);
  }
  __syncthreads();
  if (!s_last) return;

  // ---- the last CTA to arrive selects
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + L.keys);
  uint32_t* cand = reinterpret_cast<uint32_t*>(smem_raw + L.cand);
  uint32_t* cand_idx = reinterpret_cast<uint32_t*>(smem_raw + L.cand_idx);
  const uint4* src = reinterpret_cast<const uint4*>(p.x_rot);  // d is a multiple of 8
  uint4* dst = reinterpret_cast<uint4*>(keys);
  const int nv = d / 4;
  bool nonfinite = false;
  for (int v0 = tid; v0 < nv; v0 += kT * kU) {
    uint4 u[kU];
#pragma unroll
    for (int k = 0; k < kU; ++k) {
      const int v = v0 + k * kT;
      u[k] = v < nv ? __ldcg(src + v) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int k = 0; k < kU; ++k) {
      const int v = v0 + k * kT;
      if (v < nv) {
        dst[v] = u[k];
        const uint32_t w[4] = {u[k].x & kKeyMask, u[k].y & kKeyMask, u[k].z & kKeyMask,
                               u[k].w & kKeyMask};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          nonfinite |= w[e] >= 0x7f800000u;
          atomicAdd(&sel->hist[w[e] >> kFineShift], 1u);
        }
      }
    }
  }
  if (__syncthreads_or(nonfinite) && tid == 0) report(p.dev_status, LAROSA_DEV_NONFINITE);
  if (K > 0 && K < d) {
    kept_list<kT>(keys, d, K, sel, cand, cand_idx, kCandCap, 0, K, p.idx, p.val);
  } else if (K >= d) {
    for (int i = tid; i < d; i += kT) {
      p.idx[i] = i;
      p.val[i] = __uint_as_float(keys[i]);
    }
  }
  if (tid == 0) *p.ticket = 0u;  // zero again for the next call
}

// ================================================================ fused, one token
//
// rotate -> select -> gather in one cooperative launch of n_tiles * C + 1 CTAs,
// all resident at once: C CTAs per column tile of the output, and a selector.
//
//   1. every CTA computes an equal share of x_rot[j] = x . Q^T[j] (as rowdot
//      does), stores it, adds the keys (bits 30..19 of |x_rot|) to the call's
//      histogram and arrives on a ticket;
//   2. the selector (the last CTA) waits for every arrival, finds from the
//      histogram the bin B that holds the K-th largest magnitude, lists B's
//      keys in one pass over x_rot and ranks them in shared memory: the one
//      ranked K - (keys above B) - 1 is the K-th entry (T, I), which it
//      publishes.  Its L2 reads are made right after the arrivals, before the
//      gather CTAs stream weight rows, while an L2 round trip is still short.
//      It then writes the kept list for callers and clears the next call's
//      counters;
//   3. the gather CTAs (CTA tile*C + r takes column tile `tile` and owns the
//      indices [d*r/C, d*(r+1)/C)) read the histogram and their range of
//      x_rot, find B themselves and stream the rows that are certainly kept
//      (bin above B), then the few kept rows of bin B once (T, I) is
//      published; the last CTA of each tile to finish adds the tile's C
//      partial sums.
//
// Kept = the K largest |x_rot|, ties to the lower index: key > T, or
// key == T and index <= I.  Every wait is bounded (FParams::wait_ns) and reports
// LAROSA_DEV_TIMEOUT; the cooperative launch guarantees that every CTA is
// resident, so no CTA waits on one that cannot run.
//
// Synchronisation words (in the caller's workspace; all zero initially):
// sync[3] is the number of the last call whose K-th entry was published.
// Every CTA reads it before it arrives, so all CTAs of a call agree on its
// number n = sync[3] + 1 (calls that share the words must not overlap).
// Call n counts arrivals in sync[n & 1], its histogram in slot n & 1 of
// 2 x kFusedHistBins counters and its tiles' completions in slot n & 1 of
// 2 x kFusedMaxTiles counters; its selector clears the other slots, which
// call n - 1 has finished with, so no counter is reset while a CTA may still
// read it.  sync[3] becomes n when the K-th entry is published in sync[6..7].

struct FParams {
  const void* x;      // [d] activation
  const void* Qt;     // [d x d] rotation, stored transposed (unused when !rotate)
  const void* W;      // [d x d_out] counter-rotated weight
  float* x_rot;       // [d]
  int32_t* idx;       // [K] kept list (for callers)
  float* val;         // [K]
  float* y;           // [d_out]
  float* partials;    // [n_tiles x C x col_tile] per-CTA partial sums of each column tile
  unsigned* sync;     // [0, 1] arrivals, [3] the last call's number, [4, 5] the K-th entry
                      // with its call's tag (one 64-bit word, see pack_kth); then
                      // 2 x kFusedMaxTiles tile counters, 2 x kFusedHistBins histogram bins
  int d;
  int d_out;
  int K;
  int col_tile;
  int tpr;
  int range_cap;      // ceil(d / C): indices a gather CTA owns
  int n_tiles;        // column tiles (C gather CTAs each)
  int* dev_status;
  int rotate;         // 0: the identity rotation, x_rot = x
  int thresh;         // 1: keep |x_rot| >= t (key >= t_key) instead of the Top-K
  uint32_t t_key;
  int32_t* nnz;       // threshold mode: the kept count (for callers)
  unsigned long long wait_ns;  // limit of every wait
};

struct FLayout {
  size_t bins, cand, cand_idx, red, rows, vals, total;
};

constexpr int kFusedCandCap = 512;  // boundary-bin keys the selector ranks directly

// Region A (offset 0) holds, one after the other in time: the staged x; then
// in the selector the bin numbers of all d entries and the boundary
// candidates, and in a gather CTA its range of keys, then the row-group
// partials.
__host__ __device__ inline FLayout flayout(int d, int elem_bytes, int range_cap, int col_tile,
                                           int cpt) {
  FLayout L{};
  size_t o = 0;
  L.bins = o;     o = al16(o + (size_t)d * 2);
  L.cand = o;     o = al16(o + (size_t)kFusedCandCap * 4);
  L.cand_idx = o; o = al16(o + (size_t)kFusedCandCap * 4);
  const size_t x_bytes = al16((size_t)d * elem_bytes);
  const size_t range_bytes = al16((size_t)range_cap * 4);
  const size_t red_bytes = al16((size_t)(kT / (col_tile / cpt)) * col_tile * 4);
  L.red = 0;
  o = o > x_bytes ? o : x_bytes;
  o = o > range_bytes ? o : range_bytes;
  o = o > red_bytes ? o : red_bytes;
  L.rows = o;  o = al16(o + (size_t)range_cap * 4);
  L.vals = o;  o = al16(o + (size_t)range_cap * 4);
  L.total = o;
  return L;
}

constexpr int kRowKeys = 256;  // rotated rows per CTA whose keys are aggregated in shared memory
constexpr size_t kQPrefetchBytes = 32 << 10;  // rows of Q per CTA requested into L2 before the wait
// Weight rows a gather thread of the fused kernel has in flight.  Fewer than
// the kU of the standalone kernels: the fused kernel's critical path after
// the arrivals is a chain of L2 round trips (the K-th entry, the tile
// reduction) that wait behind every load queued on the SM, and four rows
// per thread (128 KB per SM) already keep HBM streaming.
constexpr int kFusedU = 4;

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_gpu(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned long long ld_acquire_gpu_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_gpu_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// The K-th entry as one word: T in bits 0..31, I (16 bits; -1 as 0xffff) in
// bits 32..47 and the call's tag (its number mod 2^16) in bits 48..63, so
// that the one acquire load that sees the publication also returns the entry.
__device__ __forceinline__ unsigned long long pack_kth(uint32_t T, int32_t I, unsigned gen) {
  return (unsigned long long)T | ((unsigned long long)(static_cast<uint32_t>(I) & 0xffffu) << 32) |
         ((unsigned long long)(gen & 0xffffu) << 48);
}

// Thread 0 waits until the word at kth carries the tag of call gen and
// returns it in *w; false after limit_ns.
__device__ __forceinline__ bool wait_kth(const unsigned long long* kth, unsigned gen, unsigned long long* w,
                                         unsigned long long limit_ns) {
  const unsigned long long tag = gen & 0xffffu;
  unsigned long long v = ld_acquire_gpu_u64(kth);
  if ((v >> 48) == tag) {
    *w = v;
    return true;
  }
  const unsigned long long t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(64);
    v = ld_acquire_gpu_u64(kth);
    if ((v >> 48) == tag) {
      *w = v;
      return true;
    }
    if ((it & 31u) == 0 && global_timer_ns() - t0 > limit_ns) return false;
  }
}

// Thread 0 waits until *word == value; false after limit_ns.  An arrival
// counter is waited on with its exact final count: it only grows during a
// call and is cleared only after the call has completed, so every waiter
// sees that value, and a counter left over from a call that gave up (it
// starts above zero) can never reach it, so such a call times out instead
// of reading a half-built selection.
__device__ __forceinline__ bool wait_word(const unsigned* word, unsigned value,
                                          unsigned long long limit_ns) {
  if (ld_acquire_gpu(word) == value) return true;
  const unsigned long long t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(64);
    if (ld_acquire_gpu(word) == value) return true;
    if ((it & 31u) == 0 && global_timer_ns() - t0 > limit_ns) return false;
  }
}

// Appends to rows/vals (from position `base`) the indices i_lo + i of the
// keys[0, n) that satisfy pred(key, i_lo + i), in ascending order, and
// returns how many (the same value in every thread).  Warp segments and
// ballots; all kT threads call it; it holds one barrier.
template <typename Pred>
__device__ __forceinline__ int compact_range(const uint32_t* keys, int n, int i_lo, Pred pred,
                                             int32_t* rows, float* vals, int base,
                                             uint32_t* warp_sums) {
  const int lane = threadIdx.x & 31;
  const uint32_t below = (1u << lane) - 1u;
  int s0, s1;
  warp_segment<kT>(n, &s0, &s1);
  uint32_t cnt = 0;
  for (int i = s0 + lane; i < s1; i += 32) cnt += pred(keys[i] & kKeyMask, i_lo + i);
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  uint32_t total = 0;
  uint32_t pos = warp_base<kT>(cnt, warp_sums, &total);
  if (cnt != 0u) {
    pos += static_cast<uint32_t>(base);
    for (int i0 = s0; i0 < s1; i0 += 32) {
      const int i = i0 + lane;
      const uint32_t u = i < s1 ? keys[i] : 0u;
      const bool hit = i < s1 && pred(u & kKeyMask, i_lo + i);
      const uint32_t m = __ballot_sync(0xffffffffu, hit);
      if (hit) {
        rows[pos + __popc(m & below)] = i_lo + i;
        vals[pos + __popc(m & below)] = __uint_as_float(u);
      }
      pos += __popc(m);
    }
  }
  return static_cast<int>(total);
}

// ---- the selector's steps, on 16-bit bin numbers in shared memory and the
// full keys in global memory (x_rot, read through L2)

// Number of keys >= t among xkeys[0, d); the same value in every thread.
__device__ __forceinline__ uint32_t count_keys_ge(const uint32_t* xkeys, int d, uint32_t t,
                                                  uint32_t* warp_sums) {
  uint32_t c = 0;
  for (int i0 = threadIdx.x; i0 < d; i0 += kT * kU) {
    uint32_t u[kU];
#pragma unroll
    for (int k = 0; k < kU; ++k) u[k] = i0 + k * kT < d ? __ldcg(xkeys + i0 + k * kT) & kKeyMask : 0u;
#pragma unroll
    for (int k = 0; k < kU; ++k) c += (i0 + k * kT < d) && u[k] >= t;
  }
  c = __reduce_add_sync(0xffffffffu, c);
  uint32_t total = 0;
  (void)warp_base<kT>(c, warp_sums, &total);
  __syncthreads();  // warp_sums may be reused
  return total;
}

// The K-th entry when the boundary bin holds more than kFusedCandCap keys
// (heavy ties): T = the largest t with count(key >= t) >= K, by bisection
// over the 31-bit keys, then I = the index of the (K - count(key > T))-th
// key equal to T in ascending index order.  Requires 1 <= K < d.  All kT
// threads call it.
__device__ __noinline__ KthEntry kth_by_bisection(const uint32_t* xkeys, int d, int K,
                                                  uint32_t* warp_sums, uint32_t* pick) {
  const int lane = threadIdx.x & 31;
  const uint32_t below = (1u << lane) - 1u;
  int s0, s1;
  warp_segment<kT>(d, &s0, &s1);
  uint32_t lo = 0u, hi = kKeyMask;
  while (lo < hi) {
    const uint32_t mid = lo + (hi - lo + 1u) / 2u;
    if (count_keys_ge(xkeys, d, mid, warp_sums) >= static_cast<uint32_t>(K))
      lo = mid;
    else
      hi = mid - 1u;
  }
  const uint32_t T = lo;
  const uint32_t n_gt = T < kKeyMask ? count_keys_ge(xkeys, d, T + 1u, warp_sums) : 0u;
  const uint32_t krem = static_cast<uint32_t>(K) - n_gt;
  uint32_t n_eq = 0;
  for (int i = s0 + lane; i < s1; i += 32) n_eq += (__ldcg(xkeys + i) & kKeyMask) == T;
  n_eq = __reduce_add_sync(0xffffffffu, n_eq);
  uint32_t base = warp_base<kT>(n_eq, warp_sums, nullptr);
  if (base < krem && krem <= base + n_eq) {  // this warp holds it
    for (int i0 = s0; i0 < s1; i0 += 32) {
      const int i = i0 + lane;
      const bool eq = i < s1 && (__ldcg(xkeys + i) & kKeyMask) == T;
      const uint32_t m = __ballot_sync(0xffffffffu, eq);
      if (eq && base + __popc(m & below) + 1u == krem) pick[1] = static_cast<uint32_t>(i);
      base += __popc(m);
      if (base >= krem) break;
    }
  }
  __syncthreads();
  return KthEntry{T, static_cast<int32_t>(pick[1])};
}

constexpr int kPre = 6;  // 16-byte vectors of x_rot per thread read with the histogram
constexpr int kSubBits = 8;  // key bits below the bin that refine_boundary resolves
static_assert(kRowKeys >= (1 << kSubBits), "the sub-bin histogram reuses s_rowkey");

// When the boundary bin B holds more keys than the candidate slots (large d,
// where a bin of bits 30..19 spans hundreds of entries): a histogram of the
// next kSubBits key bits of B's keys, in shared memory (sub, 2^kSubBits
// words), gives the sub-bin holding the krem-th largest of them (*B2), the
// number of B's keys above it (*above2) and its own count (*n2).  Also writes
// the bin numbers of all keys to bins and sets *nonfinite in a thread that
// met a NaN or Inf, as select_kth does.  Requires 1 <= krem <= (keys in B).
// All kT threads call it; it begins after and ends with a barrier.
__device__ __forceinline__ void refine_boundary(const uint32_t* xkeys, int d, uint32_t B, uint32_t krem,
                                             uint16_t* bins, uint32_t* sub, uint32_t* pick,
                                             uint32_t* B2, uint32_t* above2, uint32_t* n2,
                                             bool* nonfinite) {
  constexpr int kSub = 1 << kSubBits;
  constexpr int kLoads = 4;
  const int tid = threadIdx.x, lane = tid & 31;
  const int nv = d / 4;  // d is a multiple of 8
  for (int j = tid; j < kSub; j += kT) sub[j] = 0u;
  __syncthreads();
  bool bad = false;
  for (int v0 = tid; v0 < nv; v0 += kLoads * kT) {
    uint4 u[kLoads];
#pragma unroll
    for (int k = 0; k < kLoads; ++k) {
      const int v = v0 + k * kT;
      u[k] = v < nv ? __ldcg(reinterpret_cast<const uint4*>(xkeys) + v) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int k = 0; k < kLoads; ++k) {
      const int v = v0 + k * kT;
      if (v < nv) {
        const uint32_t w[4] = {u[k].x & kKeyMask, u[k].y & kKeyMask, u[k].z & kKeyMask, u[k].w & kKeyMask};
        uint2 packed;
        packed.x = (w[0] >> kFineShift) | ((w[1] >> kFineShift) << 16);
        packed.y = (w[2] >> kFineShift) | ((w[3] >> kFineShift) << 16);
        reinterpret_cast<uint2*>(bins)[v] = packed;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          bad |= w[e] >= 0x7f800000u;
          if ((w[e] >> kFineShift) == B)
            atomicAdd(sub + ((w[e] >> (kFineShift - kSubBits)) & (kSub - 1u)), 1u);
        }
      }
    }
  }
  *nonfinite = bad;
  __syncthreads();
  if (tid < 32) {
    // lane l holds the sub-bins hi, hi - 1, ..., hi - per + 1 (hi = kSub - 1 - per * l):
    // counts from the top, the krem-th largest key lies in the first sub-bin
    // where the running count reaches krem
    constexpr int per = kSub / 32;
    const int hi = kSub - 1 - per * lane;
    uint32_t mine = 0;
#pragma unroll
    for (int j = 0; j < per; ++j) mine += sub[hi - j];
    uint32_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    uint32_t run = incl - mine;
    if (run < krem && krem <= incl) {  // exactly one lane
      for (int j = 0; j < per; ++j) {
        const uint32_t c = sub[hi - j];
        if (run + c >= krem) {
          pick[0] = static_cast<uint32_t>(hi - j);
          pick[1] = run;
          pick[2] = c;
          break;
        }
        run += c;
      }
    }
  }
  __syncthreads();
  *B2 = pick[0];
  *above2 = pick[1];
  *n2 = pick[2];
  __syncthreads();  // pick may be written again
}

// The selector's pass over x_rot once the boundary bin B is known: writes
// the bin number (bits 30..19) of every key to bins (shared memory), lists
// the keys whose top bits (key >> shift) equal target -- B's keys, or after
// refine_boundary those of one sub-bin of B -- with their indices in
// cand_key / cand_idx (in no particular order: each warp reserves its slots
// with one atomic), ranks each against the others (larger key first, then
// lower index) and returns the one ranked krem - 1, i.e. the K-th entry
// (T, I).  Requires 1 <= krem <= (keys listed) <= kFusedCandCap.  With
// kHavePre, pre[k] holds the 16-byte vector tid + k * kT of xkeys, read
// ahead by the caller; without, pre is not read.  The kFusedCandCap slots
// of cand_key / cand_idx (16-byte aligned) hold key 0 and index 0xffffffff
// on entry; cnt: a word of shared memory, zero on entry.  Sets *nonfinite
// in a thread that met a NaN or Inf.  All kT threads call it; it begins
// after and ends with a barrier.
template <bool kHavePre>
__device__ __forceinline__ KthEntry select_kth(const uint32_t* xkeys, int d, int shift,
                                               uint32_t target, uint32_t krem, const uint4 (&pre)[kPre],
                                               uint16_t* bins, uint32_t* cand_key,
                                               uint32_t* cand_idx, uint32_t* cnt, uint32_t* pick,
                                               bool* nonfinite) {
  const int tid = threadIdx.x, lane = tid & 31;
  const int nv = d / 4;  // d is a multiple of 8
  bool bad = false;
  auto list_batch = [&](const uint4 (&u)[kPre], int vb) {
    uint32_t hits = 0;
#pragma unroll
    for (int k = 0; k < kPre; ++k) {
      const int v = vb + tid + k * kT;
      const uint32_t w[4] = {u[k].x & kKeyMask, u[k].y & kKeyMask, u[k].z & kKeyMask, u[k].w & kKeyMask};
      if (v < nv) {
        uint2 packed;
        packed.x = (w[0] >> kFineShift) | ((w[1] >> kFineShift) << 16);
        packed.y = (w[2] >> kFineShift) | ((w[3] >> kFineShift) << 16);
        reinterpret_cast<uint2*>(bins)[v] = packed;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        hits += v < nv && (w[e] >> shift) == target;
        bad |= v < nv && w[e] >= 0x7f800000u;
      }
    }
    uint32_t inc = hits;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += n;
    }
    const uint32_t wtot = __shfl_sync(0xffffffffu, inc, 31);
    if (wtot == 0u) return;  // warp-uniform
    uint32_t base = 0;
    if (lane == 31) base = atomicAdd(cnt, wtot);
    uint32_t slot = __shfl_sync(0xffffffffu, base, 31) + inc - hits;
    if (hits == 0u) return;
#pragma unroll
    for (int k = 0; k < kPre; ++k) {
      const int v = vb + tid + k * kT;
      const uint32_t w[4] = {u[k].x & kKeyMask, u[k].y & kKeyMask, u[k].z & kKeyMask, u[k].w & kKeyMask};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (v < nv && (w[e] >> shift) == target) {
          if (slot < static_cast<uint32_t>(kFusedCandCap)) {
            cand_key[slot] = w[e];
            cand_idx[slot] = static_cast<uint32_t>(4 * v + e);
          }
          ++slot;
        }
      }
    }
  };
  if constexpr (kHavePre) list_batch(pre, 0);
  for (int v0 = kHavePre ? kPre * kT : 0; v0 < nv; v0 += kPre * kT) {
    uint4 u[kPre];
#pragma unroll
    for (int k = 0; k < kPre; ++k) {
      const int v = v0 + tid + k * kT;
      u[k] = v < nv ? __ldcg(reinterpret_cast<const uint4*>(xkeys) + v) : make_uint4(0, 0, 0, 0);
    }
    list_batch(u, v0);
  }
  *nonfinite = bad;
  __syncthreads();
  // g threads per candidate (a power of two, within one warp): thread
  // c * g + s compares candidate c with the 16-byte vectors s, s + g, ... of
  // the list; the slots after the last candidate hold key 0 and index
  // 0xffffffff, which never rank above a candidate
  const int nc = static_cast<int>(min(*cnt, static_cast<uint32_t>(kFusedCandCap)));  // nB
  const int nq = (nc + 3) / 4;
  int g = 32;
  while (g > 1 && nc * g > kT) g >>= 1;
  const int c = tid / g, s = tid - c * g;
  uint32_t kc = 0, ic = 0, r = 0;
  if (c < nc) {
    kc = cand_key[c];
    ic = cand_idx[c];
    const uint4* kq = reinterpret_cast<const uint4*>(cand_key);
    const uint4* iq = reinterpret_cast<const uint4*>(cand_idx);
#pragma unroll 2
    for (int q = s; q < nq; q += g) {
      const uint4 a = kq[q], b = iq[q];
      r += (a.x > kc) | ((a.x == kc) & (b.x < ic));
      r += (a.y > kc) | ((a.y == kc) & (b.y < ic));
      r += (a.z > kc) | ((a.z == kc) & (b.z < ic));
      r += (a.w > kc) | ((a.w == kc) & (b.w < ic));
    }
  }
  for (int o = 1; o < g; o <<= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
  if (c < nc && s == 0 && r == krem - 1u) {  // ranks are unique
    pick[0] = kc;
    pick[1] = ic;
  }
  __syncthreads();
  return KthEntry{pick[0], static_cast<int32_t>(pick[1])};
}

// The K-th entry where B holds more than kFusedCandCap keys: refine_boundary
// narrows the candidates to one sub-bin of B; only when that too overflows
// (heavy ties) does the bisection over all keys decide.  Out of line, so the
// common path keeps its registers and code.  Arguments as for select_kth and
// refine_boundary; sub: 2^kSubBits words of shared memory.
__device__ __noinline__ KthEntry select_crowded(const uint32_t* xkeys, int d, int K, uint32_t B,
                                                uint32_t krem, uint16_t* bins, uint32_t* sub,
                                                uint32_t* cand_key, uint32_t* cand_idx, uint32_t* cnt,
                                                uint32_t* pick, uint32_t* warp_sums, bool* nonfinite) {
  uint32_t B2 = 0, above2 = 0, n2 = 0;
  refine_boundary(xkeys, d, B, krem, bins, sub, pick, &B2, &above2, &n2, nonfinite);
  if (n2 <= static_cast<uint32_t>(kFusedCandCap)) {
    const uint4 unused[kPre] = {};
    bool bad = false;
    const KthEntry e = select_kth<false>(xkeys, d, kFineShift - kSubBits, (B << kSubBits) | B2, krem - above2,
                                         unused, bins, cand_key, cand_idx, cnt, pick, &bad);
    *nonfinite |= bad;
    return e;
  }
  return kth_by_bisection(xkeys, d, K, warp_sums, pick);
}

// The kept list (idx, val: the K entries up to the K-th entry e, ascending
// index) of the d keys: bin above B, or bin B and up to e.  When B's keys
// were listed (cand_key, in ascending index order, i.e. in the order the
// warp segments meet them) they decide; otherwise the full key is read from
// global memory.  Warp segments and ballots, so stores are contiguous runs;
// values are read from global memory 8 x 32 at a time.  All kT threads
// call it.
__device__ __forceinline__ void fused_export(const uint32_t* xkeys, const uint16_t* bins, int d,
                                             uint32_t B, KthEntry e, bool listed,
                                             const uint32_t* cand_key, int32_t* idx, float* val,
                                             uint32_t* warp_sums) {
  const int lane = threadIdx.x & 31;
  const uint32_t below = (1u << lane) - 1u;
  int s0, s1;
  warp_segment<kT>(d, &s0, &s1);
  // bin-B entries of earlier warps (their slots in cand_key)
  uint32_t n_b = 0;
  for (int i = s0 + lane; i < s1; i += 32) n_b += bins[i] == B;
  n_b = __reduce_add_sync(0xffffffffu, n_b);
  const uint32_t slot = warp_base<kT>(n_b, warp_sums, nullptr);
  __syncthreads();  // warp_sums is used again below
  // kept count of this warp's segment
  uint32_t n_kept = 0;
  {
    uint32_t sl = slot;
    for (int i0 = s0; i0 < s1; i0 += 32) {
      const int i = i0 + lane;
      const uint32_t b = i < s1 ? bins[i] : 0u;
      const bool inb = i < s1 && b == B;
      const uint32_t mb = __ballot_sync(0xffffffffu, inb);
      bool k = i < s1 && b > B;
      if (inb) {
        const uint32_t key = listed ? cand_key[sl + __popc(mb & below)] : (__ldcg(xkeys + i) & kKeyMask);
        k = is_kept(key, i, e);
      }
      n_kept += __popc(__ballot_sync(0xffffffffu, k));
      sl += __popc(mb);
    }
  }
  uint32_t pos = warp_base<kT>(n_kept, warp_sums, nullptr);
  if (n_kept == 0u) return;
  for (int i0 = s0; i0 < s1; i0 += 32 * kU) {
    uint32_t u[kU];
#pragma unroll
    for (int k = 0; k < kU; ++k) {
      const int i = i0 + 32 * k + lane;
      u[k] = i < s1 ? __ldcg(xkeys + i) : 0u;
    }
#pragma unroll
    for (int k = 0; k < kU; ++k) {
      const int i = i0 + 32 * k + lane;
      const uint32_t b = i < s1 ? bins[i] : 0u;
      bool kept = i < s1 && b > B;
      if (i < s1 && b == B) kept = is_kept(u[k] & kKeyMask, i, e);
      const uint32_t m = __ballot_sync(0xffffffffu, kept);
      if (kept) {
        idx[pos + __popc(m & below)] = i;
        val[pos + __popc(m & below)] = __uint_as_float(u[k]);
      }
      pos += __popc(m);
    }
  }
}

// Threshold mode's kept list for callers: the indices whose key (sign-
// cleared bits of x_rot, read through L2) is >= t_key, in ascending order,
// with their values; returns their number (the same in every thread) and
// sets *nonfinite in a thread that met a NaN or Inf.  Warp segments, keys
// read kU x 32 at a time, ballots; all kT threads call it.
__device__ __noinline__ uint32_t export_threshold(const uint32_t* xkeys, int d, uint32_t t_key,
                                                  int32_t* idx, float* val, uint32_t* warp_sums,
                                                  bool* nonfinite) {
  const int lane = threadIdx.x & 31;
  const uint32_t below = (1u << lane) - 1u;
  int s0, s1;
  warp_segment<kT>(d, &s0, &s1);
  uint32_t n = 0;
  bool bad = false;
  for (int i0 = s0; i0 < s1; i0 += 32 * kU) {
    uint32_t u[kU];
#pragma unroll
    for (int k = 0; k < kU; ++k) {
      const int i = i0 + 32 * k + lane;
      u[k] = i < s1 ? __ldcg(xkeys + i) & kKeyMask : 0u;
    }
#pragma unroll
    for (int k = 0; k < kU; ++k) {
      const int i = i0 + 32 * k + lane;
      n += i < s1 && u[k] >= t_key;
      bad |= u[k] >= 0x7f800000u;
    }
  }
  *nonfinite = bad;
  n = __reduce_add_sync(0xffffffffu, n);
  uint32_t total = 0;
  uint32_t pos = warp_base<kT>(n, warp_sums, &total);
  if (n != 0u) {  // warp-uniform
    for (int i0 = s0; i0 < s1; i0 += 32 * kU) {
      uint32_t u[kU];
#pragma unroll
      for (int k = 0; k < kU; ++k) {
        const int i = i0 + 32 * k + lane;
        u[k] = i < s1 ? __ldcg(xkeys + i) : 0u;
      }
#pragma unroll
      for (int k = 0; k < kU; ++k) {
        const int i = i0 + 32 * k + lane;
        const bool kept = i < s1 && (u[k] & kKeyMask) >= t_key;
        const uint32_t m = __ballot_sync(0xffffffffu, kept);
        if (kept) {
          idx[pos + __popc(m & below)] = i;
          val[pos + __popc(m & below)] = __uint_as_float(u[k]);
        }
        pos += __popc(m);
      }
    }
  }
  return total;
}

template <typename T, int C>
__global__ void __launch_bounds__(kT, 2) fused_kernel(const FParams p) {
  constexpr int CPT = 16 / sizeof(T);
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ uint32_t s_gen;
  __shared__ uint32_t s_word[8];
  __shared__ uint32_t s_warp_sums[32];
  __shared__ uint32_t s_pick[4];
  __shared__ uint32_t s_rowkey[kRowKeys];  // keys of this CTA's rotated rows
  const FLayout L = flayout(p.d, sizeof(T), p.range_cap, p.col_tile, CPT);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = static_cast<int>(gridDim.x);  // n_tiles * C gather CTAs + the selector
  const int cta = blockIdx.x;
  const int tile = cta / C, rank = cta - tile * C;
  const int d = p.d, K = p.K;

  // ---- 1. rotation rows [r0, r1) of this CTA
  const int r0 = (int)((long long)d * cta / G);
  const int r1 = (int)((long long)d * (cta + 1) / G);
  // Launched as a programmatic dependent of the previous kernel on the
  // stream: until griddepcontrol.wait returns, that kernel may still be
  // running, and nothing it writes may be read.  This CTA's first rows of Q
  // are asked into L2 now, while the previous kernel's last CTAs leave HBM
  // idle; a prefetch into L2 (the point of coherence) only moves a read
  // earlier and never changes what a later load returns.
  if (warp == 0 && p.rotate) {
    const size_t row_bytes = (size_t)d * sizeof(T);
    const int n_pf = min(r1 - r0, static_cast<int>(kQPrefetchBytes / row_bytes) + 1);
    for (int j = lane; j < n_pf; j += 32)
      bulk_prefetch_l2(static_cast<const unsigned char*>(p.Qt) + (size_t)(r0 + j) * row_bytes,
                       static_cast<uint32_t>(row_bytes));
  }
  pdl_wait();
  pdl_launch_dependents();  // the next call may start its own prefetch as CTAs of this one finish
  if (tid == 0) s_gen = ld_acquire_gpu(p.sync + 3) + 1u;  // this call's number, read before arriving
  if (p.rotate) {
    const int nvx = d * (int)sizeof(T) / 16;
    const uint4* xg = static_cast<const uint4*>(p.x);
    for (int i = tid; i < nvx; i += kT) reinterpret_cast<uint4*>(smem_raw)[i] = __ldg(xg + i);
    __syncthreads();
    const T* xs = reinterpret_cast<const T*>(smem_raw);
    const int nv = d / 8;  // 8-element vectors per row
    constexpr int LD = Vec8<T>::kLoads;
    constexpr int KU = kU / LD;  // the same bytes in flight for both element sizes
    for (int row = r0 + warp; row < r1; row += kWarps) {
      const unsigned char* arow = static_cast<const unsigned char*>(p.Qt) + (size_t)row * d * sizeof(T);
      float acc = 0.f;
      for (int v0 = lane; v0 < nv; v0 += 32 * KU) {
        uint4 u[KU][LD];
#pragma unroll
        for (int k = 0; k < KU; ++k) {
          const int v = v0 + 32 * k;
#pragma unroll
          for (int l = 0; l < LD; ++l)
            u[k][l] = v < nv ? ld_stream(arow + (size_t)v * 8 * sizeof(T) + l * 16) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int k = 0; k < KU; ++k) {
          const int v = v0 + 32 * k;
          if (v < nv) {
            float w[8], xv[8];
            Vec8<T>::cvt(u[k], w);
            uint4 xu[LD];
#pragma unroll
            for (int l = 0; l < LD; ++l)
              xu[l] = *reinterpret_cast<const uint4*>(reinterpret_cast<const unsigned char*>(xs + (size_t)v * 8) + l * 16);
            Vec8<T>::cvt(xu, xv);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc = fmaf(w[e], xv[e], acc);
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) {
        __stcg(p.x_rot + row, acc);
        const uint32_t key = __float_as_uint(acc) & kKeyMask;
        if (row - r0 < kRowKeys)
          s_rowkey[row - r0] = key;
        else  // more rows than the buffer holds (very small grids): count directly
          atomicAdd(p.sync + kFusedSyncWords + 2 * kFusedMaxTiles + (s_gen & 1u) * kFusedHistBins +
                        (key >> kFineShift), 1u);
      }
    }
  } else {
    // the identity rotation (no Q): x_rot = x widened to fp32
    __syncthreads();  // s_gen
    const T* xv = static_cast<const T*>(p.x);
    for (int row = r0 + tid; row < r1; row += kT) {
      const float v = to_f32(xv[row]);
      __stcg(p.x_rot + row, v);
      const uint32_t key = __float_as_uint(v) & kKeyMask;
      if (row - r0 < kRowKeys)
        s_rowkey[row - r0] = key;
      else
        atomicAdd(p.sync + kFusedSyncWords + 2 * kFusedMaxTiles + (s_gen & 1u) * kFusedHistBins +
                      (key >> kFineShift), 1u);
    }
  }
  __syncthreads();  // the staged x is dead; this CTA's rows are written
  const unsigned gen = s_gen;
  unsigned* ticket = p.sync + (gen & 1u);
  unsigned* ghist = p.sync + kFusedSyncWords + 2 * kFusedMaxTiles + (gen & 1u) * kFusedHistBins;
  if (warp == 0 && !p.thresh) {
    // this CTA's rows into the call's histogram of bits 30..19 of |x_rot|:
    // equal bins among 32 rows are added once
    const int nk = min(r1 - r0, kRowKeys);
    for (int i0 = 0; i0 < nk; i0 += 32) {
      const bool has = i0 + lane < nk;
      const uint32_t bin = has ? s_rowkey[i0 + lane] >> kFineShift : 0xffffffffu;
      const uint32_t same = __match_any_sync(0xffffffffu, bin);
      if (has && lane == __ffs(same) - 1) atomicAdd(ghist + bin, static_cast<unsigned>(__popc(same)));
    }
  }
  __syncthreads();  // the histogram adds come before the arrival
  if (tid == 0) atomic_add_release_gpu(ticket, 1u);  // publishes the CTA's rows with its arrival
  const unsigned target = static_cast<unsigned>(G);

  if (cta == G - 1) {
    // ---- 2. the selector: 16-bit bin numbers of all d entries in shared
    // memory, full keys read from x_rot in L2 where a bin does not decide
    uint16_t* bins = reinterpret_cast<uint16_t*>(smem_raw + L.bins);
    uint32_t* cand = reinterpret_cast<uint32_t*>(smem_raw + L.cand);
    uint32_t* cand_idx = reinterpret_cast<uint32_t*>(smem_raw + L.cand_idx);
    const uint32_t* xkeys = reinterpret_cast<const uint32_t*>(p.x_rot);
    for (int j = tid; j < kFusedCandCap; j += kT) {  // empty candidate slots (see select_kth)
      cand[j] = 0u;
      cand_idx[j] = 0xffffffffu;
    }
    if (tid == 0) {
      const bool ok = wait_word(ticket, target, p.wait_ns);
      if (!ok) report(p.dev_status, LAROSA_DEV_TIMEOUT);
      s_word[0] = ok;
      s_word[1] = 0u;  // boundary candidates listed
    }
    __syncthreads();
    const bool ok = s_word[0] != 0u;
    // 0 keeps nothing, 1 Top-K, 2 keeps all, 3 threshold
    const uint32_t mode = !ok ? 0u : p.thresh ? 3u : (K <= 0 ? 0u : (K >= d ? 2u : 1u));
    // one batch of L2 reads, made while the gather CTAs find the boundary
    // and before they stream: this thread's share of the call's histogram
    // and the first kPre vectors of x_rot
    uint32_t hcnt[kHistShare<kT>];
    uint4 pre[kPre];
    if (mode == 1u) {
      hist_share<kT, true>(ghist, hcnt);
#pragma unroll
      for (int k = 0; k < kPre; ++k) {
        const int v = tid + k * kT;
        pre[k] = v < d / 4 ? __ldcg(reinterpret_cast<const uint4*>(xkeys) + v) : make_uint4(0, 0, 0, 0);
      }
    }
    uint32_t B = 0, above = 0, nB = 0;
    KthEntry e{0xffffffffu, -1};  // after a timeout: no bin-B row is kept
    bool nonfinite = false;
    if (mode == 1u) {
      boundary_from_share<kT>(hcnt, K, s_warp_sums, s_pick, &B, &above, &nB);
      // list B's keys, or where B holds more than the slots, those of the
      // sub-bin of B that holds the K-th entry; only when that too overflows
      // (heavy ties) does the bisection over all keys decide
      const uint32_t krem = static_cast<uint32_t>(K) - above;
      if (nB <= static_cast<uint32_t>(kFusedCandCap)) {
        e = select_kth<true>(xkeys, d, kFineShift, B, krem, pre, bins, cand, cand_idx, s_word + 1, s_pick,
                             &nonfinite);
      } else {
        e = select_crowded(xkeys, d, K, B, krem, bins, s_rowkey, cand, cand_idx, s_word + 1, s_pick, s_warp_sums,
                           &nonfinite);
      }
    }
    if (tid == 0) {
      // the entry and this call's tag in one release store; the call number,
      // read only by the next call once this one has completed, follows
      st_release_gpu_u64(reinterpret_cast<unsigned long long*>(p.sync + 4), pack_kth(e.T, e.I, gen));
      p.sync[3] = gen;
    }
    if (nonfinite) report(p.dev_status, LAROSA_DEV_NONFINITE);
    // the kept list for callers, off the gather's path
    if (mode == 1u) {
      __syncthreads();  // warp_sums may be reused
      fused_export(xkeys, bins, d, B, e, false, cand, p.idx, p.val, s_warp_sums);
    } else if (mode == 2u) {
      for (int i = tid; i < d; i += kT) {
        const uint32_t u = __ldcg(xkeys + i);
        if ((u & kKeyMask) >= 0x7f800000u) report(p.dev_status, LAROSA_DEV_NONFINITE);
        p.idx[i] = i;
        p.val[i] = __uint_as_float(u);
      }
    } else if (mode == 3u) {
      bool bad = false;
      const uint32_t n = export_threshold(xkeys, d, p.t_key, p.idx, p.val, s_warp_sums, &bad);
      if (bad) report(p.dev_status, LAROSA_DEV_NONFINITE);
      if (tid == 0) p.nnz[0] = static_cast<int32_t>(n);
    } else if (p.thresh && tid == 0) {
      p.nnz[0] = 0;  // after a timeout
    }
    // the next call's counters and histogram (call n - 1, which used them,
    // is done); last, so that these stores do not queue ahead of the
    // selection's loads
    {
      uint4* hn = reinterpret_cast<uint4*>(p.sync + kFusedSyncWords + 2 * kFusedMaxTiles +
                                           ((gen + 1u) & 1u) * kFusedHistBins);
      for (int i = tid; i < kFusedHistBins / 4; i += kT) hn[i] = make_uint4(0, 0, 0, 0);
      unsigned* tiles_next = p.sync + kFusedSyncWords + ((gen + 1u) & 1u) * kFusedMaxTiles;
      for (int t = tid; t < p.n_tiles; t += kT) tiles_next[t] = 0u;
      if (tid == 0) p.sync[(gen + 1u) & 1u] = 0u;
    }
    return;
  }

  // ---- 3. a gather CTA: rank r owns the indices [i_lo, i_hi)
  // region A: the range's keys, later the row-group partials
  uint32_t* rkeys = reinterpret_cast<uint32_t*>(smem_raw);
  int32_t* lrows = reinterpret_cast<int32_t*>(smem_raw + L.rows);
  float* lvals = reinterpret_cast<float*>(smem_raw + L.vals);
  float* red = reinterpret_cast<float*>(smem_raw + L.red);
  const int i_lo = (int)((long long)d * rank / C);
  const int n_r = (int)((long long)d * (rank + 1) / C) - i_lo;
  const int c0 = tile * p.col_tile;
  const int wc = min(p.col_tile, p.d_out - c0);
  float acc[CPT];
#pragma unroll
  for (int v = 0; v < CPT; ++v) acc[v] = 0.f;

  // every CTA's x_rot is written and counted: load this range while the
  // selector works.  With the identity rotation and a threshold, whether an
  // entry is kept depends on that entry alone and x_rot is x widened, so the
  // range's keys come straight from x and nothing waits for the other CTAs.
  // (For the Top-K, each CTA counting the histogram of all of x itself, to
  // skip the wait, was 31 % slower: its rows then stream while the selector
  // still reads x_rot, and the selector's round trips queue behind them.)
  const bool direct = !p.rotate && p.thresh;
  if (tid == 0) {
    const bool ok = direct || wait_word(ticket, target, p.wait_ns);
    if (!ok) report(p.dev_status, LAROSA_DEV_TIMEOUT);
    s_word[0] = ok;
  }
  __syncthreads();
  const bool arrived = s_word[0] != 0u;
  // 0 keeps nothing, 1 Top-K, 2 keeps all, 3 threshold
  const uint32_t mode = !arrived ? 0u : p.thresh ? 3u : (K <= 0 ? 0u : (K >= d ? 2u : 1u));
  uint32_t hcnt[kHistShare<kT>];  // this thread's share of the call's histogram
  if (mode == 1u) hist_share<kT, true>(ghist, hcnt);
  if (direct) {
    const T* xv = static_cast<const T*>(p.x) + i_lo;
    for (int j = tid; j < n_r; j += kT) rkeys[j] = __float_as_uint(to_f32(xv[j]));
  } else if (arrived) {
    for (int j0 = tid; j0 < n_r; j0 += kT * kU) {
      uint32_t u[kU];
#pragma unroll
      for (int k = 0; k < kU; ++k) {
        const int j = j0 + k * kT;
        u[k] = j < n_r ? __float_as_uint(__ldcg(p.x_rot + i_lo + j)) : 0u;
      }
#pragma unroll
      for (int k = 0; k < kU; ++k)
        if (j0 + k * kT < n_r) rkeys[j0 + k * kT] = u[k];
    }
  }
  // the boundary bin, from the call's histogram (read from L2): rows above
  // it are certainly kept
  uint32_t B = 0, above = 0, nB = 0;
  if (mode == 1u) {
    boundary_from_share<kT>(hcnt, K, s_warp_sums, s_pick, &B, &above, &nB);
  } else {
    __syncthreads();  // the range's keys are in shared memory
  }
  const int n_certain = compact_range(
      rkeys, n_r, i_lo,
      [&](uint32_t k, int) {
        return mode == 2u || (mode == 3u && k >= p.t_key) || (mode == 1u && (k >> kFineShift) > B);
      },
      lrows, lvals, 0, s_warp_sums);
  __syncthreads();  // the certain list is in place
  if (mode == 1u) {
    // Some rows of bin B are kept too; which ones is known only once the
    // selector has ranked them.  Their segments of this column tile are few
    // (about nB / C per CTA): have them brought into L2 now, so that reading
    // the kept ones later costs an L2 rather than an HBM round trip.
    const unsigned char* wtile = static_cast<const unsigned char*>(p.W) + (size_t)c0 * sizeof(T);
    const size_t pitch = (size_t)p.d_out * sizeof(T);
    for (int j = tid; j < n_r; j += kT)
      if (((rkeys[j] & kKeyMask) >> kFineShift) == B)
        bulk_prefetch_l2(wtile + (size_t)(i_lo + j) * pitch, static_cast<uint32_t>(wc * sizeof(T)));
  }
  accumulate_rows<T, kFusedU>(p.W, p.d_out, c0, wc, p.tpr, lrows, lvals, 0, n_certain, acc);

  // the K-th entry: the kept rows of bin B
  if (tid == 0) {
    bool got = false;
    unsigned long long w = 0;
    if (mode == 1u) {
      got = wait_kth(reinterpret_cast<const unsigned long long*>(p.sync + 4), gen, &w, p.wait_ns);
      if (!got) report(p.dev_status, LAROSA_DEV_TIMEOUT);
    }
    s_word[4] = got ? static_cast<uint32_t>(w) : 0u;  // T
    s_word[5] = got ? static_cast<uint32_t>(static_cast<int32_t>(static_cast<int16_t>((w >> 32) & 0xffffu)))
                    : 0u;  // I, sign-extended
    s_word[6] = got;
  }
  __syncthreads();
  const bool have_kth = s_word[6] != 0u;
  const KthEntry e{s_word[4], static_cast<int32_t>(s_word[5])};
  const int n_more = compact_range(
      rkeys, n_r, i_lo,
      [&](uint32_t k, int i) { return have_kth && (k >> kFineShift) == B && is_kept(k, i, e); },
      lrows, lvals, n_certain, s_warp_sums);
  __syncthreads();  // the list is complete; the range's keys are dead
  accumulate_rows<T, kFusedU>(p.W, p.d_out, c0, wc, p.tpr, lrows, lvals, n_certain, n_certain + n_more, acc);
  reduce_tile_last<T, C>(rank, c0, wc, p.col_tile, p.tpr, acc, red,
                         p.partials + (size_t)tile * C * p.col_tile,
                         p.sync + kFusedSyncWords + (gen & 1u) * kFusedMaxTiles + tile, p.y);
}

// ================================================================ sparse + low rank, one token
//
// R-Sparse report, 研究流程与方法 / R-Sparse框架设计 (hybrid computation): the
// entries a selection drops go through rank-r factors of the weight instead
// of being discarded, y = sum_{k} val[k] W[idx[k]] + ((x - sigma(x)) . A_r) . B_r.
// One cooperative launch of n_tiles * C column-tile CTAs and F factor CTAs,
// all resident at once:
//   * factor CTA q takes the indices [d q / F, d (q + 1) / F) of x, zeroes
//     the kept ones (what is left is its share of the dropped vector), lists
//     the nonzero entries in index order and streams only those rows of A_r,
//     every column, into a partial u_q = x_drop[range] . A_r[range]; it writes
//     u_q to the workspace and arrives on a counter.  F is chosen so that a
//     factor CTA has about two batches of row loads, which keeps u off the
//     critical path;
//   * column-tile CTA (tile, rank) streams positions [K rank / C,
//     K (rank + 1) / C) of the kept list of W for its columns, waits for
//     every factor CTA, adds the F partials of its entries [r rank / C,
//     r (rank + 1) / C) of u in factor order, streams those rows of B_r with
//     them as coefficients into the same partial sums, and the last CTA of
//     the tile adds the C partials in rank order (y = y_s + y_r).  (Asking
//     for the B_r rows to be brought into L2 before the kept rows was
//     measured 1.6 % slower: the prefetches queue ahead of the kept rows.)
// Every sum has a fixed order, so results repeat bit for bit.  Counter words
// in the workspace, all zero between calls: [0] factor CTAs done, [1]
// column-tile CTAs that have seen them (the last resets both), [2 + t]
// column tile t's CTAs done (its last CTA resets it).  A wait that runs out
// reports LAROSA_DEV_TIMEOUT; the workspace must then be zeroed.

struct LRParams {
  const float* x;       // [d] the vector the selection was made on (fp32)
  const int32_t* idx;   // [K] kept list
  const float* val;     // [K]
  const void* W;        // [d x d_out]
  const void* A_r;      // [d x r]
  const void* B_r;      // [r x d_out]
  float* y;             // [d_out]
  float* u;             // [F x r] workspace: the factor CTAs' partials of u
  float* partials;      // [n_tiles x C x col_tile] workspace
  unsigned* sync;       // [2 + n_tiles] counters, workspace
  int d;
  int d_out;
  int K;
  int r;
  int col_tile;
  int tpr;
  int list_cap;         // entries a column-tile CTA lists: max(ceil(K / C), ceil(r / C))
  int n_tiles;
  int f_ctas;           // factor CTAs F
  int f_len;            // indices of x a factor CTA covers at most: ceil(d / F)
  int* dev_status;
  unsigned long long wait_ns;
};

constexpr int kLRMaxF = kLowrankMaxFactorCtas;  // factor CTAs at most
constexpr int kLRMaxRank = 2048;   // r: one A_r row per at most kT / 2 threads
constexpr int kLRMaxLen = 4096;    // indices of x per factor CTA at most (shared memory)
constexpr int kLRMaxD = kLRMaxF * kLRMaxLen;

struct LRLayout {
  size_t keys, red, rows, vals, total;
};

// Column-tile CTA: its row-group partials (red), then the kept / B_r row
// lists.  The partials' space also serves to add the factor partials of u.
__host__ __device__ inline LRLayout lr_tile_layout(int list_cap, int col_tile, int cpt) {
  LRLayout L{};
  const size_t red = al16((size_t)(kT / (col_tile / cpt)) * col_tile * 4);
  L.keys = 0;
  L.red = 0;
  L.rows = red;
  L.vals = al16(L.rows + (size_t)list_cap * 4);
  L.total = al16(L.vals + (size_t)list_cap * 4);
  return L;
}

// Factor CTA: the keys of its range of x, the row-group partials of u, its
// list of dropped rows.
__host__ __device__ inline LRLayout lr_factor_layout(int len, int cpt) {
  LRLayout L{};
  L.keys = 0;
  L.red = al16((size_t)len * 4);
  L.rows = al16(L.red + (size_t)kT * cpt * 4);
  L.vals = al16(L.rows + (size_t)len * 4);
  L.total = al16(L.vals + (size_t)len * 4);
  return L;
}

// Floats of the column-tile CTA's partials space (used to add the factor
// partials of u, F per entry).
__host__ __device__ inline int lr_red_floats(int col_tile, int cpt) {
  return (kT / (col_tile / cpt)) * col_tile;
}

template <typename Tw, int C>
__global__ void __launch_bounds__(kT, 2) lowrank_kernel(const LRParams p) {
  constexpr int CPT = 16 / sizeof(Tw);
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ uint32_t s_word[2];
  __shared__ uint32_t s_warp_sums[32];
  const int tid = threadIdx.x;
  const int n_tile_ctas = p.n_tiles * C;
  const int cta = blockIdx.x;
  const int d = p.d, K = p.K;
  pdl_wait();
  pdl_launch_dependents();

  if (cta >= n_tile_ctas) {
    // ---- factor CTA q: u_q = x_drop[i_lo, i_hi) . A_r[i_lo, i_hi)
    const LRLayout L = lr_factor_layout(p.f_len, CPT);
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + L.keys);
    float* red = reinterpret_cast<float*>(smem_raw + L.red);
    int32_t* frows = reinterpret_cast<int32_t*>(smem_raw + L.rows);
    float* fvals = reinterpret_cast<float*>(smem_raw + L.vals);
    const int q = cta - n_tile_ctas;
    const int i_lo = (int)((long long)d * q / p.f_ctas), i_hi = (int)((long long)d * (q + 1) / p.f_ctas);
    const int n = i_hi - i_lo;
    for (int i = tid; i < n; i += kT) keys[i] = __float_as_uint(__ldg(p.x + i_lo + i));
    __syncthreads();
    bool bad = false;
    for (int k = tid; k < K; k += kT) {
      const int i = __ldg(p.idx + k);
      if (static_cast<unsigned>(i) >= static_cast<unsigned>(d))
        bad = true;
      else if (i >= i_lo && i < i_hi)
        keys[i - i_lo] = 0u;  // kept: not part of the dropped vector
    }
    if (__syncthreads_or(bad) && tid == 0 && q == 0) report(p.dev_status, LAROSA_DEV_INDEX);
    // the dropped entries with a nonzero value, in index order
    const int nd = compact_range(
        keys, n, i_lo, [](uint32_t k, int) { return k != 0u; }, frows, fvals, 0, s_warp_sums);
    __syncthreads();
    const int tpr = p.r / CPT;  // r is a multiple of CPT
    float acc[CPT];
#pragma unroll
    for (int v = 0; v < CPT; ++v) acc[v] = 0.f;
    accumulate_rows<Tw, kFusedU>(p.A_r, p.r, 0, p.r, tpr, frows, fvals, 0, nd, acc);
    const int ng = kT / tpr;
    const int g = tid / tpr;
    const int col = (tid - g * tpr) * CPT;
    if (g < ng) {
#pragma unroll
      for (int v = 0; v < CPT; ++v) red[g * p.r + col + v] = acc[v];
    }
    __syncthreads();
    float* uq = p.u + (size_t)q * p.r;
    for (int e = tid; e < p.r; e += kT) {
      float s = 0.f;
      for (int gg = 0; gg < ng; ++gg) s += red[gg * p.r + e];  // row groups in order
      __stcg(uq + e, s);
    }
    __syncthreads();  // this CTA's partial of u is written
    if (tid == 0) atomic_add_release_gpu(p.sync, 1u);
    return;
  }

  // ---- column-tile CTA
  const LRLayout L = lr_tile_layout(p.list_cap, p.col_tile, CPT);
  int32_t* lrows = reinterpret_cast<int32_t*>(smem_raw + L.rows);
  float* lvals = reinterpret_cast<float*>(smem_raw + L.vals);
  float* red = reinterpret_cast<float*>(smem_raw + L.red);
  const int tile = cta / C, rank = cta - tile * C;
  const int c0 = tile * p.col_tile;
  const int wc = min(p.col_tile, p.d_out - c0);
  const int q0 = (int)((long long)p.r * rank / C), q1 = (int)((long long)p.r * (rank + 1) / C);
  float acc[CPT];
#pragma unroll
  for (int v = 0; v < CPT; ++v) acc[v] = 0.f;
  {
    // y_s: positions [p0, p1) of the kept list
    const int p0 = (int)((long long)K * rank / C), p1 = (int)((long long)K * (rank + 1) / C);
    bool bad = false;
    for (int j = tid; j < p1 - p0; j += kT) {
      const int row = __ldg(p.idx + p0 + j);
      const bool ok = static_cast<unsigned>(row) < static_cast<unsigned>(d);
      bad |= !ok;
      lrows[j] = ok ? row : 0;
      lvals[j] = ok ? __ldg(p.val + p0 + j) : 0.f;
    }
    if (__syncthreads_or(bad) && tid == 0) report(p.dev_status, LAROSA_DEV_INDEX);
    accumulate_rows<Tw, kFusedU>(p.W, p.d_out, c0, wc, p.tpr, lrows, lvals, 0, p1 - p0, acc);
  }
  // every factor CTA has written its partial of u
  if (tid == 0) {
    const bool ok = wait_word(p.sync, static_cast<unsigned>(p.f_ctas), p.wait_ns);
    if (!ok) {
      report(p.dev_status, LAROSA_DEV_TIMEOUT);
    } else if (atomicAdd(p.sync + 1, 1u) == static_cast<unsigned>(n_tile_ctas - 1)) {
      // the last column-tile CTA to see the factor CTAs: both counters back to zero
      p.sync[0] = 0u;
      p.sync[1] = 0u;
    }
    s_word[0] = ok;
  }
  __syncthreads();  // this CTA's kept rows are consumed: the lists are free
  if (s_word[0] != 0u) {
    // u[q0, q1): the F partials of each entry, added in factor order, a
    // chunk of entries at a time through the partials space
    const int F = p.f_ctas;
    const int chunk = max(1, lr_red_floats(p.col_tile, CPT) / F);
    for (int j0 = q0; j0 < q1; j0 += chunk) {
      const int m = min(chunk, q1 - j0);
      for (int t0 = tid; t0 < m * F; t0 += 4 * kT) {
        float v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int t = t0 + k * kT;
          const int f = t / m;
          v[k] = t < m * F ? __ldcg(p.u + (size_t)f * p.r + j0 + (t - f * m)) : 0.f;
        }
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (t0 + k * kT < m * F) red[t0 + k * kT] = v[k];
      }
      __syncthreads();
      for (int j = tid; j < m; j += kT) {
        float s = 0.f;
        for (int f = 0; f < F; ++f) s += red[f * m + j];
        lrows[j0 - q0 + j] = j0 + j;
        lvals[j0 - q0 + j] = s;
      }
      __syncthreads();
    }
    // y_r: rows [q0, q1) of B_r, coefficients u
    accumulate_rows<Tw, kFusedU>(p.B_r, p.d_out, c0, wc, p.tpr, lrows, lvals, 0, q1 - q0, acc);
  }
  reduce_tile_last<Tw, C>(rank, c0, wc, p.col_tile, p.tpr, acc, red, p.partials + (size_t)tile * C * p.col_tile,
                          p.sync + 2 + tile, p.y);
  // reduce_tile_last returns in every CTA; the counter of the tile now holds
  // C, and only after its last CTA has read it: reset by that CTA (which
  // saw C - 1 and is the only one still running this tile)
  if (tid == 0 && ld_acquire_gpu(p.sync + 2 + tile) == static_cast<unsigned>(C)) {
    // every CTA of the tile has arrived; the one that reduced may still be
    // reading the partials, so only the counter is reset
    atomicCAS(p.sync + 2 + tile, static_cast<unsigned>(C), 0u);
  }
}

struct DevState {
  int sms = 0;
  bool configured[24] = {};  // kernel slots whose shared-memory ceiling is set
};
DevState g_state[64];

cudaError_t dev_state(DevState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  DevState& ds = g_state[dev];
  if (ds.sms == 0) {
    e = cudaDeviceGetAttribute(&ds.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  *out = &ds;
  return cudaSuccess;
}

cudaError_t configure(DevState* ds, int slot, void* fn, size_t smem) {
  if (!ds->configured[slot]) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    ds->configured[slot] = true;
  }
  return cudaSuccess;
}

cudaError_t launch(void* fn, int grid, size_t smem, void* params, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kT, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* args[] = {params};
  return cudaLaunchKernelExC(&cfg, fn, args);
}

template <typename T>
void* rowdot_fn(int MT) {
  switch (MT) {
    case 1: return reinterpret_cast<void*>(&rowdot_kernel<T, 1>);
    case 2: return reinterpret_cast<void*>(&rowdot_kernel<T, 2>);
    case 4: return reinterpret_cast<void*>(&rowdot_kernel<T, 4>);
    case 8: return reinterpret_cast<void*>(&rowdot_kernel<T, 8>);
    default: return reinterpret_cast<void*>(&rowdot_kernel<T, 16>);
  }
}

int round_up_mt(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16; }

}  // namespace

// The identity rotation for the composed paths: x_rot = x widened to fp32.
template <typename T>
__global__ void __launch_bounds__(kT) widen_kernel(const T* __restrict__ x, float* __restrict__ x_rot,
                                                   int n) {
  pdl_wait();
  pdl_launch_dependents();
  for (int i = blockIdx.x * kT + threadIdx.x; i < n; i += gridDim.x * kT) x_rot[i] = to_f32(x[i]);
}

// ---------------------------------------------------------------- host API

cudaError_t launch_rowdot(Elem e, const void* A, const void* x, float* y, int M, int n_in,
                          int n_out, cudaStream_t stream) {
  DevState* ds = nullptr;
  cudaError_t err = dev_state(&ds);
  if (err != cudaSuccess) return err;
  if (e == Elem::BF16 && rot_umma_applies(M, n_in, n_out))
    return launch_rot_umma(A, x, y, M, n_in, n_out, nullptr, stream);
  if (e == Elem::BF16 && M >= kMmaMinTokens && n_in % 32 == 0 && n_out % 8 == 0) {
    MParams p;
    p.A = A;
    p.x = x;
    p.y = y;
    p.n_in = n_in;
    p.n_out = n_out;
    p.M = M;
    void* fn = M > 8 ? reinterpret_cast<void*>(&rowmma_kernel<true>)
                     : reinterpret_cast<void*>(&rowmma_kernel<false>);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(n_out / 8, 1, 1);
    cfg.blockDim = dim3(kMmaWarps * 32, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {&p};
    return cudaLaunchKernelExC(&cfg, fn, args);
  }
  const int MT = round_up_mt(M);
  const int esz = e == Elem::BF16 ? 2 : 4;
  const size_t xbytes = (size_t)M * n_in * esz;
  const bool in_smem = xbytes <= (size_t)kXSmemBytes;
  const int mt_idx = MT == 1 ? 0 : MT == 2 ? 1 : MT == 4 ? 2 : MT == 8 ? 3 : 4;
  void* fn = e == Elem::BF16 ? rowdot_fn<__nv_bfloat16>(MT) : rowdot_fn<float>(MT);
  err = configure(ds, (e == Elem::BF16 ? 5 : 0) + mt_idx, fn, kXSmemBytes);
  if (err != cudaSuccess) return err;
  RParams p;
  p.A = A;
  p.x = x;
  p.y = y;
  p.n_in = n_in;
  p.n_out = n_out;
  p.M = M;
  p.x_in_smem = in_smem ? 1 : 0;
  const int per_sm = (MT <= 2 && e == Elem::BF16) ? 2 : 1;
  const int grid = std::max(1, std::min(ds->sms * per_sm, n_out));
  return launch(fn, grid, in_smem ? xbytes : 0, &p, stream);
}

cudaError_t launch_widen(const void* x, float* x_rot, int n, Elem elem, cudaStream_t stream) {
  DevState* ds = nullptr;
  cudaError_t e = dev_state(&ds);
  if (e != cudaSuccess) return e;
  const int grid = std::max(1, std::min((n + kT - 1) / kT, 2 * ds->sms));
  void* fn = elem == Elem::BF16 ? reinterpret_cast<void*>(&widen_kernel<__nv_bfloat16>)
                                : reinterpret_cast<void*>(&widen_kernel<float>);
  struct {
    const void* x;
    float* x_rot;
    int n;
  } a{x, x_rot, n};
  void* args[] = {&a.x, &a.x_rot, &a.n};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kT, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

// ---------------------------------------------------------------- rotate + select

// The kernel also holds a few words of static shared memory; the dynamic
// part stays below the per-block limit minus that.
constexpr int kRotSelSmemCeiling = kGatherSmemCeiling - 1024;

bool rotsel_fits(Elem e, int d) {
  const int esz = e == Elem::BF16 ? 2 : 4;
  return d >= 8 && d % 8 == 0 && rslayout(d, esz).total <= (size_t)kRotSelSmemCeiling;
}

cudaError_t launch_rotsel(Elem e, const RotSelArgs& a, cudaStream_t stream) {
  if (!rotsel_fits(e, a.d) || a.K < 0 || a.K > a.d) return cudaErrorInvalidValue;
  DevState* ds = nullptr;
  cudaError_t err = dev_state(&ds);
  if (err != cudaSuccess) return err;
  const int esz = e == Elem::BF16 ? 2 : 4;
  void* fn = e == Elem::BF16 ? reinterpret_cast<void*>(&rotsel_kernel<__nv_bfloat16>)
                             : reinterpret_cast<void*>(&rotsel_kernel<float>);
  // the attribute is a ceiling for every launch of fn
  err = configure(ds, 10 + (e == Elem::BF16 ? 1 : 0), fn, kRotSelSmemCeiling);
  if (err != cudaSuccess) return err;
  const size_t smem = rslayout(a.d, esz).total;
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kT, smem);
  if (err != cudaSuccess) return err;
  per_sm = std::max(1, std::min(per_sm, 2));
  RSParams p;
  p.x = a.x;
  p.Qt = a.Qt;
  p.x_rot = a.x_rot;
  p.idx = a.idx;
  p.val = a.val;
  p.ticket = a.ticket;
  p.d = a.d;
  p.K = a.K;
  p.dev_status = a.dev_status;
  const int grid = std::max(1, std::min(ds->sms * per_sm, a.d));
  return launch(fn, grid, smem, &p, stream);
}

namespace {

// Largest number of co-resident clusters of C CTAs for a kernel and shared
// memory size, cached per device.
struct ClusterOcc {
  void* fn;
  size_t smem;
  int C;
  int clusters;
};
std::mutex g_occ_mu;
ClusterOcc g_occ[64][64];
int g_occ_n[64] = {0};

cudaError_t max_clusters(int dev, void* fn, size_t smem, int C, int* out,
                         int ceiling = kGatherSmemCeiling) {
  {
    std::lock_guard<std::mutex> lock(g_occ_mu);
    for (int i = 0; i < g_occ_n[dev]; ++i) {
      const ClusterOcc& o = g_occ[dev][i];
      if (o.fn == fn && o.smem == smem && o.C == C) {
        *out = o.clusters;
        return cudaSuccess;
      }
    }
  }
  // the attribute is a ceiling for every launch of fn: set it to the largest
  // size a launch may use, not to the size probed here
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, ceiling);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, 64, 1);
  cfg.blockDim = dim3(kT, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  e = cudaOccupancyMaxActiveClusters(&n, fn, &cfg);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    n = 0;
  }
  std::lock_guard<std::mutex> lock(g_occ_mu);
  if (g_occ_n[dev] < 64) g_occ[dev][g_occ_n[dev]++] = ClusterOcc{fn, smem, C, n};
  *out = n;
  return cudaSuccess;
}

template <int C>
void* gather_fn_c(Elem w) {
  return w == Elem::BF16 ? reinterpret_cast<void*>(&gather_kernel<__nv_bfloat16, C>)
                         : reinterpret_cast<void*>(&gather_kernel<float, C>);
}

void* gather_fn(Elem w, int C) { return C == 8 ? gather_fn_c<8>(w) : gather_fn_c<4>(w); }

}  // namespace

// Launch plans already computed, per device, kernel and sizes: a plan costs
// occupancy queries, and the one-token calls are made once per token.
struct PlanKey {
  int dev, kind, elem, a, b, c, r;
  bool operator==(const PlanKey& o) const {
    return dev == o.dev && kind == o.kind && elem == o.elem && a == o.a && b == o.b && c == o.c && r == o.r;
  }
};
struct PlanEntry {
  PlanKey key;
  StreamPlan plan;
};
std::mutex g_plan_mu;
PlanEntry g_plans[512];
int g_plan_n = 0, g_plan_next = 0;

template <typename F>
cudaError_t cached_plan(PlanKey key, StreamPlan* plan, F compute) {
  cudaError_t e = cudaGetDevice(&key.dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(g_plan_mu);
    for (int i = 0; i < g_plan_n; ++i)
      if (g_plans[i].key == key) {
        *plan = g_plans[i].plan;
        return cudaSuccess;
      }
  }
  e = compute(plan);  // also sets the kernel's attributes on this device
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_plan_mu);
  PlanEntry& en = g_plans[g_plan_n < 512 ? g_plan_n++ : (g_plan_next++ & 511)];
  en = PlanEntry{key, *plan};
  return cudaSuccess;
}

static cudaError_t plan_gather_uncached(Elem w_elem, int d_out, int K, StreamPlan* plan) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const int cpt = w_elem == Elem::BF16 ? 8 : 4;
  StreamPlan best;
  *plan = best;
  long long best_ctas = -1;
  // Clusters of 8 give the widest column tiles; clusters of 4 pack the SMs
  // more evenly (the GPU holds fewer 8-CTA clusters than its CTA slots allow).
  // Take the size that keeps more CTAs streaming at once.
  for (int C : {8, 4}) {
    void* fn = gather_fn(w_elem, C);
    const int list_cap = std::max(1, (K + C - 1) / C);
    // column tile: fill the co-resident clusters, at least 64 columns wide
    // (128 bytes of bf16) and at most one 16-byte vector per thread
    const int wc_max = kT * cpt;
    const size_t smem_probe = glayout(list_cap, wc_max, cpt).total;
    if (smem_probe > (size_t)kGatherSmemCeiling) continue;
    int clusters = 0;
    e = max_clusters(dev, fn, smem_probe, C, &clusters);
    if (e != cudaSuccess) return e;
    if (clusters <= 0) continue;
    int wc = (d_out + clusters - 1) / clusters;
    wc = std::max(wc, std::min(64, d_out));
    wc = (wc + cpt - 1) / cpt * cpt;
    wc = std::min(wc, wc_max);
    const int n_tiles = (d_out + wc - 1) / wc;
    const long long ctas = (long long)std::min(n_tiles, clusters) * C;
    if (ctas > best_ctas) {
      best_ctas = ctas;
      best.ok = true;
      best.cluster = C;
      best.n_tiles = n_tiles;
      best.col_tile = wc;
      best.tpr = wc / cpt;
      best.list_cap = list_cap;
      best.smem = glayout(list_cap, wc, cpt).total;
      best.smem_alloc = smem_probe;
    }
  }
  *plan = best;
  return cudaSuccess;
}

cudaError_t launch_gather(Elem w_elem, const GatherArgs& a, const StreamPlan& pl,
                          cudaStream_t stream) {
  if (!pl.ok || (pl.cluster != 4 && pl.cluster != 8)) return cudaErrorInvalidValue;
  void* fn = gather_fn(w_elem, pl.cluster);
  GParams p;
  p.W = a.W;
  p.d_out = a.d_out;
  p.d_in = a.row_bound;
  p.K = a.n;
  p.coef = a.coef;
  p.rows = a.rows;
  p.y = a.y;
  p.col_tile = pl.col_tile;
  p.tpr = pl.tpr;
  p.list_cap = pl.list_cap;
  p.dev_status = a.dev_status;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.cluster, pl.n_tiles, 1);
  cfg.blockDim = dim3(kT, 1, 1);
  cfg.dynamicSmemBytes = pl.smem;
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

namespace {

template <int C>
void* fused_fn_c(Elem w) {
  return w == Elem::BF16 ? reinterpret_cast<void*>(&fused_kernel<__nv_bfloat16, C>)
                         : reinterpret_cast<void*>(&fused_kernel<float, C>);
}

void* fused_fn(Elem w, int C) { return C == 8 ? fused_fn_c<8>(w) : fused_fn_c<4>(w); }

// The fused kernel also holds about 1.2 KB of static shared memory.
constexpr int kFusedSmemCeiling = kGatherSmemCeiling - 4096;

}  // namespace

static cudaError_t plan_fused_uncached(Elem w_elem, int d_in, int d_out, int K, StreamPlan* plan) {
  DevState* ds = nullptr;
  cudaError_t e = dev_state(&ds);
  if (e != cudaSuccess) return e;
  StreamPlan best;
  *plan = best;
  if (d_in < 8 || d_in % 8 != 0 || K < 0 || K > d_in) return cudaSuccess;
  const int cpt = w_elem == Elem::BF16 ? 8 : 4;
  const int esz = w_elem == Elem::BF16 ? 2 : 4;
  long long best_ctas = -1;
  for (int C : {8, 4}) {
    void* fn = fused_fn(w_elem, C);
    const int range_cap = (d_in + C - 1) / C;
    const int wc_max = kT * cpt;
    const size_t smem_probe = flayout(d_in, esz, range_cap, wc_max, cpt).total;
    if (smem_probe > (size_t)kFusedSmemCeiling) continue;
    // the attribute is a ceiling for every launch of fn
    e = configure(ds, 12 + (w_elem == Elem::BF16 ? 2 : 0) + (C == 8 ? 1 : 0), fn, kFusedSmemCeiling);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kT, smem_probe);
    if (e != cudaSuccess) return e;
    const int gather_ctas = ds->sms * per_sm - 1;  // every CTA resident; one selects
    const int tiles = std::min(gather_ctas / C, kFusedMaxTiles);
    if (tiles < 1) continue;
    int wc = (d_out + tiles - 1) / tiles;
    wc = std::max(wc, std::min(64, d_out));
    wc = (wc + cpt - 1) / cpt * cpt;
    wc = std::min(wc, wc_max);
    const int n_tiles = (d_out + wc - 1) / wc;
    if (n_tiles > tiles) continue;
    const long long ctas = (long long)n_tiles * C;
    if (ctas > best_ctas) {
      best_ctas = ctas;
      best.ok = true;
      best.cluster = C;
      best.n_tiles = n_tiles;
      best.col_tile = wc;
      best.tpr = wc / cpt;
      best.list_cap = range_cap;
      best.smem = flayout(d_in, esz, range_cap, wc, cpt).total;
      best.smem_alloc = smem_probe;
      best.partial_floats = (size_t)n_tiles * C * wc;
    }
  }
  *plan = best;
  return cudaSuccess;
}

cudaError_t launch_fused(Elem w_elem, const FusedArgs& a, const StreamPlan& pl,
                         cudaStream_t stream) {
  if (!pl.ok || (pl.cluster != 4 && pl.cluster != 8) || pl.n_tiles > kFusedMaxTiles)
    return cudaErrorInvalidValue;
  void* fn = fused_fn(w_elem, pl.cluster);
  FParams p;
  p.x = a.x;
  p.Qt = a.Qt;
  p.W = a.W;
  p.x_rot = a.x_rot;
  p.idx = a.idx;
  p.val = a.val;
  p.y = a.y;
  p.partials = a.partials;
  p.sync = a.sync;
  p.d = a.d_in;
  p.d_out = a.d_out;
  p.K = a.K;
  p.col_tile = pl.col_tile;
  p.tpr = pl.tpr;
  p.range_cap = pl.list_cap;
  p.n_tiles = pl.n_tiles;
  p.dev_status = a.dev_status;
  p.rotate = a.Qt != nullptr;
  p.thresh = a.threshold;
  p.t_key = a.t_key;
  p.nnz = a.nnz;
  p.wait_ns = wait_limit_ns();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.n_tiles * pl.cluster + 1, 1, 1);
  cfg.blockDim = dim3(kT, 1, 1);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  // every CTA must be resident at once: the gather CTAs wait on the selector.
  // As a programmatic dependent the launch may begin before the previous
  // kernel on the stream ends (the kernel waits before reading its inputs).
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  void* args[] = {&p};
  return cudaLaunchKernelExC(&cfg, fn, args);
}

namespace {

template <int C>
void* lowrank_fn_c(Elem w) {
  return w == Elem::BF16 ? reinterpret_cast<void*>(&lowrank_kernel<__nv_bfloat16, C>)
                         : reinterpret_cast<void*>(&lowrank_kernel<float, C>);
}

void* lowrank_fn(Elem w, int C) { return C == 8 ? lowrank_fn_c<8>(w) : lowrank_fn_c<4>(w); }

}  // namespace

static cudaError_t plan_lowrank_uncached(Elem w_elem, int d_in, int d_out, int K, int r, StreamPlan* plan) {
  DevState* ds = nullptr;
  cudaError_t e = dev_state(&ds);
  if (e != cudaSuccess) return e;
  StreamPlan best;
  *plan = best;
  const int cpt = w_elem == Elem::BF16 ? 8 : 4;
  if (d_in < 1 || d_in > kLRMaxD || K < 0 || K > d_in || r < cpt || r > kLRMaxRank || r % cpt != 0)
    return cudaSuccess;
  // factor CTAs: about two batches of A_r row loads each over the dropped
  // entries, and at most kLRMaxLen indices of x each
  const int rows_per_batch = (kT / (r / cpt)) * kFusedU;
  const int dropped = d_in - K;
  int F = (dropped + 2 * rows_per_batch - 1) / (2 * rows_per_batch);
  F = std::max(F, (d_in + kLRMaxLen - 1) / kLRMaxLen);
  F = std::max(1, std::min(F, kLRMaxF));
  const int f_len = (d_in + F - 1) / F;
  if (f_len > kLRMaxLen) return cudaSuccess;
  const size_t f_smem = lr_factor_layout(f_len, cpt).total;
  long long best_ctas = -1;
  for (int C : {8, 4}) {
    void* fn = lowrank_fn(w_elem, C);
    const int list_cap = std::max((K + C - 1) / C, (r + C - 1) / C);
    const int wc_max = kT * cpt;
    const size_t smem_probe = std::max(lr_tile_layout(list_cap, wc_max, cpt).total, f_smem);
    if (smem_probe > (size_t)kFusedSmemCeiling) continue;
    e = configure(ds, 12 + 4 + (w_elem == Elem::BF16 ? 1 : 0) * 2 + (C == 8 ? 1 : 0), fn, kFusedSmemCeiling);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kT, smem_probe);
    if (e != cudaSuccess) return e;
    const int tiles = std::min((ds->sms * per_sm - F) / C, kFusedMaxTiles);  // every CTA resident
    if (tiles < 1) continue;
    int wc = (d_out + tiles - 1) / tiles;
    wc = std::max(wc, std::min(64, d_out));
    wc = (wc + cpt - 1) / cpt * cpt;
    wc = std::min(wc, wc_max);
    const int n_tiles = (d_out + wc - 1) / wc;
    if (n_tiles > tiles) continue;
    const long long ctas = (long long)n_tiles * C;
    if (ctas > best_ctas) {
      best_ctas = ctas;
      best.ok = true;
      best.cluster = C;
      best.n_tiles = n_tiles;
      best.col_tile = wc;
      best.tpr = wc / cpt;
      best.list_cap = list_cap;
      best.aux_ctas = F;
      best.aux_len = f_len;
      best.smem = std::max(lr_tile_layout(list_cap, wc, cpt).total, f_smem);
      best.smem_alloc = smem_probe;
      best.partial_floats = (size_t)n_tiles * C * wc;
    }
  }
  *plan = best;
  return cudaSuccess;
}

cudaError_t plan_gather(Elem w_elem, int d_out, int K, StreamPlan* plan) {
  return cached_plan(PlanKey{0, 0, static_cast<int>(w_elem), 0, d_out, K, 0}, plan,
                     [&](StreamPlan* p) { return plan_gather_uncached(w_elem, d_out, K, p); });
}

cudaError_t plan_fused(Elem w_elem, int d_in, int d_out, int K, StreamPlan* plan) {
  return cached_plan(PlanKey{0, 1, static_cast<int>(w_elem), d_in, d_out, K, 0}, plan,
                     [&](StreamPlan* p) { return plan_fused_uncached(w_elem, d_in, d_out, K, p); });
}

cudaError_t plan_lowrank(Elem w_elem, int d_in, int d_out, int K, int r, StreamPlan* plan) {
  return cached_plan(PlanKey{0, 2, static_cast<int>(w_elem), d_in, d_out, K, r}, plan,
                     [&](StreamPlan* p) { return plan_lowrank_uncached(w_elem, d_in, d_out, K, r, p); });
}

cudaError_t launch_lowrank(Elem w_elem, const LowrankArgs& a, const StreamPlan& pl, cudaStream_t stream) {
  if (!pl.ok || (pl.cluster != 4 && pl.cluster != 8) || pl.n_tiles > kFusedMaxTiles || pl.aux_ctas < 1 ||
      pl.aux_ctas > kLRMaxF)
    return cudaErrorInvalidValue;
  void* fn = lowrank_fn(w_elem, pl.cluster);
  LRParams p;
  p.x = a.x;
  p.idx = a.idx;
  p.val = a.val;
  p.W = a.W;
  p.A_r = a.A_r;
  p.B_r = a.B_r;
  p.y = a.y;
  p.u = a.u;
  p.partials = a.partials;
  p.sync = a.sync;
  p.d = a.d_in;
  p.d_out = a.d_out;
  p.K = a.K;
  p.r = a.r;
  p.col_tile = pl.col_tile;
  p.tpr = pl.tpr;
  p.list_cap = pl.list_cap;
  p.n_tiles = pl.n_tiles;
  p.f_ctas = pl.aux_ctas;
  p.f_len = pl.aux_len;
  p.dev_status = a.dev_status;
  p.wait_ns = wait_limit_ns();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.n_tiles * pl.cluster + p.f_ctas, 1, 1);
  cfg.blockDim = dim3(kT, 1, 1);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  // every CTA must be resident at once: the column-tile CTAs wait on the factor CTAs
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  void* args[] = {&p};
  return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace larosa
