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
// gather  y[c] = sum_{p < K} coef(p) * W[row(p)][c], W row-major
//         [d_in x d_out]: the sparse linear over the kept rows of the
//         counter-rotated weight (abstract: activation sparsity reduces memory
//         transfers).  One thread-block cluster per column tile; the cluster's
//         CTAs take equal consecutive parts of the kept list and add their
//         partial sums through distributed shared memory in rank order, so
//         nothing leaves the cluster but y.  The tile width is chosen so the
//         clusters that fit on the GPU at once cover d_out.
//           kGather  row(p) = idx[p], coef(p) = val[p]
//           kSelect  each cluster first selects the K largest |x_rot| itself
//                    (exact, ties to the lower index; no grid-wide handoff)
//                    and starts streaming the rows it is sure of before the
//                    last places are decided.
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

// ================================================================ gather

constexpr int kModeGather = 1;
constexpr int kModeSelect = 2;
constexpr int kC = 8;  // CTAs per cluster (one column tile)
constexpr int kGatherSmemCeiling = 227 * 1024;
// Boundary-bin candidates ranked directly; a fuller bin takes radix passes.
constexpr int kRankCap = kT;

struct GParams {
  const void* W;         // [d_in x d_out] row-major
  int d_out;
  int d_in;              // row bound; also the length of x_rot
  int K;                 // kept entries
  const void* coef;      // gather: val[K]; select: x_rot[d_in]
  const int32_t* rows;   // gather: idx[K]
  float* y;
  int col_tile;
  int tpr;
  int list_cap;          // list entries a CTA holds: ceil(K / cluster)
  int32_t* idx_out;      // select: kept indices/values (optional)
  float* val_out;
  int* dev_status;
};

// Shared memory of one CTA, laid out from sizes known at launch.
struct GLayout {
  size_t sel, merged, xchg, keys, kflag, cand, call, cflag, rows, vals, part, red, total;
};

__host__ __device__ inline size_t al16(size_t v) { return (v + 15) & ~size_t(15); }

// list_cap: list entries a CTA holds (kept positions of its part, or kept
// entries of its index range); key_cap: rotated entries a CTA owns (select).
__host__ __device__ inline GLayout glayout(int mode, int key_cap, int list_cap, int col_tile,
                                           int cpt) {
  GLayout L;
  size_t o = 0;
  const bool sel = mode == kModeSelect;
  L.sel = o;      o = al16(o + (sel ? sizeof(SelectScratch) : 64));
  L.merged = o;   o = al16(o + (sel ? kSelBins * 4 : 0));
  L.xchg = o;     o = al16(o + (sel ? 4 * 32 * 4 : 0));
  L.keys = o;     o = al16(o + (sel ? (size_t)key_cap * 4 : 0));
  L.kflag = o;    o = al16(o + (sel ? (size_t)key_cap : 0));
  L.cand = o;     o = al16(o + (sel ? (size_t)kRankCap * 8 : 0));
  L.call = o;     o = al16(o + (sel ? (size_t)kRankCap * 8 : 0));
  L.cflag = o;    o = al16(o + (sel ? (size_t)kRankCap : 0));
  L.rows = o;     o = al16(o + (size_t)list_cap * 4);
  L.vals = o;     o = al16(o + (size_t)list_cap * 4);
  L.part = o;     o = al16(o + (size_t)col_tile * 4);
  L.red = o;      o = al16(o + (size_t)kT * cpt * 4);
  L.total = o;
  return L;
}

// Split cluster barrier: arrive publishes this thread's earlier writes
// (shared and distributed shared memory) to every CTA of the cluster; wait
// returns once all threads of the cluster have arrived.
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The bin holding the krem-th largest counted key, scanning counts[nb] from
// the top: writes bin, keys above it, keys in it to pick[0], pick[1],
// pick[3].  Ends with a barrier.
template <int NT>
__device__ __forceinline__ void boundary_from_top(const uint32_t* counts, int nb, uint32_t krem,
                                                  SelectScratch* s) {
  const int tid = threadIdx.x;
  // thread t owns ranks [t*per, t*per+per) counted from the top
  constexpr int kPer = (kSelBins + NT - 1) / NT;
  const int per = (nb + NT - 1) / NT;
  uint32_t cnt[kPer];
  uint32_t own = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int k = tid * per + j;
    cnt[j] = (j < per && k < nb) ? counts[nb - 1 - k] : 0u;
    own += cnt[j];
  }
  uint32_t before = block_scan_excl_1s<NT>(own, s->warp_sums, nullptr);
  if (before < krem && krem <= before + own) {
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      if (j < per && before < krem && krem <= before + cnt[j]) {
        s->pick[0] = static_cast<uint32_t>(nb - 1 - (tid * per + j));
        s->pick[1] = before;
        s->pick[3] = cnt[j];
      }
      before += cnt[j];
    }
  }
  __syncthreads();
}

// One radix pass of a selection spread over a cluster: histogram this CTA's
// keys that match `prefix` under `mask` on digit (key >> shift) & (nb-1),
// add the cluster's histograms (rank r adds bins [r*nb/kC, (r+1)*nb/kC) and
// writes the sums into every CTA's `merged`), then find the boundary bin as
// boundary_from_top does.  `hist` (both copies) must be zero on entry and is
// zero again on return.
template <int NT>
__device__ __forceinline__ void cluster_radix_pass(cg::cluster_group& cl, int rank,
                                                   const uint32_t* keys, int n_mine,
                                                   uint32_t prefix, uint32_t mask, int shift,
                                                   int nb, uint32_t krem, SelectScratch* s,
                                                   uint32_t* merged) {
  const int tid = threadIdx.x;
  uint32_t* h = s->hist + (tid & 1) * kSelBins;
  for (int i = tid; i < n_mine; i += NT) {
    const uint32_t k = keys[i] & kKeyMask;
    if ((k & mask) == prefix) atomicAdd(&h[(k >> shift) & static_cast<uint32_t>(nb - 1)], 1u);
  }
  __syncthreads();
  for (int b = tid; b < nb; b += NT) {
    s->hist[b] += s->hist[kSelBins + b];
    s->hist[kSelBins + b] = 0u;
  }
  cl.sync();  // every CTA's histogram is final
  const int b0 = nb * rank / kC, b1 = nb * (rank + 1) / kC;
  for (int b = b0 + tid; b < b1; b += NT) {
    uint32_t v[kC];
#pragma unroll
    for (int q = 0; q < kC; ++q) v[q] = cl.map_shared_rank(s->hist, q)[b];  // all in flight
    uint32_t sum = 0;
#pragma unroll
    for (int q = 0; q < kC; ++q) sum += v[q];
#pragma unroll
    for (int q = 0; q < kC; ++q) cl.map_shared_rank(merged, q)[b] = sum;
  }
  cl.sync();  // merged everywhere; no CTA still reads another's `hist`
  for (int b = tid; b < nb; b += NT) s->hist[b] = 0u;
  boundary_from_top<NT>(merged, nb, krem, s);
}

// Rank of a boundary-bin key: larger |x| first, then the lower index.
__device__ __forceinline__ unsigned long long cand_order(uint32_t key, int idx) {
  return (static_cast<unsigned long long>(key & kKeyMask) << 32) |
         static_cast<uint32_t>(~static_cast<uint32_t>(idx));
}

// One cluster per column tile; the cluster's CTAs split the kept list in
// rank order, and their partial sums meet in distributed shared memory.
//
// Select mode.  Rank r owns the rotated entries [d*r/C, d*(r+1)/C).  Every
// CTA histograms all d keys on bits 30..20 (sign cleared) and finds the bin
// B holding the K-th largest: keys above B are kept for certain, keys in B
// are candidates for the remaining krem places.  Each CTA then streams its
// certain rows while the cluster trades candidate lists (split barrier),
// ranks the candidates exactly, and streams its kept candidates last.  The
// order of the sum over rows is a function of the data only, so results
// repeat bit for bit.
template <typename Tw, int MODE>
__global__ void __launch_bounds__(kT, 2) gather_kernel(const GParams p) {
  constexpr int CPT = 16 / sizeof(Tw);  // columns per thread per row
  extern __shared__ __align__(16) unsigned char smem_raw[];
  cg::cluster_group cl = cg::this_cluster();
  constexpr int C = kC;
  const int rank = static_cast<int>(cl.block_rank());
  const int key_cap = (p.d_in + C - 1) / C;
  const GLayout L = glayout(MODE, key_cap, p.list_cap, p.col_tile, CPT);
  SelectScratch* sel = reinterpret_cast<SelectScratch*>(smem_raw + L.sel);
  int32_t* lrows = reinterpret_cast<int32_t*>(smem_raw + L.rows);
  float* lvals = reinterpret_cast<float*>(smem_raw + L.vals);
  float* part = reinterpret_cast<float*>(smem_raw + L.part);
  float* red = reinterpret_cast<float*>(smem_raw + L.red);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.y;
  const int c0 = tile * p.col_tile;
  const int wc = min(p.col_tile, p.d_out - c0);
  const int K = p.K;

  // ---- streaming: thread (g, col) reads 16 bytes of list rows lo+g,
  // lo+g+ng, ... < hi, with kU loads in flight, into acc
  const int tpr = p.tpr;
  const int ng = kT / tpr;
  const int g = tid / tpr;
  const int col = (tid - g * tpr) * CPT;
  const bool active = g < ng && col < wc;
  float acc[CPT];
#pragma unroll
  for (int v = 0; v < CPT; ++v) acc[v] = 0.f;
  const unsigned char* wbase = static_cast<const unsigned char*>(p.W) + ((size_t)c0 + col) * sizeof(Tw);
  const size_t pitch = (size_t)p.d_out * sizeof(Tw);
  auto stream_rows = [&](int lo, int hi) {
    if (!active) return;
    for (int r0 = lo + g; r0 < hi; r0 += ng * kU) {
      uint4 u[kU];
#pragma unroll
      for (int k = 0; k < kU; ++k) {
        const int r = r0 + k * ng;
        u[k] = r < hi ? ld_stream(wbase + (size_t)lrows[r] * pitch) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int k = 0; k < kU; ++k) {
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
  };

  if constexpr (MODE == kModeSelect) {
    for (int b = tid; b < 2 * kSelBins; b += kT) sel->hist[b] = 0u;
  }
  pdl_wait();
  pdl_launch_dependents();

  if constexpr (MODE == kModeGather) {
    // rank r takes the kept positions [K*r/C, K*(r+1)/C)
    const int p0 = (int)((long long)K * rank / C);
    const int p1 = (int)((long long)K * (rank + 1) / C);
    const int len = p1 - p0;
    bool bad = false;
    for (int j = tid; j < len; j += kT) {
      const int row = p.rows[p0 + j];
      const bool ok = static_cast<unsigned>(row) < static_cast<unsigned>(p.d_in);
      bad |= !ok;
      lrows[j] = ok ? row : 0;
      lvals[j] = ok ? static_cast<const float*>(p.coef)[p0 + j] : 0.f;
    }
    if (__syncthreads_or(bad) && tid == 0) report(p.dev_status, LAROSA_DEV_INDEX);
    stream_rows(0, len);
  }

  // select mode state kept for the index/value output at the end
  const int d = p.d_in;
  const int i_lo = (int)((long long)d * rank / C);
  const int n_mine = (int)((long long)d * (rank + 1) / C) - i_lo;
  const bool all = K >= d;
  uint32_t B = 0;            // boundary bin (bits 30..20)
  uint32_t kept_low = 0;     // kept entries owned by lower ranks
  if constexpr (MODE == kModeSelect) {
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + L.keys);
    uint8_t* kflag = reinterpret_cast<uint8_t*>(smem_raw + L.kflag);  // kept candidate
    uint32_t* merged = reinterpret_cast<uint32_t*>(smem_raw + L.merged);
    // xchg[q]: certain rows of rank q; [32+q]: its candidates; [64+q] and
    // [96+q]: above / at the threshold (radix fallback)
    uint32_t* xchg = reinterpret_cast<uint32_t*>(smem_raw + L.xchg);
    unsigned long long* cand = reinterpret_cast<unsigned long long*>(smem_raw + L.cand);
    unsigned long long* call = reinterpret_cast<unsigned long long*>(smem_raw + L.call);
    uint8_t* cflag = reinterpret_cast<uint8_t*>(smem_raw + L.cflag);

    // ---- all d keys -> histogram on bits 30..20; own keys -> `keys`
    {
      uint32_t* h = sel->hist + (lane & 1) * kSelBins;
      const uint4* src = static_cast<const uint4*>(p.coef);  // d is a multiple of 8
      bool nonfinite = false;
      for (int v = tid; v < d / 4; v += kT) {
        const uint4 u4 = __ldcg(src + v);
        const uint32_t u[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t k = u[e] & kKeyMask;
          nonfinite |= k >= 0x7f800000u;
          atomicAdd(&h[k >> 20], 1u);
          const int j = 4 * v + e - i_lo;
          if (j >= 0 && j < n_mine) {
            keys[j] = u[e];
            kflag[j] = 0;
          }
        }
      }
      if (__syncthreads_or(nonfinite) && tid == 0 && tile == 0 && rank == 0)
        report(p.dev_status, LAROSA_DEV_NONFINITE);
      for (int b = tid; b < kSelBins; b += kT) {
        merged[b] = sel->hist[b] + sel->hist[kSelBins + b];
        sel->hist[b] = 0u;
        sel->hist[kSelBins + b] = 0u;
      }
      __syncthreads();
    }
    uint32_t krem = 0;  // candidates to keep
    uint32_t nB = 0;    // keys in the boundary bin, cluster-wide
    if (K > 0 && !all) {
      boundary_from_top<kT>(merged, kSelBins, static_cast<uint32_t>(K), sel);
      B = sel->pick[0];
      krem = static_cast<uint32_t>(K) - sel->pick[1];
      nB = sel->pick[3];
    }
    const bool ranked = nB <= static_cast<uint32_t>(kRankCap);  // same in every CTA

    // ---- certain rows -> the list; candidates -> `cand` (ranked case)
    const int chunk = (n_mine + kT - 1) / kT;
    const int j0 = min(n_mine, tid * chunk), j1 = min(n_mine, j0 + chunk);
    auto certain = [&](uint32_t k) { return K > 0 && (all || (k >> 20) > B); };
    auto in_bin = [&](uint32_t k) { return K > 0 && !all && (k >> 20) == B; };
    uint32_t n_def = 0, n_cand = 0;
    {
      uint32_t dc = 0, cc = 0;
      for (int j = j0; j < j1; ++j) {
        const uint32_t k = keys[j] & kKeyMask;
        dc += certain(k);
        cc += in_bin(k);
      }
      uint32_t tot = 0;
      const uint32_t packed = block_scan_excl_1s<kT>((cc << 16) | dc, sel->warp_sums, &tot);
      uint32_t dp = packed & 0xffffu, cp = packed >> 16;
      n_def = tot & 0xffffu;
      n_cand = tot >> 16;
      for (int j = j0; j < j1; ++j) {
        const uint32_t u = keys[j];
        const uint32_t k = u & kKeyMask;
        if (certain(k)) {
          lrows[dp] = i_lo + j;
          lvals[dp] = __uint_as_float(u);
          ++dp;
        } else if (ranked && in_bin(k)) {
          cand[cp++] = cand_order(k, i_lo + j);
        }
      }
      if (tid < C) {  // one remote store pair per destination rank
        cl.map_shared_rank(xchg, tid)[rank] = n_def;
        cl.map_shared_rank(xchg, tid)[32 + rank] = n_cand;
      }
      __syncthreads();  // the list is complete before it is streamed
    }
    cluster_arrive_release();
    stream_rows(0, (int)n_def);
    cluster_wait_acquire();  // every rank's counts and candidates are visible

    const bool want_positions = tile == 0 && p.idx_out != nullptr;
    int len = (int)n_def;
    for (int q = 0; q < rank; ++q) kept_low += xchg[q];
    if (ranked) {
      // ---- the cluster's candidates in index order (rank, then position)
      uint32_t run = 0, src_base = 0, lo_r = 0, hi_r = 0;
      int src = 0;
#pragma unroll
      for (int q = 0; q < C; ++q) {
        const uint32_t cq = xchg[32 + q];
        if (static_cast<uint32_t>(tid) >= run) {  // the last rank starting at or below tid
          src = q;
          src_base = run;
        }
        if (q == rank) {
          lo_r = run;
          hi_r = run + cq;
        }
        run += cq;
      }
      const int n_all = (int)run;
      if (tid < n_all) call[tid] = cl.map_shared_rank(cand, src)[tid - src_base];
      __syncthreads();
      // a warp per candidate: kept iff fewer than krem candidates outrank it
      const int c_lo = want_positions ? 0 : (int)lo_r;
      const int c_hi = (int)hi_r;
      for (int c = c_lo + warp; c < c_hi; c += kWarps) {
        const unsigned long long me = call[c];
        uint32_t above = 0;
        for (int i = lane; i < n_all; i += 32) above += call[i] > me;
        above = __reduce_add_sync(0xffffffffu, above);
        if (lane == 0) cflag[c] = above < krem;
      }
      __syncthreads();
      const bool f = tid >= c_lo && tid < c_hi && cflag[tid];
      const bool own = f && tid >= (int)lo_r;
      uint32_t tot = 0;
      const uint32_t packed = block_scan_excl_1s<kT>(((uint32_t)(f && !own) << 16) | own,
                                                     sel->warp_sums, &tot);
      if (own) {
        const int idx = (int)~static_cast<uint32_t>(call[tid]);
        const int pos = (int)n_def + (int)(packed & 0xffffu);
        lrows[pos] = idx;
        lvals[pos] = __uint_as_float(keys[idx - i_lo]);
        kflag[idx - i_lo] = 1;
      }
      len += (int)(tot & 0xffffu);
      kept_low += tot >> 16;
    } else {
      // ---- too many keys share bin B: two more radix passes inside it,
      // with histograms added across the cluster, give the exact threshold
      // T; ties at T go to the lowest indices across the cluster
      uint32_t prefix = B << 20, mask = 0x7ffu << 20;
#pragma unroll 1
      for (int pass = 1; pass < 3; ++pass) {
        const int shift = pass == 1 ? 9 : 0;
        const int nb = pass == 1 ? 2048 : 512;
        cluster_radix_pass<kT>(cl, rank, keys, n_mine, prefix, mask, shift, nb, krem, sel, merged);
        prefix |= sel->pick[0] << shift;
        mask |= static_cast<uint32_t>(nb - 1) << shift;
        krem -= sel->pick[1];
        __syncthreads();
      }
      const uint32_t T = prefix;  // krem keys equal to T are kept
      uint32_t gt = 0, eq = 0;
      for (int j = j0; j < j1; ++j) {
        const uint32_t k = keys[j] & kKeyMask;
        gt += (k >> 20) == B && k > T;
        eq += k == T;
      }
      uint32_t tot = 0;
      const uint32_t packed = block_scan_excl_1s<kT>((eq << 16) | gt, sel->warp_sums, &tot);
      if (tid < C) {
        cl.map_shared_rank(xchg, tid)[64 + rank] = tot & 0xffffu;
        cl.map_shared_rank(xchg, tid)[96 + rank] = tot >> 16;
      }
      cl.sync();  // every CTA's counts are in every CTA
      uint32_t ties_before = 0;
      for (int q = 0; q < rank; ++q) {
        const uint32_t tq = xchg[96 + q];
        kept_low += xchg[64 + q] + min(tq, krem > ties_before ? krem - ties_before : 0u);
        ties_before += tq;
      }
      const uint32_t ties_left = krem > ties_before ? krem - ties_before : 0u;
      uint32_t eqc = packed >> 16;
      uint32_t pos = n_def + (packed & 0xffffu) + min(eqc, ties_left);
      for (int j = j0; j < j1; ++j) {
        const uint32_t u = keys[j];
        const uint32_t k = u & kKeyMask;
        bool kept = false;
        if ((k >> 20) == B && k > T) {
          kept = true;
        } else if (k == T) {
          kept = eqc < ties_left;
          ++eqc;
        }
        if (kept) {
          lrows[pos] = i_lo + j;
          lvals[pos] = __uint_as_float(u);
          kflag[j] = 1;
          ++pos;
        }
      }
      len += (int)((tot & 0xffffu) + min(tot >> 16, ties_left));
    }
    __syncthreads();
    stream_rows((int)n_def, len);
  }

  // ---- row groups -> this CTA's partial, in shared memory
  if (active) {
#pragma unroll
    for (int v = 0; v < CPT; ++v) red[g * p.col_tile + col + v] = acc[v];
  }
  __syncthreads();
  for (int e = tid; e < wc; e += kT) {
    float sum = 0.f;
    for (int gg = 0; gg < ng; ++gg) sum += red[gg * p.col_tile + e];
    part[e] = sum;
  }
  // ---- the cluster's partials -> y: rank r adds its column slice in rank order
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
    p.y[c0 + e] = sum;
  }
  cl.sync();  // no CTA leaves while another may still read its partial

  // ---- the kept indices and values in ascending index order (one cluster)
  if constexpr (MODE == kModeSelect) {
    if (tile == 0 && p.idx_out != nullptr) {
      const uint32_t* keys = reinterpret_cast<const uint32_t*>(smem_raw + L.keys);
      const uint8_t* kflag = reinterpret_cast<const uint8_t*>(smem_raw + L.kflag);
      const int chunk = (n_mine + kT - 1) / kT;
      const int j0 = min(n_mine, tid * chunk), j1 = min(n_mine, j0 + chunk);
      auto kept = [&](int j) {
        return K > 0 && (all || ((keys[j] & kKeyMask) >> 20) > B || kflag[j] != 0);
      };
      uint32_t n = 0;
      for (int j = j0; j < j1; ++j) n += kept(j);
      uint32_t pos = kept_low + block_scan_excl_1s<kT>(n, sel->warp_sums, nullptr);
      for (int j = j0; j < j1; ++j) {
        if (kept(j)) {
          p.idx_out[pos] = i_lo + j;
          p.val_out[pos] = __uint_as_float(keys[j]);
          ++pos;
        }
      }
    }
  }
}

struct DevState {
  int sms = 0;
  bool configured[16] = {};
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

// ---------------------------------------------------------------- host API

cudaError_t launch_rowdot(Elem e, const void* A, const void* x, float* y, int M, int n_in,
                          int n_out, cudaStream_t stream) {
  DevState* ds = nullptr;
  cudaError_t err = dev_state(&ds);
  if (err != cudaSuccess) return err;
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

cudaError_t max_clusters(int dev, void* fn, size_t smem, int C, int* out) {
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
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kGatherSmemCeiling);
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

void* gather_fn(Elem w, int mode) {
  if (w == Elem::BF16)
    return mode == kGatherSelect ? reinterpret_cast<void*>(&gather_kernel<__nv_bfloat16, kModeSelect>)
                                 : reinterpret_cast<void*>(&gather_kernel<__nv_bfloat16, kModeGather>);
  return mode == kGatherSelect ? reinterpret_cast<void*>(&gather_kernel<float, kModeSelect>)
                               : reinterpret_cast<void*>(&gather_kernel<float, kModeGather>);
}

}  // namespace

cudaError_t plan_gather(int mode, Elem w_elem, int d_in, int d_out, int K, StreamPlan* plan) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const int cpt = w_elem == Elem::BF16 ? 8 : 4;
  const int kmode = mode == kGatherSelect ? kModeSelect : kModeGather;
  void* fn = gather_fn(w_elem, mode);
  StreamPlan best;
  long long best_ctas = -1;
  for (int C = kC; C == kC; C = 0) {
    const int key_cap = (d_in + C - 1) / C;
    // list mode: the rank's share of the kept list; select mode: the kept
    // entries of the rank's index range
    const int list_cap = std::max(1, kmode == kModeSelect ? key_cap : (K + C - 1) / C);
    // column tile: fill the co-resident clusters, at least 64 columns wide
    // (128 bytes of bf16) and at most one 16-byte vector per thread
    const int wc_max = kT * cpt;
    const size_t smem_probe = glayout(kmode, key_cap, list_cap, wc_max, cpt).total;
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
      best.smem = glayout(kmode, key_cap, list_cap, wc, cpt).total;
      best.smem_alloc = smem_probe;
    }
  }
  *plan = best;
  return cudaSuccess;
}

cudaError_t launch_gather(int mode, Elem w_elem, const GatherArgs& a, const StreamPlan& pl,
                          cudaStream_t stream) {
  if (!pl.ok) return cudaErrorInvalidValue;
  void* fn = gather_fn(w_elem, mode);
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
  p.idx_out = a.idx_out;
  p.val_out = a.val_out;
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

}  // namespace larosa
