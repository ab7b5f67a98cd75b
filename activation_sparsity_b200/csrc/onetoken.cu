// Decode-path kernels (sm_100a): the GEMVs of one token, and of up to 16
// tokens for the row-dot form.  All are bound by HBM bandwidth (about one
// flop per byte), so the design goal is bytes in flight and one read of every
// weight byte:
//
//   * one CTA of 512 threads per SM; every lane keeps eight independent
//     16-byte loads in flight (ld.global.cs: streamed, evict-first), which a
//     streaming probe on B200 measured at about 7 TB/s, the copy peak; TMA
//     bulk copies into a shared ring reached only about 4.2 TB/s with one CTA
//     per SM and were left out;
//   * a fixed reduction order everywhere, so results are bit-reproducible.
//
// rowdot  y[m][j] = sum_i x[m][i] * A[j][i], A row-major [n_out x n_in].
//         The rotation x_rot = x . Q reads Q through A = Q^T ("La RoSA"
//         summary, 方法详解 / 技术框架: each layer's input activation is
//         multiplied by that layer's orthogonal matrix); the dense baseline
//         reads W in torch.nn.Linear layout.  Each warp owns whole output rows:
//         no cross-CTA reduction at all.
//
// gather  y[c] = sum_{p < n} coef(p) * W[row(p)][c], W row-major
//         [d_in x d_out]: the sparse linear over the kept rows of the
//         counter-rotated weight (abstract: activation sparsity reduces memory
//         transfers).  Work = (column tile, list position) pairs, tile-major,
//         cut into equal contiguous ranges, one per CTA (at most two tiles per
//         range).  Partials of a tile are added in CTA order by the
//         last-arriving contributor (atomic ticket, no waiting).
//           kGather  row(p) = idx[p], coef(p) = val[p]
//           kSelect  every CTA first selects the K largest |x_rot| itself
//                    (exact, ties to the lower index; no grid-wide handoff),
//                    then gathers them.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

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
__global__ void __launch_bounds__(kT, 1) rowdot_kernel(const RParams p) {
  extern __shared__ __align__(16) unsigned char xs_raw[];
  const T* xs = reinterpret_cast<const T*>(xs_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_wait();
  pdl_launch_dependents();
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
}

// ================================================================ gather

constexpr int kModeGather = 1;
constexpr int kModeSelect = 2;
constexpr int kMaxUnits = 4096;   // list positions a CTA holds
constexpr int kCandCap = 2048;
constexpr int kXrotMax = 32768;   // selection buffer (fp32 words)

struct GParams {
  const void* W;         // [d_in x d_out] row-major
  int d_out;
  int row_bound;         // d_in (also the length of x_rot)
  int n;                 // list length (K)
  const void* coef;      // gather: val; select: x_rot
  const int32_t* rows;   // gather: idx
  float* y;
  float* partials;
  unsigned* tickets;
  int col_tile;
  int n_tiles;
  int tpr;
  int max_slots;
  int32_t* idx_out;      // select: kept indices/values (optional)
  float* val_out;
  int* dev_status;
};

struct GSmem {
  SelectScratch sel;
  int flags[4];
  int32_t rows[kMaxUnits];
  float coefs[kMaxUnits];
  uint32_t cand[kCandCap];
  float red[kT * 8];     // row groups x column tile (<= 4096 floats of 8 per thread)
};

__device__ __forceinline__ void tile_contributors(long long U, int G, int n, int t, int* first,
                                                  int* last) {
  const long long a = ((long long)t * n + 1) * G - 1;
  const long long b = ((long long)(t + 1) * n) * G - 1;
  *first = (int)max(0LL, a / U);
  *last = (int)min((long long)G - 1, b / U);
}

template <typename Tw, int MODE>
__global__ void __launch_bounds__(kT, 1) gather_kernel(const GParams p) {
  constexpr int CPT = 16 / sizeof(Tw);  // columns per thread per row
  extern __shared__ __align__(16) unsigned char smem_raw[];
  GSmem& S = *reinterpret_cast<GSmem*>(smem_raw);
  uint32_t* bits = reinterpret_cast<uint32_t*>(smem_raw + sizeof(GSmem));  // select buffer

  const int tid = threadIdx.x;
  const int G = gridDim.x, cta = blockIdx.x;
  pdl_wait();
  pdl_launch_dependents();

  const int n = p.n;
  if (n == 0) {  // nothing kept: y = 0
    const int per = (p.d_out + G - 1) / G;
    for (int i = cta * per + tid; i < min(p.d_out, (cta + 1) * per); i += kT) p.y[i] = 0.f;
    return;
  }

  // ---- this CTA's (at most two) segments: tile t, positions [a, b), slot offset
  const long long U = (long long)p.n_tiles * n;
  const long long u0 = U * cta / G;
  const long long u1 = U * (cta + 1) / G;
  const int t0 = (int)(u0 / n);
  const int s0a = (int)(u0 - (long long)t0 * n);
  const int s0b = (int)min((long long)n, u1 - (long long)t0 * n);
  const bool two = u1 > (long long)(t0 + 1) * n;
  const int t1 = t0 + 1;
  const int s1b = two ? (int)(u1 - (long long)t1 * n) : 0;
  const int len0 = s0b - s0a;
  const int len1 = s1b;  // segment 1 starts at position 0 of tile t1

  if constexpr (MODE == kModeGather) {
    bool bad = false;
    for (int j = tid; j < len0 + len1; j += kT) {
      const int pos = j < len0 ? s0a + j : j - len0;
      const int row = p.rows[pos];
      const bool ok = static_cast<unsigned>(row) < static_cast<unsigned>(p.row_bound);
      bad |= !ok;
      S.rows[j] = ok ? row : 0;
      S.coefs[j] = ok ? static_cast<const float*>(p.coef)[pos] : 0.f;
    }
    if (__syncthreads_or(bad) && tid == 0) report(p.dev_status, LAROSA_DEV_INDEX);
  } else {
    const int d = p.row_bound;
    {
      const uint4* src = static_cast<const uint4*>(p.coef);
      const int nv = d >> 2;
      bool nonfinite = false;
#pragma unroll 4
      for (int i = tid; i < nv; i += kT) {
        const uint4 u = __ldcg(src + i);
        reinterpret_cast<uint4*>(bits)[i] = u;
        nonfinite |= ((u.x & kKeyMask) >= 0x7f800000u) | ((u.y & kKeyMask) >= 0x7f800000u) |
                     ((u.z & kKeyMask) >= 0x7f800000u) | ((u.w & kKeyMask) >= 0x7f800000u);
      }
      if (__syncthreads_or(nonfinite) && tid == 0 && cta == 0)
        report(p.dev_status, LAROSA_DEV_NONFINITE);
    }
    const int K = n;
    const bool all = K >= d;
    uint32_t T = 0, krem = 0;
    if (!all) select_threshold<kT>(bits, d, K, &S.sel, S.cand, kCandCap, &T, &krem);
    const int chunk = (d + kT - 1) / kT;
    const int i0 = min(d, tid * chunk);
    const int i1 = min(d, i0 + chunk);
    uint32_t gt = 0, eq = 0;
    if (!all) kept_chunk_base<kT>(bits, i0, i1, T, &S.sel, &gt, &eq);
    const bool write_out = p.idx_out != nullptr;
    for (int i = i0; i < i1; ++i) {
      const uint32_t u = bits[i];
      const uint32_t k = u & kKeyMask;
      int pos;
      if (all) {
        pos = i;
      } else if (k > T) {
        pos = (int)(gt + min(eq, krem));
        ++gt;
      } else if (k == T && eq < krem) {
        pos = (int)(gt + eq);
        ++eq;
      } else {
        if (k == T) ++eq;
        continue;
      }
      const float val = __uint_as_float(u);
      if (pos >= s0a && pos < s0b) {
        S.rows[pos - s0a] = i;
        S.coefs[pos - s0a] = val;
        if (t0 == 0 && write_out) {
          p.idx_out[pos] = i;
          p.val_out[pos] = val;
        }
      }
      if (pos < s1b) {
        S.rows[len0 + pos] = i;
        S.coefs[len0 + pos] = val;
      }
    }
    __syncthreads();
  }

  // ---- stream the rows: thread (g, col) reads 16 bytes of rows g, g+ng, ...
  const int tpr = p.tpr;
  const int g = tid / tpr;
  const int ng = kT / tpr;
  const int col = (tid % tpr) * CPT;
  float acc[2][CPT];
#pragma unroll
  for (int s = 0; s < 2; ++s)
#pragma unroll
    for (int v = 0; v < CPT; ++v) acc[s][v] = 0.f;

#pragma unroll
  for (int s = 0; s < 2; ++s) {
    const int t = s == 0 ? t0 : t1;
    const int len = s == 0 ? len0 : len1;
    const int off = s == 0 ? 0 : len0;
    if (len == 0) continue;
    const int c0 = t * p.col_tile;
    const int wc = min(p.col_tile, p.d_out - c0);
    if (col >= wc) continue;
    const unsigned char* wbase = static_cast<const unsigned char*>(p.W) + ((size_t)c0 + col) * sizeof(Tw);
    const size_t pitch = (size_t)p.d_out * sizeof(Tw);
    for (int r0 = g; r0 < len; r0 += ng * kU) {
      uint4 u[kU];
#pragma unroll
      for (int k = 0; k < kU; ++k) {
        const int r = r0 + k * ng;
        u[k] = r < len ? ld_stream(wbase + (size_t)S.rows[off + r] * pitch) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int k = 0; k < kU; ++k) {
        const int r = r0 + k * ng;
        if (r < len) {
          const float cf = S.coefs[off + r];
          if constexpr (CPT == 8) {
            float w[8];
            Vec8<__nv_bfloat16>::cvt(&u[k], w);
#pragma unroll
            for (int v = 0; v < 8; ++v) acc[s][v] = fmaf(cf, w[v], acc[s][v]);
          } else {
            acc[s][0] = fmaf(cf, __uint_as_float(u[k].x), acc[s][0]);
            acc[s][1] = fmaf(cf, __uint_as_float(u[k].y), acc[s][1]);
            acc[s][2] = fmaf(cf, __uint_as_float(u[k].z), acc[s][2]);
            acc[s][3] = fmaf(cf, __uint_as_float(u[k].w), acc[s][3]);
          }
        }
      }
    }
  }

  // ---- per segment: row groups -> CTA partial -> tile result
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    const int t = s == 0 ? t0 : t1;
    const int len = s == 0 ? len0 : len1;
    if (len == 0) continue;  // uniform across the CTA
    const int c0 = t * p.col_tile;
    const int wc = min(p.col_tile, p.d_out - c0);
    __syncthreads();  // S.red free
    if (col < wc) {
#pragma unroll
      for (int v = 0; v < CPT; ++v) S.red[g * p.col_tile + col + v] = acc[s][v];
    }
    __syncthreads();
    int first = 0, last = 0;
    tile_contributors(U, G, n, t, &first, &last);
    const int n_contrib = last - first + 1;
    float* mine = p.partials + ((size_t)t * p.max_slots + (cta - first)) * p.col_tile;
    for (int e = tid; e < wc; e += kT) {
      float sum = 0.f;
      for (int gg = 0; gg < ng; ++gg) sum += S.red[gg * p.col_tile + e];
      if (n_contrib == 1)
        p.y[c0 + e] = sum;
      else
        mine[e] = sum;
    }
    if (n_contrib > 1) {
      __threadfence();
      __syncthreads();
      if (tid == 0) S.flags[0] = static_cast<int>(atomicAdd(&p.tickets[t], 1u));
      __syncthreads();
      if (S.flags[0] == n_contrib - 1) {
        __threadfence();
        const float* all = p.partials + (size_t)t * p.max_slots * p.col_tile;
        for (int e4 = tid * 4; e4 < wc; e4 += kT * 4) {
          float4 acc4 = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int q = 0; q < n_contrib; ++q) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(all + (size_t)q * p.col_tile + e4));
            acc4.x += v.x; acc4.y += v.y; acc4.z += v.z; acc4.w += v.w;
          }
          *reinterpret_cast<float4*>(p.y + c0 + e4) = acc4;
        }
        if (tid == 0) atomicExch(&p.tickets[t], 0u);
      }
    }
  }
}

constexpr size_t kGatherSmem = sizeof(GSmem);
constexpr size_t kSelectSmem = sizeof(GSmem) + (size_t)kXrotMax * 4;

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
  const int grid = std::max(1, std::min(ds->sms, n_out));
  return launch(fn, grid, in_smem ? xbytes : 0, &p, stream);
}

cudaError_t plan_gather(Elem w_elem, int d_out, int n, StreamPlan* plan) {
  DevState* ds = nullptr;
  cudaError_t e = dev_state(&ds);
  if (e != cudaSuccess) return e;
  const int G = ds->sms;
  const int cpt = w_elem == Elem::BF16 ? 8 : 4;
  StreamPlan best, fallback;
  // the widest column tile whose last-contributor reduction stays small
  for (int tpr = kT; tpr >= 32; tpr /= 2) {
    const int wc = tpr * cpt;
    if (tpr > 32 && wc / 2 >= d_out) continue;  // mostly idle threads
    const int n_tiles = (d_out + wc - 1) / wc;
    if (n_tiles > G) continue;
    const long long U = (long long)n_tiles * n;
    const int grid = (int)std::max(1LL, std::min<long long>(G, U));
    if ((U + grid - 1) / grid > kMaxUnits) continue;
    int max_slots = 1;
    for (int t = 0; n > 0 && t < n_tiles; ++t) {
      const long long a = ((long long)t * n + 1) * grid - 1;
      const long long b = ((long long)(t + 1) * n) * grid - 1;
      const int first = (int)std::max(0LL, a / U);
      const int last = (int)std::min((long long)grid - 1, b / U);
      max_slots = std::max(max_slots, last - first + 1);
    }
    StreamPlan pl;
    pl.ok = true;
    pl.grid = grid;
    pl.col_tile = wc;
    pl.tpr = tpr;
    pl.n_tiles = n_tiles;
    pl.max_slots = max_slots;
    pl.partial_floats = (size_t)n_tiles * max_slots * wc;
    pl.ticket_words = n_tiles;
    fallback = pl;
    if ((size_t)max_slots * wc * 4 <= 64 * 1024) {
      best = pl;
      break;
    }
  }
  *plan = best.ok ? best : fallback;
  return cudaSuccess;
}

cudaError_t launch_gather(int mode, Elem w_elem, const GatherArgs& a, const StreamPlan& pl,
                          cudaStream_t stream) {
  if (!pl.ok) return cudaErrorInvalidValue;
  DevState* ds = nullptr;
  cudaError_t e = dev_state(&ds);
  if (e != cudaSuccess) return e;
  const bool sel = mode == kGatherSelect;
  void* fn;
  if (w_elem == Elem::BF16)
    fn = sel ? reinterpret_cast<void*>(&gather_kernel<__nv_bfloat16, kModeSelect>)
             : reinterpret_cast<void*>(&gather_kernel<__nv_bfloat16, kModeGather>);
  else
    fn = sel ? reinterpret_cast<void*>(&gather_kernel<float, kModeSelect>)
             : reinterpret_cast<void*>(&gather_kernel<float, kModeGather>);
  const size_t smem = sel ? kSelectSmem : kGatherSmem;
  e = configure(ds, 10 + (w_elem == Elem::BF16 ? 2 : 0) + (sel ? 1 : 0), fn, smem);
  if (e != cudaSuccess) return e;
  GParams p;
  p.W = a.W;
  p.d_out = a.d_out;
  p.row_bound = a.row_bound;
  p.n = a.n;
  p.coef = a.coef;
  p.rows = a.rows;
  p.y = a.y;
  p.partials = a.partials;
  p.tickets = a.tickets;
  p.col_tile = pl.col_tile;
  p.n_tiles = pl.n_tiles;
  p.tpr = pl.tpr;
  p.max_slots = pl.max_slots;
  p.idx_out = a.idx_out;
  p.val_out = a.val_out;
  p.dev_status = a.dev_status;
  return launch(fn, pl.grid, smem, &p, stream);
}

}  // namespace larosa
