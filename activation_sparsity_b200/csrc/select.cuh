// Exact Top-K-by-magnitude selection for one vector held in shared memory,
// cooperative over a whole CTA of NT threads (NT a multiple of 32).
//
// LaRoSA keeps the K entries of largest magnitude of every rotated
// activation vector ("La RoSA" summary, 方法详解 / 技术框架; abstract: Top-K
// gives the same sparsity on every token).  Here ties go to the lower index
// and +0 / -0 are equal.
//
// An fp32 magnitude orders exactly like its bit pattern with the sign bit
// cleared, read as an unsigned integer (a 31-bit "key").  select_threshold()
// finds the K-th largest key T and how many keys equal to T are kept (the
// lowest-indexed ones) with an MSB-first radix select:
//
//   pass 1   histogram of bits 30..20 over all d keys (shared-memory atomics
//            on two lane-interleaved copies of the histogram, which halves
//            same-address contention within a warp),
//   compact  the keys of the boundary bin into a candidate list (when it is
//            small; otherwise passes 2-3 scan all keys with a prefix test),
//   pass 2,3 histograms of bits 19..9 and 8..0 over the candidates.
//
// Every pass finds its boundary bin with one block-wide scan of the bin
// counts taken from the top.  kept_chunk_base() then gives each kept entry
// its rank in ascending index order from one packed (#greater, #equal) scan
// over contiguous per-thread chunks.
//
// All buffers are shared memory passed by pointer; the functions are inlined
// into their kernels so the compiler keeps shared-memory addressing.
#pragma once

#include "common.cuh"

namespace larosa {

constexpr int kSelBins = 2048;
constexpr uint32_t kKeyMask = 0x7fffffffu;

// Shared-memory scratch of one selection.
struct SelectScratch {
  uint32_t hist[2 * kSelBins];  // two interleaved copies during counting
  uint32_t warp_sums[32];
  uint32_t pick[8];  // [0] bin [1] keys above [2] candidates [3] bin count [4] ties kept [5] T
};

// Inclusive prefix sum of v over the NT threads of the block.  Contains
// __syncthreads(); every thread of the block must call it.
template <int NT>
__device__ __forceinline__ uint32_t block_scan_incl(uint32_t v, uint32_t* warp_sums) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_sums[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < NW ? warp_sums[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    if (lane < NW) warp_sums[lane] = w;
  }
  __syncthreads();
  if (warp > 0) v += warp_sums[warp - 1];
  __syncthreads();
  return v;
}

// Finds, among nb bins (sum of both histogram copies), the bin holding the
// krem-th largest counted key, counting from the top; writes it to pick[0],
// the count in higher bins to pick[1] and the bin's count to pick[3].
template <int NT>
__device__ __forceinline__ void find_boundary_bin(SelectScratch* s, int nb, uint32_t krem) {
  constexpr int kMaxPer = (kSelBins + NT - 1) / NT;
  const int per = (nb + NT - 1) / NT;
  const int t = threadIdx.x;
  uint32_t own = 0;
  uint32_t cnt[kMaxPer];
#pragma unroll
  for (int j = 0; j < kMaxPer; ++j) {
    const int k = t + j * NT;  // k-th bin from the top (strided: conflict-free)
    const int b = nb - 1 - k;
    cnt[j] = (j < per && k < nb) ? s->hist[b] + s->hist[kSelBins + b] : 0u;
  }
  // the scan needs each thread's bins to be contiguous from the top, so
  // rebuild the per-thread view: thread t owns ranks [t*per, t*per + per)
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kMaxPer; ++j) {
    const int k = t + j * NT;
    if (j < per && k < nb) s->hist[k] = cnt[j];  // copy 0 now holds counts by rank
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kMaxPer; ++j) {
    const int k = t * per + j;
    cnt[j] = (j < per && k < nb) ? s->hist[k] : 0u;
    own += cnt[j];
  }
  const uint32_t incl = block_scan_incl<NT>(own, s->warp_sums);
  uint32_t before = incl - own;
  if (before < krem && krem <= incl) {
#pragma unroll
    for (int j = 0; j < kMaxPer; ++j) {
      if (j < per && before < krem && krem <= before + cnt[j]) {
        s->pick[0] = static_cast<uint32_t>(nb - 1 - (t * per + j));
        s->pick[1] = before;
        s->pick[3] = cnt[j];
      }
      before += cnt[j];
    }
  }
  __syncthreads();
}

template <int NT>
__device__ __forceinline__ void clear_hist(SelectScratch* s, int nb) {
  for (int b = threadIdx.x; b < nb; b += NT) {
    s->hist[b] = 0u;
    s->hist[kSelBins + b] = 0u;
  }
}

// K-th largest key T of the d raw fp32 words in `bits` and the number
// krem >= 1 of keys equal to T that belong to the top K.  `cand` holds up to
// cand_cap candidate keys.  Requires 1 <= K < d.  All NT threads call it.
template <int NT>
__device__ __forceinline__ void select_threshold(const uint32_t* bits, int d, int K,
                                                 SelectScratch* s, uint32_t* cand, int cand_cap,
                                                 uint32_t* T_out, uint32_t* krem_out) {
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  uint32_t* h = s->hist + (lane & 1) * kSelBins;
  uint32_t krem = static_cast<uint32_t>(K);

  // ---- pass 1: bits 30..20 over all keys
  clear_hist<NT>(s, kSelBins);
  if (tid == 0) s->pick[2] = 0;
  __syncthreads();
#pragma unroll 4
  for (int i = tid; i < d; i += NT) atomicAdd(&h[(bits[i] & kKeyMask) >> 20], 1u);
  __syncthreads();
  find_boundary_bin<NT>(s, kSelBins, krem);
  const uint32_t b1 = s->pick[0];
  const uint32_t n1 = s->pick[3];
  krem -= s->pick[1];
  uint32_t prefix = b1 << 20;
  uint32_t mask = 0x7ff00000u;

  // ---- candidates: the keys of the boundary bin
  const bool compact = n1 <= static_cast<uint32_t>(cand_cap);
  if (compact) {
    for (int i0 = 0; i0 < d; i0 += NT) {
      const int i = i0 + tid;
      const uint32_t k = i < d ? (bits[i] & kKeyMask) : 0u;
      const bool hit = i < d && (k & mask) == prefix;
      const uint32_t lanes = __ballot_sync(0xffffffffu, hit);
      uint32_t base = 0;
      if (lane == 0 && lanes) base = atomicAdd(&s->pick[2], __popc(lanes));
      base = __shfl_sync(0xffffffffu, base, 0);
      if (hit) cand[base + __popc(lanes & ((1u << lane) - 1u))] = k;
    }
  }
  const int nc = compact ? static_cast<int>(n1) : d;

  // ---- passes 2 and 3
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
    const int shift = pass == 0 ? 9 : 0;
    const int nb = pass == 0 ? 2048 : 512;
    clear_hist<NT>(s, nb);
    __syncthreads();
    for (int i = tid; i < nc; i += NT) {
      const uint32_t k = compact ? cand[i] : (bits[i] & kKeyMask);
      if ((k & mask) == prefix) atomicAdd(&h[(k >> shift) & static_cast<uint32_t>(nb - 1)], 1u);
    }
    __syncthreads();
    find_boundary_bin<NT>(s, nb, krem);
    prefix |= s->pick[0] << shift;
    mask |= static_cast<uint32_t>(nb - 1) << shift;
    krem -= s->pick[1];
  }
  *T_out = prefix;
  *krem_out = krem;
}

// For the chunk [i0, i1) of this thread: the numbers of keys greater than T
// and equal to T before i0 (exclusive block scan).  All threads call it.
template <int NT>
__device__ __forceinline__ void kept_chunk_base(const uint32_t* bits, int i0, int i1, uint32_t T,
                                                SelectScratch* s, uint32_t* gt_before,
                                                uint32_t* eq_before) {
  uint32_t gt = 0, eq = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t k = bits[i] & kKeyMask;
    gt += k > T;
    eq += k == T;
  }
  const uint32_t packed = (eq << 16) | gt;  // d < 65536: no carry between halves
  const uint32_t excl = block_scan_incl<NT>(packed, s->warp_sums) - packed;
  *gt_before = excl & 0xffffu;
  *eq_before = excl >> 16;
}

// Exclusive prefix sum of v over the NT threads with a single barrier.  The
// caller must place a barrier between two uses of warp_sums.
template <int NT>
__device__ __forceinline__ uint32_t block_scan_excl_1s(uint32_t v, uint32_t* warp_sums,
                                                       uint32_t* total) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  uint32_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) warp_sums[warp] = inc;
  __syncthreads();
  uint32_t base = 0, all = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const uint32_t ws = warp_sums[w];
    base += w < warp ? ws : 0u;
    all += ws;
  }
  if (total != nullptr) *total = all;
  return base + inc - v;
}

// Same result as select_threshold, with fewer barriers: after the pass-1
// histogram the keys of the boundary bin (at most cand_cap of them) are ranked
// against each other directly -- larger key first, lower index first among
// equal keys -- instead of two more radix passes.  Falls back to
// select_threshold when the boundary bin holds more than cand_cap keys.
// cand_key / cand_idx: shared arrays of cand_cap entries.  Requires
// 1 <= K < d; s->hist must be zero on entry (both copies, all 2048 bins) and
// the first barrier after that must come before this call's counting, which
// the caller provides.
template <int NT>
__device__ __forceinline__ void select_threshold_fast(const uint32_t* bits, int d, int K,
                                                      SelectScratch* s, uint32_t* cand_key,
                                                      uint32_t* cand_idx, int cand_cap,
                                                      uint32_t* T_out, uint32_t* krem_out) {
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  constexpr int NW = NT / 32;
  uint32_t* h = s->hist + (lane & 1) * kSelBins;

  // ---- pass 1: bits 30..20 over all keys
#pragma unroll 4
  for (int i = tid; i < d; i += NT) atomicAdd(&h[(bits[i] & kKeyMask) >> 20], 1u);
  if (tid == 0) {
    s->pick[2] = 0;
    s->pick[4] = 0;
  }
  __syncthreads();

  // ---- boundary bin with one barrier: thread t owns ranks [t*per, t*per+per)
  constexpr int kPer = (kSelBins + NT - 1) / NT;
  uint32_t cnt[kPer];
  uint32_t own = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int k = tid * kPer + j;  // rank from the top
    const int b = kSelBins - 1 - k;
    cnt[j] = k < kSelBins ? s->hist[b] + s->hist[kSelBins + b] : 0u;
    own += cnt[j];
  }
  const uint32_t before0 = block_scan_excl_1s<NT>(own, s->warp_sums, nullptr);
  {
    uint32_t before = before0;
    const uint32_t krem = static_cast<uint32_t>(K);
    if (before < krem && krem <= before + own) {
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        if (before < krem && krem <= before + cnt[j]) {
          s->pick[0] = static_cast<uint32_t>(kSelBins - 1 - (tid * kPer + j));
          s->pick[1] = before;
          s->pick[3] = cnt[j];
        }
        before += cnt[j];
      }
    }
  }
  __syncthreads();
  const uint32_t b1 = s->pick[0];
  const uint32_t n1 = s->pick[3];
  const uint32_t krem1 = static_cast<uint32_t>(K) - s->pick[1];  // to take from bin b1
  constexpr int kMaxOwn = 4;  // candidates ranked per thread
  if (n1 > static_cast<uint32_t>(cand_cap) || n1 > static_cast<uint32_t>(kMaxOwn * NT)) {
    // too many keys share the boundary bin: exact radix passes instead
    __syncthreads();
    select_threshold<NT>(bits, d, K, s, cand_key, cand_cap, T_out, krem_out);
    return;
  }

  // ---- the boundary bin's keys, with their indices
  for (int i0 = 0; i0 < d; i0 += NT) {
    const int i = i0 + tid;
    const uint32_t k = i < d ? (bits[i] & kKeyMask) : 0u;
    const bool hit = i < d && (k >> 20) == b1;
    const uint32_t lanes = __ballot_sync(0xffffffffu, hit);
    uint32_t base = 0;
    if (lane == 0 && lanes) base = atomicAdd(&s->pick[2], __popc(lanes));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (hit) {
      const uint32_t slot = base + __popc(lanes & ((1u << lane) - 1u));
      cand_key[slot] = k;
      cand_idx[slot] = static_cast<uint32_t>(i);
    }
  }
  __syncthreads();

  // ---- rank every candidate (larger key first, then lower index); the one
  // ranked krem1-1 holds the K-th largest key overall
  const int nc = static_cast<int>(n1);
  uint32_t my_key[kMaxOwn], my_rank[kMaxOwn];
#pragma unroll
  for (int q = 0; q < kMaxOwn; ++q) {
    const int c = tid + q * NT;
    my_key[q] = 0;
    my_rank[q] = 0xffffffffu;
    if (c < nc) {
      const uint32_t kc = cand_key[c], ic = cand_idx[c];
      uint32_t rank = 0;
      for (int j = 0; j < nc; ++j) {
        const uint32_t kj = cand_key[j];
        rank += (kj > kc) | ((kj == kc) & (cand_idx[j] < ic));
      }
      my_key[q] = kc;
      my_rank[q] = rank;
      if (rank == krem1 - 1) s->pick[5] = kc;  // ranks are unique
    }
  }
  __syncthreads();
  const uint32_t T = s->pick[5];
  // keys equal to T that are kept = those ranked below krem1
  uint32_t eq_kept = 0;
#pragma unroll
  for (int q = 0; q < kMaxOwn; ++q) eq_kept += (my_rank[q] < krem1) & (my_key[q] == T);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) eq_kept += __shfl_xor_sync(0xffffffffu, eq_kept, o);
  if (lane == 0 && eq_kept) atomicAdd(&s->pick[4], eq_kept);
  __syncthreads();
  *T_out = T;
  *krem_out = s->pick[4];
  (void)warp;
  (void)NW;
}

// kept_chunk_base with a single-barrier scan; also returns the CTA total of
// kept entries would-be positions are relative to 0.  All threads call it.
template <int NT>
__device__ __forceinline__ void kept_chunk_base_1s(const uint32_t* bits, int i0, int i1,
                                                   uint32_t T, SelectScratch* s,
                                                   uint32_t* gt_before, uint32_t* eq_before) {
  uint32_t gt = 0, eq = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t k = bits[i] & kKeyMask;
    gt += k > T;
    eq += k == T;
  }
  const uint32_t packed = (eq << 16) | gt;  // d < 65536: no carry between halves
  const uint32_t excl = block_scan_excl_1s<NT>(packed, s->warp_sums, nullptr);
  *gt_before = excl & 0xffffu;
  *eq_before = excl >> 16;
}

}  // namespace larosa
