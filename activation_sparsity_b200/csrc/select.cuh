// Exact Top-K-by-magnitude selection for one vector held in shared memory,
// cooperative over a whole CTA of NT threads (NT a multiple of 32).
//
// LaRoSA keeps the K entries of largest magnitude of every rotated
// activation vector ("La RoSA" summary, 方法详解 / 技术框架; abstract: Top-K
// gives the same sparsity on every token).  Here ties go to the lower index
// and +0 / -0 are equal.
//
// An fp32 magnitude orders exactly like its bit pattern with the sign bit
// cleared, read as an unsigned integer (a 31-bit "key"), so the selection is
// integer work only and bit-exact.
//
//   kept_list()         the path every kernel takes (its steps are also used
//                       on their own): a 4096-bin histogram of bits 30..19
//                       (counted by the caller as it loads the vector), one
//                       scan for the boundary bin, the boundary bin's keys
//                       ranked against each other to find the K-th entry, and
//                       one scan that places every kept entry in ascending
//                       index order.
//   select_threshold()  its fallback when the boundary bin holds too many keys
//                       (heavy ties): an MSB-first radix select over bits
//                       30..20, 19..9 and 8..0 that yields the K-th largest
//                       key T and how many keys equal to T are kept (the
//                       lowest-indexed ones).
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

// Exclusive prefix over warps: every lane of warp w passes the same count c_w
// and receives c_0 + ... + c_{w-1}; *total (if not null) receives the sum
// over all warps.  One barrier; the caller must place a barrier between two
// uses of warp_sums.
template <int NT>
__device__ __forceinline__ uint32_t warp_base(uint32_t warp_count, uint32_t* warp_sums,
                                              uint32_t* total) {
  constexpr int NW = NT / 32;
  static_assert(NW <= 32, "one lane per warp");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) warp_sums[warp] = warp_count;
  __syncthreads();
  const uint32_t c = lane < NW ? warp_sums[lane] : 0u;
  if (total != nullptr) *total = __reduce_add_sync(0xffffffffu, c);
  return __reduce_add_sync(0xffffffffu, lane < warp ? c : 0u);
}

// ---------------------------------------------------------------- kept list
//
// The K kept entries of one vector -- the K largest keys, ties to the lower
// index -- are exactly those that come no later than the K-th entry (T, I)
// in the order (key descending, index ascending): every key above T, and the
// keys equal to T at indices <= I.  Finding (T, I):
//
//   1. the caller counts bits 30..19 of every key into kFineBins bins
//      (s->hist read as one array of kFineBins words);
//   2. fine_boundary(): one block scan over the bins from the top finds the
//      bin B holding the K-th largest key, the number of keys above B and in B;
//   3. kth_entry(): B's keys are listed in ascending index order and each is
//      ranked against the others; the one ranked krem - 1 is (T, I).  When B
//      holds more than cand_cap keys (heavy ties), select_threshold() gives T
//      and one more scan finds I.
//
// write_kept() then places the kept entries at their positions.  Steps 3 and
// write_kept walk warp segments: warp w owns the indices [w*seg, (w+1)*seg),
// seg a multiple of 32, lane l reads index w*seg + 32*j + l, and ballots
// order 32 consecutive indices at a time, so shared-memory reads are
// conflict-free and every store instruction writes one contiguous run.
constexpr int kFineBins = 4096;
constexpr int kFineShift = 19;
static_assert(2 * kSelBins >= kFineBins, "the fine histogram lives in SelectScratch::hist");

struct KthEntry {
  uint32_t T;  // key of the K-th entry
  int32_t I;   // its index
};

__device__ __forceinline__ bool is_kept(uint32_t key, int i, KthEntry e) {
  return key > e.T || (key == e.T && i <= e.I);
}

// Step 2 split in two, so the caller can overlap the histogram read with
// other loads: hist_share() reads this thread's kFineBins / NT counters,
// ranks [t*kPer, t*kPer+kPer) counted from the top, from global memory (through
// L2) or shared memory; boundary_from_share() finds the bin B holding the K-th
// largest counted key, the keys above B and the keys in B.  Requires
// 1 <= K <= (keys counted).  warp_sums (32 words) and pick (4 words) are
// shared memory.  boundary_from_share ends with a barrier.
template <int NT>
constexpr int kHistShare = kFineBins / NT;

template <int NT, bool kGlobal>
__device__ __forceinline__ void hist_share(const uint32_t* hist, uint32_t (&cnt)[kHistShare<NT>]) {
  static_assert(kFineBins % (4 * NT) == 0, "each thread owns whole 4-bin vectors");
  constexpr int kPer = kHistShare<NT>;
  const uint4* hv = reinterpret_cast<const uint4*>(hist + kFineBins - kPer * (threadIdx.x + 1));
#pragma unroll
  for (int q = 0; q < kPer / 4; ++q) {
    uint4 v;
    if constexpr (kGlobal) {
      v = __ldcg(hv + q);
    } else {
      v = hv[q];
    }
    cnt[kPer - 1 - 4 * q] = v.x;
    cnt[kPer - 2 - 4 * q] = v.y;
    cnt[kPer - 3 - 4 * q] = v.z;
    cnt[kPer - 4 - 4 * q] = v.w;
  }
}

template <int NT>
__device__ __forceinline__ void boundary_from_share(const uint32_t (&cnt)[kHistShare<NT>], int K,
                                                    uint32_t* warp_sums, uint32_t* pick,
                                                    uint32_t* B, uint32_t* above, uint32_t* nB) {
  constexpr int kPer = kHistShare<NT>;
  const int tid = threadIdx.x;
  uint32_t own = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) own += cnt[j];
  uint32_t before = block_scan_excl_1s<NT>(own, warp_sums, nullptr);
  const uint32_t k = static_cast<uint32_t>(K);
  if (before < k && k <= before + own) {
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      if (before < k && k <= before + cnt[j]) {
        pick[0] = static_cast<uint32_t>(kFineBins - 1 - (kPer * tid + j));
        pick[1] = before;
        pick[3] = cnt[j];
      }
      before += cnt[j];
    }
  }
  __syncthreads();
  *B = pick[0];
  *above = pick[1];
  *nB = pick[3];
}

template <int NT, bool kGlobal>
__device__ __forceinline__ void fine_boundary_at(const uint32_t* hist, int K, uint32_t* warp_sums,
                                                 uint32_t* pick, uint32_t* B, uint32_t* above,
                                                 uint32_t* nB) {
  uint32_t cnt[kHistShare<NT>];
  hist_share<NT, kGlobal>(hist, cnt);
  boundary_from_share<NT>(cnt, K, warp_sums, pick, B, above, nB);
}

// Step 2 on the histogram in s->hist (shared memory).
template <int NT>
__device__ __forceinline__ void fine_boundary(SelectScratch* s, int K, uint32_t* B, uint32_t* above,
                                              uint32_t* nB) {
  fine_boundary_at<NT, false>(s->hist, K, s->warp_sums, s->pick, B, above, nB);
}

// Warp segment [s0, s1) of the indices [0, d) for the calling warp.
template <int NT>
__device__ __forceinline__ void warp_segment(int d, int* s0, int* s1) {
  constexpr int NW = NT / 32;
  const int seg = ((d + NW - 1) / NW + 31) & ~31;
  *s0 = min(d, (static_cast<int>(threadIdx.x) >> 5) * seg);
  *s1 = min(d, *s0 + seg);
}

// Step 3: the K-th entry of the d keys in `bits`, given step 2's boundary
// (B, krem = K - above, nB).  Requires 1 <= K < d.  All NT threads call it;
// it begins and ends with a barrier.  cand_key / cand_idx: cand_cap entries
// of shared memory, cand_key 16-byte aligned.
template <int NT>
__device__ __forceinline__ KthEntry kth_entry(const uint32_t* bits, int d, int K, uint32_t B,
                                              uint32_t krem, uint32_t nB, SelectScratch* s,
                                              uint32_t* cand_key, uint32_t* cand_idx,
                                              int cand_cap) {
  const int tid = threadIdx.x, lane = tid & 31;
  const uint32_t below = (1u << lane) - 1u;  // lanes before this one
  int s0, s1;
  warp_segment<NT>(d, &s0, &s1);
  __syncthreads();  // pick[] of step 2 has been read by every thread

  if (nB > static_cast<uint32_t>(cand_cap)) {
    // ---- heavy ties: exact threshold T by radix passes; then I = the index
    // of the krem2-th key equal to T in ascending order
    uint32_t T = 0, krem2 = 0;
    select_threshold<NT>(bits, d, K, s, cand_key, cand_cap, &T, &krem2);
    uint32_t n_eq = 0;
    for (int i = s0 + lane; i < s1; i += 32) n_eq += (bits[i] & kKeyMask) == T;
    n_eq = __reduce_add_sync(0xffffffffu, n_eq);
    uint32_t base = warp_base<NT>(n_eq, s->warp_sums, nullptr);
    if (base < krem2 && krem2 <= base + n_eq) {  // this warp holds it
      for (int i0 = s0; i0 < s1; i0 += 32) {
        const int i = i0 + lane;
        const bool eq = i < s1 && (bits[i] & kKeyMask) == T;
        const uint32_t m = __ballot_sync(0xffffffffu, eq);
        if (eq && base + __popc(m & below) + 1u == krem2) s->pick[6] = static_cast<uint32_t>(i);
        base += __popc(m);
        if (base >= krem2) break;
      }
    }
    __syncthreads();
    return KthEntry{T, static_cast<int32_t>(s->pick[6])};
  }

  // ---- B's keys, with their indices, in ascending index order
  uint32_t n_cand = 0;
  for (int i = s0 + lane; i < s1; i += 32) n_cand += ((bits[i] & kKeyMask) >> kFineShift) == B;
  n_cand = __reduce_add_sync(0xffffffffu, n_cand);
  const uint32_t cbase = warp_base<NT>(n_cand, s->warp_sums, nullptr);
  if (n_cand != 0u) {  // warp-uniform
    uint32_t slot = cbase;
    for (int i0 = s0; i0 < s1; i0 += 32) {
      const int i = i0 + lane;
      const uint32_t k = i < s1 ? (bits[i] & kKeyMask) : 0u;
      const bool hit = i < s1 && (k >> kFineShift) == B;
      const uint32_t m = __ballot_sync(0xffffffffu, hit);
      if (hit) {
        cand_key[slot + __popc(m & below)] = k;
        cand_idx[slot + __popc(m & below)] = static_cast<uint32_t>(i);
      }
      slot += __popc(m);
    }
  }
  __syncthreads();

  // ---- rank each candidate (larger key first, then lower index, which is
  // the lower slot); the one ranked krem - 1 is the K-th entry
  const int nc = static_cast<int>(nB);
  for (int c = tid; c < nc; c += NT) {
    const uint32_t kc = cand_key[c];
    uint32_t r = 0;
    int j = 0;
    for (; j + 4 <= nc; j += 4) {
      const uint4 q = *reinterpret_cast<const uint4*>(cand_key + j);
      r += (q.x > kc) | ((q.x == kc) & (j < c));
      r += (q.y > kc) | ((q.y == kc) & (j + 1 < c));
      r += (q.z > kc) | ((q.z == kc) & (j + 2 < c));
      r += (q.w > kc) | ((q.w == kc) & (j + 3 < c));
    }
    for (; j < nc; ++j) {
      const uint32_t kj = cand_key[j];
      r += (kj > kc) | ((kj == kc) & (j < c));
    }
    if (r == krem - 1u) {  // ranks are unique
      s->pick[5] = kc;
      s->pick[6] = cand_idx[c];
    }
  }
  __syncthreads();
  return KthEntry{s->pick[5], static_cast<int32_t>(s->pick[6])};
}

// Kept entries of the d keys in `bits` at positions [p0, p1) of the kept
// list (ascending index order): rows[pos - p0] = index, vals[pos - p0] = the
// raw fp32 value.  All NT threads call it; it holds one barrier.
template <int NT>
__device__ __forceinline__ void write_kept(const uint32_t* bits, int d, KthEntry e, int p0, int p1,
                                           int32_t* rows, float* vals, SelectScratch* s) {
  const int lane = threadIdx.x & 31;
  const uint32_t below = (1u << lane) - 1u;
  int s0, s1;
  warp_segment<NT>(d, &s0, &s1);
  uint32_t n_kept = 0;
  for (int i = s0 + lane; i < s1; i += 32) n_kept += is_kept(bits[i] & kKeyMask, i, e);
  n_kept = __reduce_add_sync(0xffffffffu, n_kept);
  uint32_t pos = warp_base<NT>(n_kept, s->warp_sums, nullptr);
  if (pos < static_cast<uint32_t>(p1) && pos + n_kept > static_cast<uint32_t>(p0)) {
    for (int i0 = s0; i0 < s1 && pos < static_cast<uint32_t>(p1); i0 += 32) {
      const int i = i0 + lane;
      const uint32_t u = i < s1 ? bits[i] : 0u;
      const bool kept = i < s1 && is_kept(u & kKeyMask, i, e);
      const uint32_t m = __ballot_sync(0xffffffffu, kept);
      const uint32_t at = pos + __popc(m & below);
      if (kept && at >= static_cast<uint32_t>(p0) && at < static_cast<uint32_t>(p1)) {
        rows[at - p0] = i;
        vals[at - p0] = __uint_as_float(u);
      }
      pos += __popc(m);
    }
  }
}

// Positions [p0, p1) of the kept list of the d keys in `bits`, whose bits
// 30..19 the caller has counted into s->hist (then a barrier).  Requires
// 1 <= K < d.  All NT threads call it.
template <int NT>
__device__ __forceinline__ void kept_list(const uint32_t* bits, int d, int K, SelectScratch* s,
                                          uint32_t* cand_key, uint32_t* cand_idx, int cand_cap,
                                          int p0, int p1, int32_t* rows, float* vals) {
  uint32_t B, above, nB;
  fine_boundary<NT>(s, K, &B, &above, &nB);
  const KthEntry e = kth_entry<NT>(bits, d, K, B, static_cast<uint32_t>(K) - above, nB, s, cand_key,
                                   cand_idx, cand_cap);
  write_kept<NT>(bits, d, e, p0, p1, rows, vals, s);
}

}  // namespace larosa
