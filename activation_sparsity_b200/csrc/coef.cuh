// Coefficient rows for the tensor-core sparse linear (rot_umma.cu): each fp32
// coefficient c enters the bf16 MMA as a head and a tail.
#pragma once

#include <cuda_bf16.h>

namespace larosa {

// head = bf16(c), tail = bf16(c - head), both rounded to nearest even (about
// 16 significant bits of c kept in all).
__device__ __forceinline__ void split_head_tail(float c, __nv_bfloat16* head, __nv_bfloat16* tail) {
  const __nv_bfloat16 h = __float2bfloat16_rn(c);
  *head = h;
  *tail = __float2bfloat16_rn(c - __bfloat162float(h));
}

// Writes hi[0, d) and lo[0, d): the head and tail of coef(i) for every i,
// with the block's NT threads, 8 entries (one 16-byte store to each row) per
// step.  d a multiple of 8; hi and lo 16-byte aligned.
template <int NT, typename Coef>
__device__ __forceinline__ void write_head_tail_rows(int d, Coef coef, __nv_bfloat16* hi, __nv_bfloat16* lo) {
  for (int v = threadIdx.x; v < d / 8; v += NT) {
    __align__(16) __nv_bfloat16 h[8], t[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) split_head_tail(coef(8 * v + e), &h[e], &t[e]);
    reinterpret_cast<uint4*>(hi)[v] = *reinterpret_cast<const uint4*>(h);
    reinterpret_cast<uint4*>(lo)[v] = *reinterpret_cast<const uint4*>(t);
  }
}

}  // namespace larosa
