// Device-side building blocks shared by the library's kernels (sm_100a).
//
// mbarrier + bulk-copy (TMA, non-tensor) pipeline primitives, programmatic
// dependent launch controls, bounded waits and the device status word.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "larosa.h"

namespace larosa {

// Every wait inside a kernel gives up after a limit of %globaltimer
// nanoseconds, reports LAROSA_DEV_TIMEOUT and lets the kernel exit.  The
// limit is read on the host at each launch (larosa_set_wait_limit_ns) and
// passed in the kernel's parameters; this is its default.
constexpr unsigned long long kDefaultWaitLimitNs = 2000000000ull;

// The wait limit for launches enqueued now (api.cu).
unsigned long long wait_limit_ns();

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void report(int* dev_status, int bits) {
  if (dev_status != nullptr) atomicOr(dev_status, bits);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- PDL

// Blocks until every grid this one depends on (the previous kernel on the
// stream, when launched with programmatic stream serialisation) has completed
// and its memory is visible.  A no-op for ordinary launches.
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Lets the next kernel on the stream start launching its blocks.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- gpu-scope ordering

// Adds v to *p with release semantics at GPU scope: every write that happens
// before it (this thread's, and through a CTA barrier the whole CTA's) is
// visible to a thread that observes the new value with acquire semantics.
// Returns the old value.
__device__ __forceinline__ unsigned atomic_add_release_gpu(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.add.release.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// The same with acquire-release semantics: the caller also sees every write
// released by earlier adds to *p.
__device__ __forceinline__ unsigned atomic_add_acq_rel_gpu(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Makes barrier initialisation visible to the async (TMA) proxy and to the
// rest of the cluster.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Waits for phase `parity` of `bar` to complete.  Returns false (without
// reporting) if it did not within limit_ns, or as soon as *abort becomes
// nonzero.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort, unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  unsigned long long t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (abort != nullptr && *abort) return false;
      if (global_timer_ns() - t0 > limit_ns) return false;
    }
  }
}

// ---------------------------------------------------------------- bulk copy

// L2 policy: lines fetched with it are the first candidates for eviction
// (weights are streamed once per call and should not push out activations).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// One-dimensional bulk copy global -> shared through the TMA unit, completing
// `bytes` of transaction count on `bar`.  src and dst 16-byte aligned, bytes a
// multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(void* dst_smem, const void* src, uint32_t bytes,
                                              uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst_smem)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Asks the TMA unit to bring `bytes` of global memory at `src` into L2.  A
// hint: nothing waits for it and it changes no result.  src 16-byte aligned,
// bytes a multiple of 16.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ---------------------------------------------------------------- conversions

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

// Unpacks N consecutive elements of type T starting at a shared-memory
// address aligned to N * sizeof(T) bytes into fp32.
template <typename T, int N>
struct VecLoad;

template <>
struct VecLoad<__nv_bfloat16, 8> {
  static __device__ __forceinline__ void load(const void* p, float (&out)[8]) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      out[2 * i] = __uint_as_float(w[i] << 16);
      out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};
template <>
struct VecLoad<__nv_bfloat16, 4> {
  static __device__ __forceinline__ void load(const void* p, float (&out)[4]) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    out[0] = __uint_as_float(u.x << 16);
    out[1] = __uint_as_float(u.x & 0xffff0000u);
    out[2] = __uint_as_float(u.y << 16);
    out[3] = __uint_as_float(u.y & 0xffff0000u);
  }
};
template <>
struct VecLoad<__nv_bfloat16, 2> {
  static __device__ __forceinline__ void load(const void* p, float (&out)[2]) {
    uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    out[0] = __uint_as_float(u << 16);
    out[1] = __uint_as_float(u & 0xffff0000u);
  }
};
template <>
struct VecLoad<float, 4> {
  static __device__ __forceinline__ void load(const void* p, float (&out)[4]) {
    float4 v = *reinterpret_cast<const float4*>(p);
    out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
  }
};
template <>
struct VecLoad<float, 2> {
  static __device__ __forceinline__ void load(const void* p, float (&out)[2]) {
    float2 v = *reinterpret_cast<const float2*>(p);
    out[0] = v.x; out[1] = v.y;
  }
};
template <>
struct VecLoad<float, 1> {
  static __device__ __forceinline__ void load(const void* p, float (&out)[1]) {
    out[0] = *reinterpret_cast<const float*>(p);
  }
};

}  // namespace larosa
