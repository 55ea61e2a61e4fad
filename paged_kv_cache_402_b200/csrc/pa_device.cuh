// Device helpers shared by the paged-cache kernels: the error word, mbarrier
// waits with an iteration limit, 1-D bulk copies (TMA engine) into shared
// memory, and 16-byte vector loads widened to fp32.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pagedattn.h"

namespace pa {

// Per-device error word (PA_DEVERR_* bits); read and cleared by the host.
__device__ int32_t g_error;

__device__ __forceinline__ void raise_error(int32_t bits) { atomicOr(&g_error, bits); }

// Where the first wait that gave up was: [taken, shared-memory address of
// its mbarrier, parity | block index << 1, thread index]; read and cleared
// by pa_read_wait_timeout.
__device__ uint32_t g_wait_timeout[4];

// Programmatic dependent launch: every kernel of the library is launched so
// that it may be scheduled before the kernel ahead of it in the stream has
// finished; it then waits here, before touching any memory, until that
// kernel has completed and its writes are visible.  Launched without that
// attribute, the wait returns at once.
__device__ __forceinline__ void wait_prior_grid() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Lets the kernel that follows in the stream be scheduled now (it still
// waits for this one to complete before it reads anything).
__device__ __forceinline__ void allow_next_grid() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Orders mbarrier initialisation before their use by other threads and by
// the async proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Arrives once and announces `bytes` of transaction that copies will bring.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Default limit of one mbarrier wait: a copy or MMA this library issued from
// valid memory completes in microseconds, so a wait this long means something
// is broken and the kernel should give up rather than hang.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// Waits for the phase of parity `parity` to complete.  Gives up after
// `limit_ns` nanoseconds of %globaltimer time and returns false (the caller
// records PA_DEVERR_TIMEOUT and drops its work).  try_wait may itself suspend
// the thread for a while, so the bound is on time, not on polls.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          uint64_t limit_ns = kWaitLimitNs) {
  const uint32_t addr = smem_u32(bar);
  uint64_t start = 0;
  for (uint32_t i = 0;; ++i) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(addr), "r"(parity)
        : "memory");
    if (done) return true;
    if (i == 0) {
      start = global_ns();
    } else if ((i & 63) == 0 && global_ns() - start > limit_ns) {
      if (atomicCAS(&g_wait_timeout[0], 0u, 1u) == 0u) {
        g_wait_timeout[1] = addr;
        g_wait_timeout[2] = parity | (blockIdx.x << 1);
        g_wait_timeout[3] = threadIdx.x;
      }
      return false;
    }
  }
}

// mbar_wait for a warp that is not on a critical path: between polls it
// sleeps, so that it leaves the issue slots of its sub-partition to the
// warps beside it.
__device__ __forceinline__ bool mbar_wait_idle(uint64_t *bar, uint32_t parity,
                                               uint64_t limit_ns = kWaitLimitNs) {
  const uint32_t addr = smem_u32(bar);
  const uint64_t start = global_ns();
  for (;;) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(addr), "r"(parity)
        : "memory");
    if (done) return true;
    if (global_ns() - start > limit_ns) {
      if (atomicCAS(&g_wait_timeout[0], 0u, 1u) == 0u) {
        g_wait_timeout[1] = addr;
        g_wait_timeout[2] = parity | (blockIdx.x << 1);
        g_wait_timeout[3] = threadIdx.x;
      }
      return false;
    }
    __nanosleep(100);
  }
}

// Makes this thread's earlier generic-proxy shared-memory accesses ordered
// before later async-proxy (bulk copy) accesses of the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Global -> shared bulk copy through the TMA engine; completion is counted in
// transaction bytes on `bar`.  dst, src 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_copy_g2s(void *dst, const void *src, uint32_t bytes,
                                              uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// L2 policy for data streamed once (the key/value tiles): evict first.
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ------------------------------------------------------------ element access

template <typename T>
struct Vec16;

// 16 bytes = 4 floats
template <>
struct Vec16<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const float *p, float (&x)[4]) {
    float4 v = *reinterpret_cast<const float4 *>(p);
    x[0] = v.x;
    x[1] = v.y;
    x[2] = v.z;
    x[3] = v.w;
  }
};

// 16 bytes = 8 bfloat16; widening is exact (a bf16 is the top half of an fp32)
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float (&x)[8]) {
    uint4 u = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};

__device__ __forceinline__ void store_out(float *p, float x) { *p = x; }
__device__ __forceinline__ void store_out(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

}  // namespace pa
