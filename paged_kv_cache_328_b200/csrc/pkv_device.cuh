// Device helpers for libpagedkv: the sticky error word, shared-memory mbarriers,
// bulk global->shared copies and 16-byte element conversions (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "pagedkv.h"

namespace pkv {

// One word per device.  The first reason recorded wins; pkv_get_device_error
// reads and clears it.
__device__ int g_error_word = 0;

__device__ __forceinline__ void flag_error(int reason) { atomicCAS(&g_error_word, 0, reason); }

// Bound on any spin on a shared-memory barrier: about one second at the B200's
// maximum SM clock.  A wait that runs out records PKV_DEV_WAIT_TIMEOUT.
constexpr long long kWaitLimitCycles = 2000000000LL;

// Offset of row (block, head, slot) in a [num_blocks][num_heads][block_size][row]
// pool, in units of the row's elements (or of 16-byte vectors when `row` counts
// vectors).  Every kernel that addresses the pool goes through this helper.
__device__ __forceinline__ size_t pool_row(long long block, int head, long long slot, int num_heads,
                                           int block_size, int row) {
  return (((size_t)block * num_heads + head) * block_size + slot) * row;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Makes barrier initialisation visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Waits for the phase with the given parity to complete.  Returns false if the
// CTA-wide abort flag is raised or the wait exceeds kWaitLimitCycles.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                  long long limit_cycles = kWaitLimitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > limit_cycles) return false;
  }
}

// Self-test of the bounded wait: one thread waits on a barrier that nothing
// arrives on; the wait must give up after `limit_cycles` and record
// PKV_DEV_WAIT_TIMEOUT, after which the kernel returns normally.
__device__ int g_selftest_waited_out = 0;

__global__ void wait_timeout_selftest_kernel(long long limit_cycles) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait_bounded(&bar, 0, &abort_flag, limit_cycles);
    if (!ok) flag_error(PKV_DEV_WAIT_TIMEOUT);
    g_selftest_waited_out = ok ? 0 : 1;
  }
}

// L2 policy for data read exactly once per call (the streamed K/V chunks).
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t policy;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
  return policy;
}

// 2^x with the hardware approximation (one MUFU instruction; relative error
// ~2^-22; -inf gives +0, flush-to-zero).
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Bulk (TMA-engine) copy of `bytes` contiguous bytes from global to this CTA's
// shared memory; completion is reported to `bar` as transaction bytes.  Both
// addresses 16-byte aligned, bytes a multiple of 16.  The copy lands in this CTA only.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar,
                                          uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(smem_addr(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// Named barrier over `count` threads (multiple of 32) of this CTA.
__device__ __forceinline__ void named_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ---------------------------------------------------------------------------
// Storage element types.  A 16-byte chunk holds kPerChunk elements; widen() turns
// it into floats exactly (fp16 and bf16 are subsets of fp32).
// ---------------------------------------------------------------------------
template <typename T>
struct Elem;

template <>
struct Elem<float> {
  static constexpr int kPerChunk = 4;
  __device__ __forceinline__ static void widen(const uint4& c, float* f) {
    f[0] = __uint_as_float(c.x);
    f[1] = __uint_as_float(c.y);
    f[2] = __uint_as_float(c.z);
    f[3] = __uint_as_float(c.w);
  }
};

template <>
struct Elem<__half> {
  static constexpr int kPerChunk = 8;
  __device__ __forceinline__ static void widen(const uint4& c, float* f) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h2;
      memcpy(&h2, &w[i], 4);
      const float2 v = __half22float2(h2);
      f[2 * i] = v.x;
      f[2 * i + 1] = v.y;
    }
  }
};

template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kPerChunk = 8;
  // A bf16 value is the upper half of the fp32 with the same value.
  __device__ __forceinline__ static void widen(const uint4& c, float* f) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};

}  // namespace pkv
