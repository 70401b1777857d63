// pa_device.cuh -- sm_100a device helpers for the paged-attention decode
// kernels: the visible-span rule (shared by host planning and kernels),
// mbarrier and bulk-copy PTX wrappers, bf16 unpacking and exp2/log2.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/pagedattn.h"
#include "pa_span.h"

namespace pa {

// Device-side status word (bits of PA_DEV_*), read and cleared by
// pa_device_status().  This header is included by exactly one translation
// unit (pa_kernels.cu), which owns the definition.
__device__ unsigned int g_pa_status = 0;

constexpr float kNegInf = -__builtin_huge_valf();

// ---------------------------------------------------------------------------
// PTX wrappers (shared-memory mbarriers, bulk copies, math)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// Bounded wait: spins on try_wait for at most ~kWaitCycles SM clocks (about a
// second).  On timeout it records PA_DEV_TIMEOUT in the status word and
// returns false; callers then stop consuming and leave the kernel cleanly.
constexpr long long kWaitCycles = 2000000000LL;

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) {
      atomicOr(&g_pa_status, PA_DEV_TIMEOUT);
      return false;
    }
  }
  return true;
}

// 1-D bulk copy global -> shared (the TMA engine's non-tensor path); completes
// `bytes` transaction bytes on `bar`.  Addresses 16-byte aligned, bytes a
// multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// 2^x with the SFU (ex2.approx, flush-to-zero); 2^-inf = +0.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two packed bf16 (element 0 in the low half) -> float2, exact.
__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

__device__ __forceinline__ uint4 lds128(const void* p) {
  return *reinterpret_cast<const uint4*>(p);
}

__device__ __forceinline__ uint4 ldg128_nc(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Sum of query_lens[0..b): the packed offset of row b's first query token
// (a negative length counts as 0).  Warp-cooperative; every lane returns the
// same value.
__device__ __forceinline__ int row_token_offset(const int32_t* query_lens, int b, int lane) {
  int s = 0;
  for (int i = lane; i < b; i += 32) s += max(query_lens[i], 0);
  return __reduce_add_sync(0xffffffffu, s);
}

}  // namespace pa
