// pa_device.cuh -- sm_100a device helpers for the paged-attention decode
// kernels: the visible-span rule (shared by host planning and kernels),
// mbarrier and bulk-copy PTX wrappers, bf16 unpacking and exp2/log2.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/pagedattn.h"
#include "pa_kernels.cuh"
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

// try_wait with a suspend-time hint: the thread sleeps until the phase
// completes or ~1 us passes, instead of spinning through instructions other
// warps could issue.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity), "r"(1000u)
      : "memory");
  return done != 0;
}

// Bounded wait: spins on try_wait for at most ~kWaitCycles SM clocks (about a
// second).  On timeout it records PA_DEV_TIMEOUT in the status word and
// returns false; callers then stop consuming and leave the kernel cleanly.

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait_sleep(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) {
      atomicOr(&g_pa_status, PA_DEV_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Epoch-tagged counters of the work-list schedule live in the caller's
// workspace, which is never initialised: the high 32 bits hold the epoch of
// the call that last touched the counter, the low 32 bits its count.  The
// first touch of a call resets a stale counter (one CAS: if it fails, another
// CTA of the same call reset or advanced it first, so it is current).
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// epoch_touch split in two: `seen` is a value of the counter read earlier
// (ld_relaxed_u64); a stale one is reset by a CAS that fails harmlessly if
// another CTA of this call got there first.
__device__ __forceinline__ void epoch_reset_if_stale(unsigned long long* c,
                                                     unsigned long long seen,
                                                     unsigned int epoch) {
  if ((unsigned int)(seen >> 32) != epoch) atomicCAS(c, seen, (unsigned long long)epoch << 32);
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ void epoch_touch(unsigned long long* c, unsigned int epoch) {
  const unsigned long long cur = ld_acquire_u64(c);
  if ((unsigned int)(cur >> 32) != epoch) atomicCAS(c, cur, (unsigned long long)epoch << 32);
}

// First stage index of a claim from the counter's previous value v (an
// atomicAdd's result); INT_MAX (stop) if the counter was not this call's,
// which cannot happen after epoch_touch.
__device__ __forceinline__ int claim_value(unsigned long long v, unsigned int epoch) {
  return (unsigned int)(v >> 32) == epoch ? (int)(unsigned int)v : 0x7fffffff;
}

__device__ __forceinline__ void epoch_arrive(unsigned long long* c, unsigned int epoch) {
  epoch_touch(c, epoch);
  atomicAdd(c, 1ull);
}

// Bounded wait for `target` arrivals of this epoch on a counter other CTAs
// bump: at most `limit` SM clocks (the call's wait_cycles, ~1 s unless a test
// shortens it); on timeout PA_DEV_TIMEOUT is recorded and false returned.
__device__ __forceinline__ bool epoch_wait(const unsigned long long* c, unsigned int epoch,
                                           unsigned int target, long long limit) {
  const long long t0 = clock64();
  while (true) {
    const unsigned long long v = ld_acquire_u64(c);
    if ((unsigned int)(v >> 32) == epoch && (unsigned int)v >= target) return true;
    if (clock64() - t0 > limit) {
      atomicOr(&g_pa_status, PA_DEV_TIMEOUT);
      return false;
    }
  }
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

// The same bulk copy with an L2 cache policy (createpolicy).
__device__ __forceinline__ void bulk_g2s_hint(uint32_t dst, const void* src, uint32_t bytes,
                                              uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

// 2-D tiled TMA load global -> shared (no multicast) of the box at (x, y)
// of `map` (a __grid_constant__ kernel parameter); completes the box's bytes
// on `bar`.  x * element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// 3-D tiled TMA load (no multicast) of the box at (x, y, z).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* map, int x, int y, int z,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// The same load with an L2 cache policy (createpolicy), e.g. evict-first for
// data that is read once.
__device__ __forceinline__ void tma_load_3d_hint(uint32_t dst, const void* map, int x, int y,
                                                 int z, uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar), "l"(policy)
      : "memory");
}

// L2 policy whose lines are evicted first: the KV stream, read once, then
// leaves block tables, lengths, q and partials in L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// L2 prefetch of the box at (x, y, z) of `map` (no multicast): no
// shared-memory destination and no barrier; a later load of the box is served
// from L2.
__device__ __forceinline__ void tma_prefetch_3d(const void* map, int x, int y, int z) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(z)
               : "memory");
}

// Loads through L2 only (ld.global.cg) as volatile asm: issued in program
// order, so a batch of them is in flight before the first use.
__device__ __forceinline__ float ld_cg_f32(const float* p) {
  float v;
  asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ float4 ld_cg_f32x4(const float4* p) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

// Relaxed (non-racing) load of an int that another grid may be writing.
__device__ __forceinline__ int ld_relaxed_s32(const int32_t* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void prefetch_tensormap(const void* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Four 8x8 b16 matrices from shared memory (rows addressed by lanes 0-7,
// 8-15, 16-23, 24-31); .trans delivers them transposed.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D += A * B on the tensor cores: A 16x16 bf16 (row), B 16x8 bf16 (col),
// D 16x8 fp32.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Two FP8 e4m3 codes (low byte -> low half) to two f16 values: every e4m3
// number, subnormals included, is exactly representable in f16; the NaN code
// stays NaN.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t codes16) {
  uint32_t y;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(y) : "h"((unsigned short)codes16));
  return y;
}

// Four FP8 e4m3 codes (bytes 0..3) to two f16 pairs: lo = bytes 0, 1;
// hi = bytes 2, 3.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t codes, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(codes));
}

// Two floats to two e4m3 codes (round to nearest even, saturating at
// +-448); lo goes to the low byte.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  unsigned short y;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(y) : "f"(hi), "f"(lo));
  return y;
}

// bf16 pair -> f16 pair (exact for |x| in f16's normal range; larger values
// become inf, smaller ones round to f16 subnormals).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  return pack_f16x2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// f16 pair -> bf16 pair; exact for values that came from e4m3 codes.
__device__ __forceinline__ uint32_t f16x2_to_bf16x2(uint32_t w) {
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w));
  return pack_bf16x2(f.x, f.y);
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
