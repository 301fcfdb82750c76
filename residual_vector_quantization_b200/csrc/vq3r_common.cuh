// Shared device helpers of the VQ3R library: element loads, IEEE binary16
// conversion, the device error word and the mbarrier / bulk-copy (TMA)
// primitives used to stage tables in shared memory.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "vq3r.h"

namespace vq3r {

constexpr int kStages = VQ3R_STAGES;
constexpr int kCodewords = VQ3R_CODEWORDS;
constexpr int kDim = VQ3R_DIM;
constexpr int kCodebookFloats = kStages * kCodewords * kDim;  // 6144
constexpr int kCodebookBytes = kCodebookFloats * 4;           // 24 KiB

// Index formats.  FMT_VQ3R: three 1-byte indices into 256-entry codebooks
// [3][256][8], one byte plane per stage.  FMT_VQ4P (page §5, VQ3R's sibling at
// the same 3.00 bits/weight): four 6-bit indices into 64-entry codebooks
// [4][64][8], packed into the 24-bit word i1 | i2 << 6 | i3 << 12 | i4 << 18
// whose byte p is stored in plane p.  Both read three byte planes per vector.
constexpr int FMT_VQ3R = 0, FMT_VQ4P = 1;

// Error codes a kernel may leave in the device error word.
constexpr int kDevErrMbarTimeout = 1;  // a bulk copy into shared memory did not complete within ~1 s
constexpr int kDevErrBarrierTimeout = 2;  // not all CTAs of a tiled GEMV reached its grid barrier within ~1 s

// Device error word (one per GPU that loads the library).
__device__ int g_device_error;

__device__ __forceinline__ void set_device_error(int code) { atomicCAS(&g_device_error, 0, code); }

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }
__device__ __forceinline__ float f16_bits_to_f32(uint32_t h) {
  return __half2float(__ushort_as_half((unsigned short)h));
}

// Eight consecutive elements starting at element `off` (16-byte aligned), widened to float.
template <int DT>
__device__ __forceinline__ void load8(const void* base, int64_t off, float w[8]) {
  if constexpr (DT == VQ3R_F32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + off);
    float4 a = __ldcs(p), b = __ldcs(p + 1);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + off);
    uint4 a = __ldcs(p);
    uint32_t u[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
      if constexpr (DT == VQ3R_BF16) {
        w[2 * i] = bf16_bits_to_f32(u[i] & 0xFFFFu);
        w[2 * i + 1] = bf16_bits_to_f32(u[i] >> 16);
      } else {
        w[2 * i] = f16_bits_to_f32(u[i] & 0xFFFFu);
        w[2 * i + 1] = f16_bits_to_f32(u[i] >> 16);
      }
    }
  }
}

// One element, widened to float.
template <int DT>
__device__ __forceinline__ float load1(const void* base, int64_t off) {
  if constexpr (DT == VQ3R_F32) return static_cast<const float*>(base)[off];
  else if constexpr (DT == VQ3R_BF16) return bf16_bits_to_f32(static_cast<const uint16_t*>(base)[off]);
  else return f16_bits_to_f32(static_cast<const uint16_t*>(base)[off]);
}

// binary64 -> binary16 bits, round to nearest even on the exact binary64
// value, overflow (|x| >= 65520) saturating to +-65504, NaN -> quiet NaN.
// Works on the bit pattern: keep 11 significant bits, round on the rest.
__device__ __forceinline__ uint16_t f64_to_f16_sat_rne(double x) {
  const uint64_t b = (uint64_t)__double_as_longlong(x);
  const uint16_t sign = (uint16_t)((b >> 48) & 0x8000u);
  const uint64_t a = b & 0x7FFFFFFFFFFFFFFFull;
  if (a > 0x7FF0000000000000ull) return 0x7E00;
  if (a == 0) return sign;
  if (a >= 0x40EFFE0000000000ull) return sign | 0x7BFF;  // |x| >= 65520
  int e = (int)(a >> 52) - 1023;
  const uint64_t m = (a & 0x000FFFFFFFFFFFFFull) | (1ull << 52);
  if (e >= -14) {
    uint64_t q = m >> 42;
    const uint64_t rem = m & ((1ull << 42) - 1), half = 1ull << 41;
    if (rem > half || (rem == half && (q & 1))) q++;
    if (q == 2048) { q = 1024; e++; }
    return sign | (uint16_t)(((e + 15) << 10) | (int)(q - 1024));
  }
  const int sh = 28 - e;  // units of 2^-24
  if (sh > 54) return sign;
  uint64_t q = m >> sh;
  const uint64_t rem = m & ((1ull << sh) - 1), half = 1ull << (sh - 1);
  if (rem > half || (rem == half && (q & 1))) q++;
  return sign | (uint16_t)q;
}

// ---- streaming loads ----

// L2 cache policy that makes lines the first candidates for eviction: used
// for data read exactly once (the index stream), so that it does not push
// out what is read again (tables' inputs, partial sums).
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 16-byte read-only load that allocates in neither L1 nor (preferentially) L2.
__device__ __forceinline__ uint4 ldg_stream16(const void* p, uint64_t pol) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p), "l"(pol));
  return v;
}

// ---- shared-memory mbarrier and bulk asynchronous copy (TMA, no multicast) ----

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* mbar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(mbar)), "r"(count) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* mbar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(mbar)), "r"(bytes)
               : "memory");
}

// Global -> shared bulk copy completing on mbar; dst, src 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* mbar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(mbar))
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* mbar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(mbar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Orders this thread's earlier generic-proxy accesses of shared memory before
// later asynchronous-proxy (bulk copy) writes to it.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Non-blocking test of the phase with the given parity.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* mbar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(mbar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase with the given parity to complete, giving up after
// about one second (records kDevErrMbarTimeout and returns false).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* mbar, uint32_t parity) {
  if (mbar_try_wait(mbar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    if (mbar_try_wait(mbar, parity)) return true;
    if (global_timer_ns() - t0 > 1000000000ull) {
      set_device_error(kDevErrMbarTimeout);
      return false;
    }
  }
}

// Self-test of the failure path: one warp initialises a shared-memory barrier
// that nothing arrives at and waits on it.  The bounded wait gives up after
// about one second, records kDevErrMbarTimeout, and the kernel returns.
__global__ void __launch_bounds__(32) selftest_wait_kernel() {
  __shared__ uint64_t mbar;
  if (threadIdx.x == 0) mbar_init(&mbar, 1);
  __syncwarp();
  (void)mbar_wait_bounded(&mbar, 0);
}

}  // namespace vq3r
