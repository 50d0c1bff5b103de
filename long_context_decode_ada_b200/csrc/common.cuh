// common.cuh -- device helpers shared by the libskv kernels (sm_100a).
//
// Everything here is hand-written for Blackwell: mbarrier-tracked bulk
// asynchronous copies (cp.async.bulk, no multicast), legacy-form mma.sync
// for the small P.V contraction, exact integer / IEEE-rounded conversions
// for the bit-exact encode.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/skv.h"

namespace skv {

constexpr int kHeadDim = 128;
constexpr int kPairs = 64;
constexpr int kHdrBytes = 16;
constexpr uint8_t kPageMagic = 0x5A;

// Bytes per (token, kv head) of each tier at d = 128.
__host__ __device__ constexpr int tier_row_bytes(int tier) {
  return tier == 0 ? 512 : (tier == 1 ? 196 : (tier == 2 ? 180 : 0));
}

// Record the first device-side error.
__device__ __forceinline__ void report(int32_t* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// ---------------------------------------------------------------------------
// shared-memory addresses, mbarriers, bulk copies
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

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
          bar),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of a phase (never suspends the thread).
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait that lets the thread sleep (until the phase completes, or at
// most `hint_ns`) instead of returning at once: waiting warps then take no
// issue slots and no shared-memory pipe bandwidth from the working warps.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity,
                                                    uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// A bounded wait: `limit` SM clocks at most (kWaitLimitCycles, ~1 s, by
// default).  Returns false when the limit runs out or when another thread
// of the CTA has raised *abort.
constexpr long long kWaitLimitCycles = 2000000000LL;

__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  volatile int* abort_flag,
                                                  long long limit = kWaitLimitCycles) {
  if (limit < kWaitLimitCycles) {
    // a short limit (set to exercise the timeout path): poll without
    // suspending, so that the limit and not a sleep decides
    const long long t0 = clock64();
    while (!mbar_test_wait(bar, parity))
      if (*abort_flag || clock64() - t0 > limit) return false;
    return true;
  }
  if (mbar_try_wait(bar, parity)) return true;
  long long t0 = clock64();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, 200000u)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > limit) return false;
  }
}

// 1-D bulk asynchronous copy global -> this CTA's shared memory, completing
// `bytes` of transaction count on `bar`.  No multicast.  dst, src and bytes
// must be 16-byte aligned / a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// arithmetic helpers
// ---------------------------------------------------------------------------

// Four signed int8 (one 32-bit word, byte i = element i) -> two f16x2:
// lo = (e0, e1), hi = (e2, e3).  Exact: 0x64XX is 1024 + XX in fp16, with
// XX = e + 128, and 1152 = 1024 + 128 is subtracted.
__device__ __forceinline__ void s8x4_to_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  uint32_t u = w ^ 0x80808080u;
  uint32_t a = __byte_perm(u, 0x64646464u, 0x4140);
  uint32_t b = __byte_perm(u, 0x64646464u, 0x4342);
  const __half2 bias = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));
  __half2 ha = __hsub2(*reinterpret_cast<__half2*>(&a), bias);
  __half2 hb = __hsub2(*reinterpret_cast<__half2*>(&b), bias);
  lo = *reinterpret_cast<uint32_t*>(&ha);
  hi = *reinterpret_cast<uint32_t*>(&hb);
}

// The same four int8 as fp16 values offset by +1152 (0x64XX = 1024 + XX,
// XX = e + 128): exact, one subtraction fewer; the caller removes 1152.
__device__ __forceinline__ void s8x4_to_f16x2x2_biased(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t u = w ^ 0x80808080u;
  lo = __byte_perm(u, 0x64646464u, 0x4140);
  hi = __byte_perm(u, 0x64646464u, 0x4342);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// D += A * B, m16n8k8, f16 (or bf16) inputs, f32 accumulation.
__device__ __forceinline__ void mma_16816_f16(float* d, uint32_t a0, uint32_t a1, uint32_t b) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b));
}

__device__ __forceinline__ void mma_16816_bf16(float* d, uint32_t a0, uint32_t a1, uint32_t b) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b));
}

// D += A * B, m16n8k16 (A: 4 x f16x2, B: 2 x f16x2), f32 accumulation.
__device__ __forceinline__ void mma_16816k16_f16(float* d, uint32_t a0, uint32_t a1, uint32_t a2,
                                                 uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_16816k16_bf16(float* d, uint32_t a0, uint32_t a1, uint32_t a2,
                                                  uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Unsigned 128-bit integer to double, correctly rounded (nearest-even): keep
// the top 64 significant bits with every lower bit folded into a sticky
// lowest bit, convert, then scale by the dropped power of two (exact).
__device__ __forceinline__ double u128_to_double_rn(unsigned long long hi,
                                                    unsigned long long lo) {
  if (hi == 0) return __ull2double_rn(lo);
  int s = 64 - __clzll(hi);  // bits above the low 64, 1..64
  unsigned long long top, rest;
  if (s == 64) {
    top = hi;
    rest = lo;
  } else {
    top = (hi << (64 - s)) | (lo >> s);
    rest = lo & ((1ull << s) - 1);
  }
  top |= (rest != 0ull) ? 1ull : 0ull;
  double x = __ull2double_rn(top);
  return __dmul_rn(x, __longlong_as_double((long long)(1023 + s) << 52));
}

// fp16 bit pattern -> integer m with value = m * 2^-24 (|m| < 2^41).
__device__ __forceinline__ long long half_bits_to_m(uint32_t h) {
  uint32_t e = (h >> 10) & 31u, f = h & 1023u;
  long long m = (e == 0) ? (long long)f : ((long long)(1024u + f) << (e - 1));
  return (h & 0x8000u) ? -m : m;
}

}  // namespace skv
