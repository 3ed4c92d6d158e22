// common.cuh -- device helpers shared by the decode-step kernels (sm_100a).
//
// Thin inline-PTX wrappers: mbarrier + bulk-copy (TMA engine) pipeline pieces,
// bounded waits, number-format conversions done by single hardware instructions
// (E2M1/E4M3 -> f16x2, f32 -> E4M3), E8M0 -> fp32 by exponent placement, and the
// warp-level m16n8k16 tensor-core products used by the GEMV kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Device-side error codes written to the workspace status word.
enum : int { DEV_OK = 0, DEV_ERR_TIMEOUT = 7 };

// Every spin-wait gives up after a bounded time of %globaltimer, sets the status word
// and lets the kernel return instead of hanging the GPU.  The status word is the first
// word of a 256-byte control block; the 64-bit word 16 bytes after it holds the limit
// in nanoseconds (0: WAIT_LIMIT_NS).  Callers shorten it only to test the timeout path.
constexpr unsigned long long WAIT_LIMIT_NS = 2000000000ull;  // 2 s
__device__ __forceinline__ unsigned long long wait_limit(const int* status) {
  if (!status) return WAIT_LIMIT_NS;
  const unsigned long long v =
      *reinterpret_cast<const volatile unsigned long long*>(reinterpret_cast<const char*>(status) + 16);
  return v ? v : WAIT_LIMIT_NS;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// mbarrier + bulk copy
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// As mbar_try_wait, but the thread may be suspended in hardware for up to ns
// nanoseconds until the phase completes, instead of spinning.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}
// Wait for the phase with the given parity to complete.  Bounded: after
// WAIT_LIMIT_NS it records DEV_ERR_TIMEOUT in *status and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns(), lim = wait_limit(status);
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > lim) {
      if (status) atomicExch(status, DEV_ERR_TIMEOUT);
      return false;
    }
  }
}

// Bulk copy global -> shared through the TMA engine, completing on an mbarrier.
// dst and src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
// L2 policy for weights that are read exactly once per step.
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ---------------------------------------------------------------------------
// Format conversions (single hardware instructions; no table constants)
// ---------------------------------------------------------------------------
// Four bytes of packed E2M1 pairs -> four f16x2 (byte i -> out[i]; low nibble -> low half).
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t& o0, uint32_t& o1, uint32_t& o2,
                                                uint32_t& o3) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(o0), "=r"(o1), "=r"(o2), "=r"(o3)
      : "r"(w));
}
// Four E4M3 bytes -> two f16x2 (bytes 0,1 -> lo; bytes 2,3 -> hi; lower byte -> lower half).
__device__ __forceinline__ void e4m3x4_to_f16x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\t"
      "mov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}
// Two fp32 -> two E4M3 (round to nearest even, saturating to +-448); a -> low byte.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
  return r;
}
// E8M0 scale byte -> 2^(e-127) as fp32 (e = 0 is the subnormal 2^-127, e = 255 NaN).
__device__ __forceinline__ float e8m0_to_f32(uint32_t e) {
  uint32_t bits = e ? (e << 23) : 0x00400000u;
  bits = (e == 255u) ? 0x7FC00000u : bits;
  return __uint_as_float(bits);
}

// 2^k as fp32 for |k| <= 126.
__device__ __forceinline__ float exp2i(int k) { return __uint_as_float(static_cast<uint32_t>(k + 127) << 23); }

// Mixed-precision multiply-add: one 16-bit half of each packed operand, product exact
// in fp32, one fp32 rounding (d = a * b + c).
__device__ __forceinline__ float fma_f16_lo(uint32_t a2, uint32_t b2, float c) {
  float d;
  asm("{\n\t.reg .f16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
      "fma.rn.f32.f16 %0, a0, b0, %3;\n\t}"
      : "=f"(d) : "r"(a2), "r"(b2), "f"(c));
  return d;
}
__device__ __forceinline__ float fma_f16_hi(uint32_t a2, uint32_t b2, float c) {
  float d;
  asm("{\n\t.reg .f16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
      "fma.rn.f32.f16 %0, a1, b1, %3;\n\t}"
      : "=f"(d) : "r"(a2), "r"(b2), "f"(c));
  return d;
}
__device__ __forceinline__ float fma_bf16_lo(uint32_t a2, uint32_t b2, float c) {
  float d;
  asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
      "fma.rn.f32.bf16 %0, a0, b0, %3;\n\t}"
      : "=f"(d) : "r"(a2), "r"(b2), "f"(c));
  return d;
}
__device__ __forceinline__ float fma_bf16_hi(uint32_t a2, uint32_t b2, float c) {
  float d;
  asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
      "fma.rn.f32.bf16 %0, a1, b1, %3;\n\t}"
      : "=f"(d) : "r"(a2), "r"(b2), "f"(c));
  return d;
}

// Power-of-two exponent p with amax * 2^p in [2^14, 2^15): moves a row into the
// f16 range without touching its significands.  0 for amax == 0 or not finite.
// Every positive finite fp32 amax gives p in [-113, 163].
__device__ __forceinline__ int f16_range_shift(float amax) {
  if (!(amax > 0.0f) || !(amax <= 3.4028235e38f)) return 0;
  int e;
  (void)frexpf(amax, &e);  // amax = f 2^e, f in [0.5, 1): floor(log2 amax) = e - 1
  return 14 - (e - 1);
}
// v * 2^k for |k| <= 252 as two exact power-of-two multiplications (each factor is a
// normal fp32 number): exact unless the result itself leaves the fp32 range.
__device__ __forceinline__ float mul_pow2(float v, int k) {
  const int k1 = k / 2;
  return (v * exp2i(k1)) * exp2i(k - k1);
}
// 2^d as fp32: exact for d in [-149, 127] (subnormal below -126), 0 below, 2^127 above.
__device__ __forceinline__ float pow2_clamped(int d) {
  if (d > 127) d = 127;
  if (d >= -126) return __uint_as_float(static_cast<uint32_t>(d + 127) << 23);
  return d >= -149 ? __uint_as_float(1u << (d + 149)) : 0.0f;
}

// ---------------------------------------------------------------------------
// Warp tensor-core products, D = A*B + C, m16n8k16, fp32 accumulate.
// Fragment ownership (g = lane/4, t = lane%4):
//   A: a0 (row g, k 2t..2t+1), a1 (row g+8, k 2t..2t+1), a2 (row g, k 2t+8..2t+9), a3 (row g+8, ...)
//   B: b0 (k 2t..2t+1, col g), b1 (k 2t+8..2t+9, col g)
//   C: c0 (row g, col 2t), c1 (row g, col 2t+1), c2 (row g+8, col 2t), c3 (row g+8, col 2t+1)
// ---------------------------------------------------------------------------
// Register-only instructions: not volatile, so the compiler may schedule the shared
// loads of the next products around them (worth ~17% in a one-tile microbenchmark).
__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 lds128(const void* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_u32(p)));
  return v;
}
__device__ __forceinline__ uint4 ldg128_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float silu_f32(float g) { return g / (1.0f + expf(-g)); }

// Orderable 32-bit key of a float: larger float -> larger key (NaN above +inf).
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

// Row stride (bytes) of a padded shared-memory row: the raw length rounded up so
// that consecutive rows start 16 banks apart (conflict-free 128-bit row reads).
__host__ __device__ __forceinline__ uint32_t padded_stride(uint32_t bytes) {
  uint32_t words = (bytes + 15u) / 16u * 4u;  // 16-byte granules, in words
  uint32_t m = words % 32u;
  words += (m <= 16u) ? (16u - m) : (48u - m);
  return words * 4u;
}

}  // namespace moe
