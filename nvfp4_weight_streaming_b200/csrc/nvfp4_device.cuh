// nvfp4_device.cuh -- device helpers shared by the NVFP4 kernels (sm_100a).
//
// Decode. An NVFP4 element is an E2M1 code (OCP MX v1.0: values 0, 0.5, 1,
// 1.5, 2, 3, 4, 6 and negatives) times its block's E4M3 scale. Both factors,
// and their product (at most 6 significant bits, magnitude in [2^-10, 2688]),
// are exact in IEEE half precision, so the hardware conversions
// cvt.rn.f16x2.e2m1x2 / cvt.rn.f16x2.e4m3x2 followed by one packed f16
// multiply give the dequantised weight (without the global scale) exactly.
// Element 2j of a row is the low nibble of byte j; the conversion puts the
// low nibble in the low half of the f16x2 result.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

namespace nvfp4 {

// Four bytes (eight E2M1 codes) -> four f16x2, in element order.
__device__ __forceinline__ void e2m1x8_to_f16x2x4(uint32_t w, uint32_t out[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
      : "r"(w));
}

// Two E4M3 bytes (low byte first) -> f16x2 (low byte in the low half), exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_bytes) {
  uint32_t r;
  uint16_t h = static_cast<uint16_t>(two_bytes);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(h));
  return r;
}

// f16x2 with both halves equal to the low / high half of v.
__device__ __forceinline__ uint32_t bcast_lo(uint32_t v) { return __byte_perm(v, 0, 0x1010); }
__device__ __forceinline__ uint32_t bcast_hi(uint32_t v) { return __byte_perm(v, 0, 0x3232); }

// Packed f16 multiply, round to nearest (exact for the NVFP4 products).
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ float2 f16x2_to_float2(uint32_t v) {
  __half2 h = *reinterpret_cast<__half2*>(&v);
  return __half22float2(h);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

// Streaming 16-byte load: read once, do not keep in L1.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t ld_stream_u32(const void* p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t ld_stream_u16(const void* p) {
  uint16_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(r) : "l"(p));
  return r;
}

// ---- shared memory barriers and TMA ----------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(b), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(b) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(b), "r"(bytes)
               : "memory");
}
// Non-blocking-forever probe of an mbarrier phase (the hardware may suspend
// the thread for a bounded time inside try_wait).
__device__ __forceinline__ bool mbar_test(uint32_t b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(b), "r"(parity) : "memory");
  return ok != 0;
}
// Same probe, but the thread may sleep in hardware until the phase completes
// or about `hint_ns` nanoseconds pass, instead of spinning on the barrier.
__device__ __forceinline__ bool mbar_wait_hint(uint32_t b, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(b), "r"(parity), "r"(hint_ns) : "memory");
  return ok != 0;
}
// 2D tiled TMA load into shared memory, completing on an mbarrier.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(tmap), "r"(x), "r"(y), "r"(bar) : "memory");
}
// L2 policy for data read once: evict first, so a weight stream does not
// push small, reused buffers (activations, counters, partial sums) out of L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// 2D tiled TMA load with an L2 cache policy.
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const void* tmap, int x, int y,
                                                 uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;"
      ::"r"(dst), "l"(tmap), "r"(x), "r"(y), "r"(bar), "l"(policy) : "memory");
}
__device__ __forceinline__ void named_bar(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// bar.red.and over `count` threads: every participant gets the AND of `ok`.
__device__ __forceinline__ bool named_bar_and(int id, int count, bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r) : "r"(ok ? 1u : 0u), "r"(id), "r"(count) : "memory");
  return r != 0;
}
// ---- X as f16 planes ------------------------------------------------------------
// Exponent of a nonzero finite bf16 value and its 8-bit significand (128..255).
__device__ __forceinline__ int bf16_exp(uint32_t b, uint32_t& sig) {
  const uint32_t e8 = (b >> 7) & 0xFFu, mant = b & 0x7Fu;
  if (e8) { sig = 0x80u | mant; return int(e8) - 127; }
  const int msb = 31 - __clz(int(mant));
  sig = mant << (7 - msb);
  return msb - 133;
}
// f16 bits of sign * sig/128 * 2^t for a normal f16 exponent t (else 0).
__device__ __forceinline__ uint32_t make_f16(uint32_t sign, int t, uint32_t sig) {
  if (t < -14 || t > 15) return 0;
  return (sign << 15) | (uint32_t(t + 15) << 10) | ((sig & 0x7Fu) << 3);
}

// Number of work-range boundaries floor(c * L / W), c in [1, W), lying in (lo, hi].
__device__ __forceinline__ long long boundaries_in(long long lo, long long hi, long long L, long long W) {
  if (hi <= lo) return 0;
  long long cmin = ((lo + 1) * W + L - 1) / L;
  long long cmax = ((hi + 1) * W + L - 1) / L - 1;
  if (cmin < 1) cmin = 1;
  if (cmax > W - 1) cmax = W - 1;
  return cmax >= cmin ? cmax - cmin + 1 : 0;
}

}  // namespace nvfp4
