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
#include <climits>

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

// E4M3 round-to-nearest-even with saturation (hardware conversion); the
// result's low byte is the code of `u`.
__device__ __forceinline__ uint32_t e4m3_rne_sat(float u) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(u));
  return r & 0xFFu;
}

// Two E2M1 codes (RNE, saturating): `lo` in bits 0..3, `hi` in bits 4..7.
// A code of magnitude 0 is stored as 0x0 (no negative zero).
__device__ __forceinline__ uint32_t e2m1x2_rne_sat(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r) : "f"(hi), "f"(lo));
  if ((r & 0x07u) == 0) r &= 0xF0u;
  if ((r & 0x70u) == 0) r &= 0x0Fu;
  return r;
}


// One 16-element block of the NVFP4 quantiser under the per-tensor scale gs:
// s = E4M3_RNE_satfinite((amax_b / 6) / gs), codes = E2M1_RNE_satfinite(v /
// (e4m3(s) * gs)), each an fp32 operation in that order (all codes zero when
// e4m3(s) * gs is 0). packed: element 2j in the low nibble of byte j.
__device__ __forceinline__ void quantize_block16(const float v[16], float gs, uint32_t& s_code,
                                                 uint32_t packed[2]) {
  float amax_b = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax_b = fmaxf(amax_b, fabsf(v[i]));
  const float t = __fdiv_rn(amax_b, 6.0f);
  const float u = (gs > 0.0f) ? __fdiv_rn(t, gs) : 0.0f;
  s_code = e4m3_rne_sat(u);
  const float ds = __half2float(__ushort_as_half(
      static_cast<unsigned short>(e4m3x2_to_f16x2(s_code) & 0xFFFFu)));
  const float denom = __fmul_rn(ds, gs);
  packed[0] = packed[1] = 0u;
  if (denom > 0.0f) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t byte = e2m1x2_rne_sat(__fdiv_rn(v[2 * j], denom), __fdiv_rn(v[2 * j + 1], denom));
      packed[j / 4] |= byte << (8 * (j % 4));
    }
  }
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
// 3D tiled TMA load with an L2 cache policy.
__device__ __forceinline__ void tma_load_3d_hint(uint32_t dst, const void* tmap, int x, int y, int z,
                                                 uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;"
      ::"r"(dst), "l"(tmap), "r"(x), "r"(y), "r"(z), "r"(bar), "l"(policy) : "memory");
}
// Untiled bulk copy global -> shared (both addresses 16-byte aligned, size a
// multiple of 16 bytes), completing on an mbarrier.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
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
// f16 bits of sign * sig/128 * 2^t, sig in [128, 255], t <= 15, rounded to
// nearest even: exact for a normal exponent (t >= -14: 8 significant bits fit
// the 11 of f16); below that the value is a multiple of the subnormal step
// 2^-24 after rounding, sig * 2^(t + 17) steps (0 once that is below a half).
__device__ __forceinline__ uint32_t make_f16_rn(uint32_t sign, int t, uint32_t sig) {
  if (t >= -14) return make_f16(sign, t, sig);
  const int sh = t + 17;                       // <= 2
  uint32_t q;
  if (sh >= 0) {
    q = sig << sh;                             // <= 1020: a subnormal mantissa
  } else {
    const int n = -sh;
    if (n > 9) return sign << 15;              // sig / 2^n < 1/2
    const uint32_t half = 1u << (n - 1), rest = sig & ((1u << n) - 1u);
    q = sig >> n;
    if (rest > half || (rest == half && (q & 1u))) ++q;
  }
  return (sign << 15) | q;
}

// Power of two between the hi and the lo f16 plane of X.
constexpr int X_LO_SHIFT = 29;

// Largest bf16 magnitude (bits, sign cleared) among the eight values of a
// 16-byte chunk, with one packed 16-bit max per pair.
__device__ __forceinline__ uint32_t bf16_mag_max8(const uint4& v) {
  const uint32_t m = __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                              __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
  return max(m & 0xFFFFu, m >> 16);
}

// Exponent floor(log2 |x|) of the bf16 magnitude `mag`; INT_MIN for zero.
__device__ __forceinline__ int bf16_mag_exp(uint32_t mag) {
  if (mag == 0u) return INT_MIN;
  const uint32_t e8 = mag >> 7;
  if (e8) return int(e8) - 127;
  return (31 - __clz(int(mag & 0x7Fu))) - 133;     // subnormal
}

// Two bf16 values (one word) -> their hi f16 pair and lo f16 pair for the
// token's shift: x * 2^sh (exact: the scale is applied as two powers of two
// f1 * f2) rounded to f16 is the hi plane (exact for |x * 2^sh| >= 2^-14:
// 8 significant bits), the exact remainder scaled by 2^X_LO_SHIFT is the lo
// plane. Returns the lo pair.
__device__ __forceinline__ uint32_t x_split2(uint32_t w, float f1, float f2, uint32_t& hi) {
  const float s0 = (__uint_as_float(w << 16) * f1) * f2;
  const float s1 = (__uint_as_float(w & 0xFFFF0000u) * f1) * f2;
  const __half2 h = __floats2half2_rn(s0, s1);       // low half = element 0
  hi = *reinterpret_cast<const uint32_t*>(&h);
  const float2 hb = __half22float2(h);
  constexpr float kLo = 536870912.0f;                 // 2^X_LO_SHIFT
  const __half2 l = __floats2half2_rn((s0 - hb.x) * kLo, (s1 - hb.y) * kLo);
  return *reinterpret_cast<const uint32_t*>(&l);
}

// Eight bf16 values (four words) -> hi and lo planes for the token's shift
// sh (largest magnitude at 2^14); returns whether any lo element is nonzero.
__device__ __forceinline__ bool x_split8(const uint32_t w[4], int sh, uint32_t hi[4], uint32_t lo[4]) {
  static_assert(X_LO_SHIFT == 29, "kLo above is 2^29");
  const float f1 = __int_as_float((127 + sh / 2) << 23), f2 = __int_as_float((127 + sh - sh / 2) << 23);
  uint32_t any = 0u;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    lo[q] = x_split2(w[q], f1, f2, hi[q]);
    any |= lo[q] & 0x7FFF7FFFu;
  }
  return any != 0u;
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
