// k_basic.cu -- the unpack/scale-decode check kernel and the GPU quantiser.
//
// Format: page "Qwen3.8-27B-NVFP4-RTX5090 API & Inference Endpoint", section
// "Recipe (NVIDIA ModelOpt)" (NVFP4, 16-element scale groups, per-tensor
// scale); section "Serving" (codes packed two per byte). Readings: low nibble
// first, scales row-major [N][K/16], w_hat = e2m1 * e4m3 * gs.
#include "kernels.h"
#include "nvfp4_device.cuh"

namespace nvfp4 {

// ---------------------------------------------------------------------------
// pack_check: one thread per 16-element block. Writes e2m1 * e4m3 (no global
// scale) as bf16 and counts NaN scale codes and a bad global scale.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
k_pack_check(const uint8_t* __restrict__ wp, const uint8_t* __restrict__ ws,
             const float* __restrict__ gsp, int64_t nblocks, uint16_t* __restrict__ out,
             unsigned* __restrict__ bad) {
  unsigned local_bad = 0;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    float g = *gsp;
    if (isnan(g) || isinf(g) || g < 0.0f) local_bad += 1;
  }
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t b = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; b < nblocks; b += stride) {
    const uint2 q = *reinterpret_cast<const uint2*>(wp + 8 * b);
    const uint32_t s = ws[b];
    if ((s & 0x7Fu) == 0x7Fu) local_bad += 1;
    if (out == nullptr) continue;
    const uint32_t sc = bcast_lo(e4m3x2_to_f16x2(s));
    uint32_t h[8];
    e2m1x8_to_f16x2x4(q.x, h);
    e2m1x8_to_f16x2x4(q.y, h + 4);
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 f = f16x2_to_float2(hmul2(h[i], sc));   // exact products
      __nv_bfloat162 bb = __floats2bfloat162_rn(f.x, f.y);  // exact conversion
      o[i] = *reinterpret_cast<uint32_t*>(&bb);
    }
    uint4* dst = reinterpret_cast<uint4*>(out + 16 * b);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
  // warp-aggregated count
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) local_bad += __shfl_xor_sync(0xffffffffu, local_bad, off);
  if ((threadIdx.x & 31) == 0 && local_bad && bad) atomicAdd(bad, local_bad);
}

cudaError_t launch_pack_check(const uint8_t* wp, const uint8_t* ws, const float* gs,
                              int64_t nblocks16, uint16_t* out, unsigned* bad, int num_sms,
                              cudaStream_t st) {
  int64_t want = (nblocks16 + 255) / 256;
  int grid = int(want < int64_t(num_sms) * 8 ? (want > 0 ? want : 1) : int64_t(num_sms) * 8);
  k_pack_check<<<grid, 256, 0, st>>>(wp, ws, gs, nblocks16, out, bad);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Quantiser. Step 1: amax of |W| into *gs (as uint bits; non-negative floats
// order like their bit patterns, NaN above +inf). Step 2: per block quantise
// with gs = amax / 2688. Step 3: *gs = amax / 2688.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
k_amax(const float* __restrict__ w, int64_t n, unsigned* __restrict__ amax_bits,
       unsigned* __restrict__ bad) {
  float m = 0.0f;
  unsigned nonfinite = 0;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  const int64_t n4 = n / 4;
  const float4* w4 = reinterpret_cast<const float4*>(w);
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 v = w4[i];
    float a[4] = {fabsf(v.x), fabsf(v.y), fabsf(v.z), fabsf(v.w)};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (!isfinite(a[j])) nonfinite += 1;
      m = __uint_as_float(max(__float_as_uint(m), __float_as_uint(a[j])));
    }
  }
  for (int64_t i = n4 * 4 + int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    float a = fabsf(w[i]);
    if (!isfinite(a)) nonfinite += 1;
    m = __uint_as_float(max(__float_as_uint(m), __float_as_uint(a)));
  }
  unsigned mb = __float_as_uint(m);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, off));
    nonfinite += __shfl_xor_sync(0xffffffffu, nonfinite, off);
  }
  if ((threadIdx.x & 31) == 0) {
    atomicMax(amax_bits, mb);
    if (nonfinite && bad) atomicAdd(bad, nonfinite);
  }
}

__global__ void __launch_bounds__(256)
k_quantize_blocks(const float* __restrict__ w, int64_t nblocks, const unsigned* __restrict__ amax_bits,
                  uint8_t* __restrict__ wp, uint8_t* __restrict__ ws) {
  const float amax = __uint_as_float(*amax_bits);
  const float gs = __fdiv_rn(amax, 2688.0f);   // 6 * 448
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t b = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; b < nblocks; b += stride) {
    const float4* src = reinterpret_cast<const float4*>(w + 16 * b);
    float v[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float4 t = src[i];
      v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
    }
    uint32_t s_code, packed[2];
    quantize_block16(v, gs, s_code, packed);
    *reinterpret_cast<uint2*>(wp + 8 * b) = make_uint2(packed[0], packed[1]);
    ws[b] = static_cast<uint8_t>(s_code);
  }
}

__global__ void k_quantize_finalize(float* gs) {
  const float amax = __uint_as_float(*reinterpret_cast<unsigned*>(gs));
  *gs = __fdiv_rn(amax, 2688.0f);
}

cudaError_t launch_quantize(const float* w, int64_t N, int64_t K, uint8_t* wp, uint8_t* ws,
                            float* gs, unsigned* bad, int num_sms, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(gs, 0, sizeof(float), st);
  if (e != cudaSuccess) return e;
  const int64_t n = N * K;
  if (n > 0) {
    int64_t want = (n / 4 + 255) / 256;
    int grid = int(want < int64_t(num_sms) * 8 ? (want > 0 ? want : 1) : int64_t(num_sms) * 8);
    k_amax<<<grid, 256, 0, st>>>(w, n, reinterpret_cast<unsigned*>(gs), bad);
    const int64_t nb = n / 16;
    want = (nb + 255) / 256;
    grid = int(want < int64_t(num_sms) * 16 ? (want > 0 ? want : 1) : int64_t(num_sms) * 16);
    k_quantize_blocks<<<grid, 256, 0, st>>>(w, nb, reinterpret_cast<const unsigned*>(gs), wp, ws);
  }
  k_quantize_finalize<<<1, 1, 0, st>>>(gs);
  return cudaGetLastError();
}

__global__ void k_zero_bf16(uint16_t* y, int64_t count) {
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < count; i += stride) y[i] = 0;
}

// ---------------------------------------------------------------------------
// FP8 weight tier quantiser: one warp per row. s_n = amax|W[n]| / 448 and
// code = E4M3_RNE_satfinite(w / s_n), each one fp32 operation; a row with
// s_n = 0 gets zero codes. Four elements per lane and step (K % 16 == 0).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e4m3x2_from_f32(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__global__ void __launch_bounds__(256)
k_quantize_fp8_rows(const float* __restrict__ w, int64_t N, int64_t K, uint8_t* __restrict__ codes,
                    float* __restrict__ row_scales, unsigned* __restrict__ bad) {
  const int lane = threadIdx.x & 31;
  const int64_t nw = int64_t(gridDim.x) * (blockDim.x >> 5);
  unsigned local_bad = 0;
  for (int64_t n = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); n < N; n += nw) {
    const float4* row = reinterpret_cast<const float4*>(w + n * K);
    float amax = 0.0f;
    for (int64_t c = lane; c < K / 4; c += 32) {
      const float4 v = row[c];
      const float a[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (!isfinite(a[i])) ++local_bad;
        amax = fmaxf(amax, fabsf(a[i]));
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float sn = amax / 448.0f;
    if (lane == 0) row_scales[n] = sn;
    uint32_t* out = reinterpret_cast<uint32_t*>(codes + n * K);
    for (int64_t c = lane; c < K / 4; c += 32) {
      uint32_t q = 0u;
      if (sn > 0.0f) {
        const float4 v = row[c];
        q = e4m3x2_from_f32(v.x / sn, v.y / sn) | (e4m3x2_from_f32(v.z / sn, v.w / sn) << 16);
      }
      out[c] = q;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) local_bad += __shfl_xor_sync(0xffffffffu, local_bad, off);
  if (lane == 0 && local_bad && bad) atomicAdd(bad, local_bad);
}

cudaError_t launch_quantize_fp8(const float* w, int64_t N, int64_t K, uint8_t* codes, float* row_scales,
                                unsigned* bad, int num_sms, cudaStream_t st) {
  if (N <= 0) return cudaSuccess;
  const int64_t want = (N + 7) / 8;                       // 8 rows (warps) per block
  const int grid = int(want < int64_t(num_sms) * 16 ? want : int64_t(num_sms) * 16);
  k_quantize_fp8_rows<<<grid, 256, 0, st>>>(w, N, K, codes, row_scales, bad);
  return cudaGetLastError();
}

cudaError_t launch_zero_bf16(uint16_t* y, int64_t count, cudaStream_t st) {
  if (count <= 0) return cudaSuccess;
  int64_t want = (count + 255) / 256;
  int grid = int(want < 1024 ? want : 1024);
  k_zero_bf16<<<grid, 256, 0, st>>>(y, count);
  return cudaGetLastError();
}

}  // namespace nvfp4
