// k_gemv.cu -- CUDA-core warp GEMV for the NVFP4 linear, small M.
//
// One warp owns one weight row at a time and walks it in 16-byte (32-element)
// chunks, lane l taking chunks l, l+32, ...; the four per-lane partial dot
// products are combined with __shfl_xor. X is staged once per CTA in shared
// memory as fp32 (bf16 -> fp32 is exact). Each 16-byte chunk is decoded
// to exact half-precision products e2m1 * e4m3 and accumulated in fp32 FMA.
// Epilogue: y = bf16_rne(gs * acc).
//
// The linear: page "InventDB Sparkle", section "How it answers quickly"
// (decode reads each weight once per token; M = 1 + drafted tokens); format:
// page "Qwen3.8-27B-NVFP4-RTX5090 API & Inference Endpoint", section "Recipe
// (NVIDIA ModelOpt)".
#include "kernels.h"
#include "nvfp4_device.cuh"

namespace nvfp4 {

namespace {

constexpr int kGemvWarps = 8;

// X[m][k] lives at xs[m*K + phys(k)], where 16-byte granules (4 floats) are
// XOR-swizzled inside groups of eight so that the eight lanes of a shared
// memory phase, which read the same granule slot of eight consecutive chunks,
// hit eight different bank quads.
__device__ __forceinline__ int x_phys(int k) {
  const int g = k >> 2;
  return (((g & ~7) | ((g ^ (g >> 3)) & 7)) << 2) | (k & 3);
}

template <int M>
__global__ void __launch_bounds__(kGemvWarps * 32)
k_gemv(const uint8_t* __restrict__ wp, const uint8_t* __restrict__ ws,
       const float* __restrict__ gsp, const uint16_t* __restrict__ x,
       uint16_t* __restrict__ y, int N, int K) {
  extern __shared__ float xs[];
  for (int i = threadIdx.x; i < M * K; i += blockDim.x) {
    const int m = i / K, k = i - m * K;
    xs[m * K + x_phys(k)] = bf16_bits_to_float(x[i]);
  }
  __syncthreads();
  const float gs = *gsp;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nchunks = K >> 5;
  for (int row = blockIdx.x * kGemvWarps + warp; row < N; row += gridDim.x * kGemvWarps) {
    const uint8_t* prow = wp + size_t(row) * size_t(K >> 1);
    const uint8_t* srow = ws + size_t(row) * size_t(K >> 4);
    float acc[M];
#pragma unroll
    for (int m = 0; m < M; ++m) acc[m] = 0.0f;
#pragma unroll 2
    for (int c = lane; c < nchunks; c += 32) {
      const uint4 q = ld_stream_v4(prow + 16 * c);
      const uint32_t s2 = ld_stream_u16(srow + 2 * c);
      const uint32_t sp = e4m3x2_to_f16x2(s2);
      const uint32_t sa = bcast_lo(sp), sb = bcast_hi(sp);
      const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int wi = 0; wi < 4; ++wi) {
        uint32_t h[4];
        e2m1x8_to_f16x2x4(words[wi], h);
        const uint32_t sc = (wi < 2) ? sa : sb;
        float wv[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = f16x2_to_float2(hmul2(h[j], sc));
          wv[2 * j] = f.x;
          wv[2 * j + 1] = f.y;
        }
        const int k0 = 32 * c + 8 * wi;
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const float4 xa = *reinterpret_cast<const float4*>(xs + m * K + x_phys(k0));
          const float4 xb = *reinterpret_cast<const float4*>(xs + m * K + x_phys(k0 + 4));
          acc[m] = fmaf(wv[0], xa.x, acc[m]);
          acc[m] = fmaf(wv[1], xa.y, acc[m]);
          acc[m] = fmaf(wv[2], xa.z, acc[m]);
          acc[m] = fmaf(wv[3], xa.w, acc[m]);
          acc[m] = fmaf(wv[4], xb.x, acc[m]);
          acc[m] = fmaf(wv[5], xb.y, acc[m]);
          acc[m] = fmaf(wv[6], xb.z, acc[m]);
          acc[m] = fmaf(wv[7], xb.w, acc[m]);
        }
      }
    }
#pragma unroll
    for (int m = 0; m < M; ++m) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], off);
    }
    if (lane == 0) {
#pragma unroll
      for (int m = 0; m < M; ++m) y[size_t(m) * N + row] = float_to_bf16_bits(gs * acc[m]);
    }
  }
}

template <int M>
cudaError_t launch_m(const GemvConfig& c, const uint8_t* wp, const uint8_t* ws, const float* gs,
                     const uint16_t* x, uint16_t* y, cudaStream_t st) {
  k_gemv<M><<<c.grid, c.block, c.smem, st>>>(wp, ws, gs, x, y, c.N, c.K);
  return cudaGetLastError();
}

template <int M>
cudaError_t config_m(GemvConfig& c, int num_sms) {
  // per-function attribute shared by all plans: raise it to the opt-in maximum
  int dev = 0, optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  if (c.smem > size_t(optin)) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(k_gemv<M>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_gemv<M>, c.block, c.smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int rows_per_cta = kGemvWarps;
  const int need = (c.N + rows_per_cta - 1) / rows_per_cta;
  const int cap = per_sm * num_sms;
  c.grid = need < cap ? (need > 0 ? need : 1) : cap;
  return cudaSuccess;
}

}  // namespace

cudaError_t gemv_configure(GemvConfig& c, int num_sms) {
  c.block = kGemvWarps * 32;
  c.smem = size_t(c.M) * size_t(c.K) * sizeof(float);
  switch (c.M) {
    case 1: return config_m<1>(c, num_sms);
    case 2: return config_m<2>(c, num_sms);
    case 3: return config_m<3>(c, num_sms);
    case 4: return config_m<4>(c, num_sms);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemv(const GemvConfig& c, const uint8_t* wp, const uint8_t* ws, const float* gs,
                        const uint16_t* x, uint16_t* y, cudaStream_t st) {
  switch (c.M) {
    case 1: return launch_m<1>(c, wp, ws, gs, x, y, st);
    case 2: return launch_m<2>(c, wp, ws, gs, x, y, st);
    case 3: return launch_m<3>(c, wp, ws, gs, x, y, st);
    case 4: return launch_m<4>(c, wp, ws, gs, x, y, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace nvfp4
