// kernels.h -- host-side launch interface between the C ABI (api.cu) and the
// kernel translation units. Internal to the library.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

namespace nvfp4 {

// Unpack + scale-decode check (k_basic.cu).
cudaError_t launch_pack_check(const uint8_t* wp, const uint8_t* ws, const float* gs,
                              int64_t nblocks16, uint16_t* out, unsigned* bad,
                              int num_sms, cudaStream_t st);

// GPU quantiser: amax, per-block quantise, finalise gs (k_basic.cu).
cudaError_t launch_quantize(const float* w, int64_t N, int64_t K, uint8_t* wp, uint8_t* ws,
                            float* gs, unsigned* bad, int num_sms, cudaStream_t st);

// FP8 tier quantiser: per-row scale amax / 448, E4M3 codes (k_basic.cu).
cudaError_t launch_quantize_fp8(const float* w, int64_t N, int64_t K, uint8_t* codes, float* row_scales,
                                unsigned* bad, int num_sms, cudaStream_t st);

// Zero-fill Y (K == 0).
cudaError_t launch_zero_bf16(uint16_t* y, int64_t count, cudaStream_t st);

// CUDA-core warp GEMV (k_gemv.cu). smem_bytes = M*K*4.
struct GemvConfig {
  int M, N, K;
  int grid, block;
  size_t smem;
};
cudaError_t gemv_configure(GemvConfig& c, int num_sms);
cudaError_t launch_gemv(const GemvConfig& c, const uint8_t* wp, const uint8_t* ws,
                        const float* gs, const uint16_t* x, uint16_t* y, cudaStream_t st);

// tcgen05 tensor-core variant (k_tc.cu).
struct TcConfig {
  int M, N, K;
  int tiles, S, P, ks_base, ks_rem, nb, xk_max, pmax, grid;
  bool split;
  size_t smem, ws_counters_off, ws_partials_off, ws_bytes;
};
cudaError_t tc_configure(TcConfig& c, int num_sms);
// Encode the TMA descriptors (CUtensorMap, 128 bytes each) of one weight set:
// codes in boxes of 128 bytes x box_rows rows (128-byte swizzle), scales in
// boxes of 16 bytes x box_rows rows.
bool encode_weight_maps(int N, int K, int box_rows, const uint8_t* wp, const uint8_t* ws,
                        void* map_w, void* map_s);
bool tensor_maps_supported();
// TMA descriptor of the f16 X planes the mma variant keeps in its workspace.
bool encode_x_planes_map(const void* planes, int pitch_bytes, int cols, int box_bytes, void* map);
cudaError_t launch_tc(const TcConfig& c, const void* map_w, const void* map_s, const float* gs,
                      const uint16_t* x, uint16_t* y, void* workspace, long long timeout_cycles,
                      bool stall, cudaStream_t st);

// W4A4 on the block-scaled FP4 tensor cores (k_tc4.cu): X quantised to NVFP4
// once per call into the workspace, tcgen05.mma kind::mxf4nvf4 on the raw
// codes with the E4M3 block scales in tensor memory. Three launches per call.
struct Tc4Config {
  int M, N, K;
  int tiles, S, ks_base, ks_rem, units, grid;
  size_t smem, ws_amax_off, ws_gsx_off, ws_counters_off, ws_x_off, ws_partials_off, ws_bytes;
};
cudaError_t tc4_configure(Tc4Config& c, int num_sms);
// map_w / map_s: encode_weight_maps with 256-row boxes.
cudaError_t launch_tc4(const Tc4Config& c, const void* map_w, const void* map_s, const float* gs,
                       const uint16_t* x, uint16_t* y, void* workspace, long long timeout_cycles, bool stall,
                       bool pdl, cudaStream_t st);

// Register-direct warp-MMA variant (k_mma.cu).
struct MmaConfig {
  int M, N, K;
  int epi;   // 0: Y; 1: SiLU-gated pairs of rows; 2: per-token argmax (k_mma.cu)
  int tiles, S, P, ks_base, ks_rem, ncols, xk_max, xstride, pmax, nstage, grid;
  int tpc;   // whole tiles per CTA (no split tiles), 0: stream-K
  int act4;  // W4A4: X quantised to NVFP4 inside the kernel (staged X only)
  int fmt;   // 0: NVFP4 weights; 1: FP8 weights (E4M3 codes [N][K], fp32 row scales [N]; M <= 4, staged X)
  bool split;
  // X in the ring (M > 4): X planes prepared once per call in the workspace
  bool xr;
  int x_pitch, x_box, xbytes;
  int xchunks;   // X-conversion blocks per token (grid M x xchunks)
  size_t ws_x_off, ws_xmeta_off;
  size_t smem, ws_counters_off, ws_epi_off, ws_partials_off, ws_bytes;
};
cudaError_t mma_configure(MmaConfig& c, int num_sms);
// map_x: descriptor of the X planes in `workspace` (encode_x_planes_map), used when c.xr.
cudaError_t launch_mma(const MmaConfig& c, const void* map_w, const void* map_s, const void* map_x,
                       const float* gs, const float* row_scale, const uint16_t* x, uint16_t* y,
                       void* workspace, long long timeout_cycles, bool stall, bool pdl, cudaStream_t st);
// FP8 weight tier codes map for the MMA variant.
bool encode_fp8_codes_map(int N, int K, const uint8_t* wp, void* map_w);
constexpr int kMmaTileRows = 256;

// The driver's cuTensorMapEncodeTiled (null if unavailable); k_tc.cu.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// Row-block streaming variant, M <= 2 (k_row.cu): 16-row x K-slice units
// taken dynamically, block-diagonal B operand, X converted and kept in
// shared memory by every CTA.
struct RowConfig {
  int M, N, K;
  int fmt;   // 0: NVFP4 weights; 1: FP8 weights (E4M3 codes [N][K], fp32 row scales [N])
  int units16, KS, units, IT, ipu, nst, xstride, sp_row, grid;
  size_t smem, ws_counters_off, ws_gcnt_off, ws_partials_off, ws_bytes;
};
cudaError_t row_configure(RowConfig& c, int num_sms);
// TMA descriptors of one weight set for this variant: one box per unit of 16
// rows x `ipu` 512-element items (codes with the 128-byte swizzle, scales).
bool encode_row_maps(int N, int K, int ipu, int fmt, const uint8_t* wp, const uint8_t* ws, void* map_w,
                     void* map_s);
// One launch.
cudaError_t launch_row(const RowConfig& c, const void* map_w, const void* map_s, const float* row_scale,
                       const float* gs, const uint16_t* x, uint16_t* y, void* workspace,
                       long long timeout_cycles, bool stall, bool pdl, cudaStream_t st);

}  // namespace nvfp4
