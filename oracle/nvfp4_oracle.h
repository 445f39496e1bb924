/*
 * nvfp4_oracle.h -- CPU reference ("oracle") for the NVFP4 weight-streaming linear.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or calls
 * this library: it is used by tests/, by the smoke check and by the CPU
 * baseline leg of the benchmark. It shares no code, header, table or helper
 * with the CUDA library under nvfp4_weight_streaming_b200/.
 *
 * What it computes (all host code, plain loops, fp64 where the result is
 * floating point):
 *
 *   - E2M1 and E4M3 decode/encode, written from the OCP 8-bit floating point
 *     specification (E4M3 "fn": bias 7, no infinities, 0x7F/0xFF = NaN, max 448)
 *     and the OCP Microscaling spec v1.0 (E2M1: bias 1, values
 *     {0, 0.5, 1, 1.5, 2, 3, 4, 6} and their negatives).
 *   - The NVFP4 weight quantiser: one E4M3 scale per 16 consecutive K elements
 *     and one fp32 per-tensor scale. Page "Qwen3.8-27B-NVFP4-RTX5090 API &
 *     Inference Endpoint", section "Recipe (NVIDIA ModelOpt)": weights are
 *     NVFP4 with 16-element scale groups; section "Serving": the checkpoint
 *     keeps the 4-bit codes packed two to a byte (uint8 tensors).
 *   - The reference linear Y[M,N] = X[M,K] * W^T with W dequantised exactly and
 *     the sum accumulated in fp64. Page "InventDB Sparkle", section "How it
 *     answers quickly" (decode reads every weight once per token; the
 *     guess-and-check scheme verifies several drafted tokens in one pass, so
 *     M = 1..16).
 *   - Two epilogues of that linear: the SiLU-gated output of a fused gate+up
 *     projection (page "SparkInfer" README, section "Layout & scoring": the
 *     engine's FFN kernels are fused; page "Qwen3.8-27B-NVFP4-RTX5090 API &
 *     Inference Endpoint", section "Recipe (NVIDIA ModelOpt)": the MLP is
 *     NVFP4), and the greedy argmax / top-k of the logits (page "SparkInfer"
 *     README, section "DSpark speculative decode": greedy decoding; page
 *     "Qwen3.8-27B-NVFP4-RTX5090 API & Inference Endpoint", section
 *     "SparkInfer + DSpark": a verify pass keeps a drafted token only where it
 *     equals the target's own choice, and near ties at the top can flip).
 *   - Two more tiers of the same linear: W4A4, where X is NVFP4 too (page
 *     "Qwen3.8-27B-NVFP4-RTX5090 API & Inference Endpoint", section "Recipe
 *     (NVIDIA ModelOpt)": weights and activations NVFP4 W4A4, group size 16,
 *     with a per-layer input scale), and 8-bit E4M3 weights as the comparison
 *     tier (page "InventDB Sparkle", section "How it answers quickly": 8-bit
 *     weights; same model card, section "Measured against the other NVFP4
 *     builds of this model": the FP8 tier costs 1.5-2.1x on these shapes).
 *
 * Readings taken where the pages are silent (each is also stated where it is used):
 *   R1 nibble order: element 2j of a row is the low nibble of byte j.
 *   R2 layouts: W packed [N][K/2] row-major, scales [N][K/16] row-major.
 *   R3 global scale multiplies: w_hat = e2m1(q) * e4m3(s) * gs, gs = amax/(6*448).
 *   R4 rounding: round-to-nearest-even with saturation to the largest finite
 *      value (448 for E4M3, 6 for E2M1).
 *   R5 a block whose decoded scale times gs is 0 gets all-zero codes.
 *   R6 values that round to zero get code 0x0, never 0x8.
 *   R7 every quantiser step is an fp32 operation in the order written in
 *      ora_quantize (the decisions are taken on fp32 values).
 *   R10 an argmax or top-k tie goes to the lowest index.
 *   R11 a fused gate+up projection interleaves its rows: row 2c is the gate
 *      and row 2c+1 the up row of output column c; the gated output is
 *      silu(gate) * up (the SiLU-gated MLP of the model family).
 *   R14 W4A4: activations are NVFP4 like the weights (16-element blocks of a
 *      token row, E4M3 block scales) under their own per-tensor scale, which
 *      the caller gives (a calibrated input scale; synthetic inputs use
 *      amax(|X|)/(6*448) of the call's X); the same quantiser steps as W.
 *   R15 FP8 weight tier: E4M3 codes with one fp32 scale per output row,
 *      s_n = amax(|W[n]|)/448.
 *
 * Parity pins: every function here is pinned by tests under tests/ that do not
 * call back into the same code path (exhaustive tables, brute force, closed
 * forms, library conversions, the pages' printed sizes). See the test files.
 */
#ifndef NVFP4_ORACLE_H
#define NVFP4_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Host threads the row-parallel functions (quantiser, linears) use for n rows
 * when given nthreads: 1 below 4096 rows, else the number of non-empty
 * contiguous pieces. */
int ora_threads_for(int64_t n, int nthreads);

/* Value of an E2M1 code (low 4 bits used). Code 0x8 decodes to -0.0. */
double ora_e2m1_decode(uint32_t code);
/* Value of an E4M3 ("fn") byte. 0x7F and 0xFF decode to NaN. */
double ora_e4m3_decode(uint32_t code);
/* 1 if the E4M3 byte is a NaN code (0x7F or 0xFF), else 0. */
int ora_e4m3_is_nan(uint32_t code);
/* Nearest E2M1 code to r, ties to the even code, saturating at +-6.
 * Results of magnitude 0 are returned as code 0 (reading R6). NaN -> 0. */
uint32_t ora_e2m1_encode(float r);
/* Nearest E4M3 byte to u, ties to the even code, saturating at +-448.
 * NaN -> 0x7F. A negative value rounding to zero keeps its sign (0x80). */
uint32_t ora_e4m3_encode(float u);

/* Per-tensor scale gs = amax(|W|) / (6*448), one fp32 division. Returns 0 on
 * success, -2 if W holds a non-finite value. n may be 0 (gs = 0). */
int ora_global_scale(const float* w, int64_t n, float* gs, int nthreads);

/* Quantise rows of W (fp32 [nrows][K], K % 16 == 0) under a given global
 * scale: packed [nrows][K/2], scales [nrows][K/16]. Returns 0, or -1 on bad
 * arguments. */
int ora_quantize_rows(const float* w, int64_t nrows, int64_t K, float gs,
                      uint8_t* packed, uint8_t* scales, int nthreads);

/* Full quantiser: gs from the whole tensor, then ora_quantize_rows. Returns 0,
 * -1 on bad arguments, -2 if W is not finite. */
int ora_quantize(const float* w, int64_t N, int64_t K, uint8_t* packed,
                 uint8_t* scales, float* gs, int nthreads);

/* Dequantised weight including the global scale, fp64 [N][K]. */
int ora_dequant_f64(const uint8_t* packed, const uint8_t* scales, float gs,
                    int64_t N, int64_t K, double* out);

/* Exact product e2m1(code) * e4m3(scale), WITHOUT the global scale, as a bf16
 * bit pattern [N][K] (the product always fits bf16; NaN scales give 0x7FC0). */
int ora_dequant_bf16_nogs(const uint8_t* packed, const uint8_t* scales,
                          int64_t N, int64_t K, uint16_t* out);

/* Number of NaN scale codes in scales[n_scales], plus 1 if gs is NaN, infinite
 * or negative. */
int64_t ora_count_bad(const uint8_t* scales, int64_t n_scales, float gs);

/* Reference linear. x_bf16 is [M][K] bf16 bit patterns. Output rows are the
 * weight rows listed in rows[0..nrows) (rows == NULL means 0..N-1 and nrows
 * must equal N). y[m*nrows + i] = sum_k w_hat[rows[i]][k] * x[m][k] in fp64;
 * absdot (nullable) gets sum_k |w_hat * x| for the tolerance bound. */
int ora_linear(const uint8_t* packed, const uint8_t* scales, float gs,
               const uint16_t* x_bf16, int64_t M, int64_t N, int64_t K,
               const int64_t* rows, int64_t nrows, double* y, double* absdot,
               int nthreads);

/* SiLU(v) = v * sigmoid(v) = v / (1 + exp(-v)), fp64. */
double ora_silu(double v);

/* Gated (SwiGLU) output of a fused gate+up projection W [N2][K], N2 even.
 * Reading R11: rows 2c and 2c+1 of W are the gate and up rows of output column
 * c. For the columns listed in cols[0..ncols) (NULL means 0..N2/2-1 and ncols
 * must equal N2/2):
 *   gate[m][i] = sum_k w_hat[2c][k] x[m][k],  up[m][i] = sum_k w_hat[2c+1][k] x[m][k]
 *   h[m][i]    = silu(gate[m][i]) * up[m][i]            (all fp64, c = cols[i])
 * gate, up and the absdot sums of each (for the tolerance bound) are nullable
 * outputs, each [M][ncols]. Returns 0, or -1 on bad arguments. */
int ora_swiglu_linear(const uint8_t* packed, const uint8_t* scales, float gs,
                      const uint16_t* x_bf16, int64_t M, int64_t N2, int64_t K,
                      const int64_t* cols, int64_t ncols, double* h, double* gate,
                      double* up, double* absdot_gate, double* absdot_up, int nthreads);

/* Indices of the k largest entries of each row of y [M][N], largest first,
 * equal values by ascending index (reading R10); idx is [M][k]. k = 1 is the
 * greedy argmax. Returns 0, -1 on bad arguments, -3 if y holds a NaN. */
int ora_topk(const double* y, int64_t M, int64_t N, int64_t k, int64_t* idx);

/* W4A4 reference linear (reading R14): X is NVFP4 too, given as x_packed
 * [M][K/2], x_scales [M][K/16] and its per-tensor scale gs_x (quantise it with
 * ora_quantize_rows under that scale). y[m*nrows + i] = sum_k w_hat[rows[i]][k]
 * * x_hat[m][k] in fp64, both operands dequantised exactly; absdot nullable.
 * Row selection as in ora_linear. Returns 0, or -1 on bad arguments. */
int ora_linear_w4a4(const uint8_t* w_packed, const uint8_t* w_scales, float gs_w,
                    const uint8_t* x_packed, const uint8_t* x_scales, float gs_x,
                    int64_t M, int64_t N, int64_t K, const int64_t* rows, int64_t nrows,
                    double* y, double* absdot, int nthreads);

/* FP8 weight tier (reading R15): per output row n, s_n = amax(|W[n]|)/448 in
 * fp32 and codes[n][k] = E4M3(w[n][k] / s_n) (RNE, saturating; the sign of a
 * negative value that rounds to zero is kept, 0x80); s_n = 0 gives zero codes.
 * codes is uint8 [N][K], row_scales fp32 [N]. Returns 0, -1 on bad arguments,
 * -2 if W is not finite. */
int ora_quantize_fp8_rows(const float* w, int64_t N, int64_t K, uint8_t* codes,
                          float* row_scales, int nthreads);

/* FP8 weight tier reference linear: y[m*nrows + i] = sum_k e4m3(codes[n][k])
 * * s_n * x[m][k] in fp64 (n = rows[i]); absdot nullable; rows as in
 * ora_linear. Returns 0, or -1 on bad arguments. */
int ora_linear_fp8(const uint8_t* codes, const float* row_scales, const uint16_t* x_bf16,
                   int64_t M, int64_t N, int64_t K, const int64_t* rows, int64_t nrows,
                   double* y, double* absdot, int nthreads);

/* Round an fp64 value to bf16 (round to nearest even, overflow to inf), as bits. */
uint16_t ora_bf16_rne(double v);
/* Value of a bf16 bit pattern. */
double ora_bf16_value(uint16_t bits);

/* Bytes one call moves: N*K/2 + N*K/16 + 2*M*K + 2*M*N. */
double ora_bytes_model(int64_t M, int64_t N, int64_t K);

#ifdef __cplusplus
}
#endif

#endif
