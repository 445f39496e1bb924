/*
 * nvfp4_linear.h -- C ABI of the NVFP4 weight-streaming linear for NVIDIA B200
 * (sm_100a).
 *
 * The operation. Y[M][N] = X[M][K] * W^T, where W[N][K] is stored as NVFP4:
 *   - 4-bit E2M1 codes, two per byte, element 2j of a row in the LOW nibble of
 *     byte j, rows contiguous: w_packed is uint8 [N][K/2];
 *   - one E4M3 ("fn") scale byte per 16 consecutive K elements of a row:
 *     w_scales is uint8 [N][K/16], row-major;
 *   - one fp32 per-tensor scale gs (device memory), so that
 *       w_hat[n][k] = e2m1(code[n][k]) * e4m3(scale[n][k/16]) * gs.
 * X and Y are bf16, row-major, M in [1, 16]: one decode token (M = 1) or one
 * token plus up to 15 drafted tokens checked in a single pass (M <= 16).
 *
 * Where the operation is defined. Page "Qwen3.8-27B-NVFP4-RTX5090 API &
 * Inference Endpoint": section "Recipe (NVIDIA ModelOpt)" (every Linear, the
 * output projection included, is NVFP4 with 16-element scale groups and a
 * per-tensor scale), section "Serving" (the codes are stored packed in uint8
 * tensors) and section "Why lm_head is NVFP4, and why MTP is gone" (decode is
 * bound by the weight read, so every byte saved is speed). Page "InventDB
 * Sparkle", section "How it answers quickly" (a helper model drafts several
 * tokens and the large model checks all of them in one pass: M = 1 + drafts).
 * The pages fix neither the nibble order nor the scale layout; the library
 * takes the readings stated above (low nibble first, plain row-major scales,
 * global scale multiplies).
 *
 * Numerics. Each w_hat/gs product e2m1 * e4m3 is exact in half precision; the
 * contraction accumulates in fp32 (tensor cores or CUDA cores, by variant);
 * the epilogue computes y = gs * acc in fp32 and rounds to bf16 (nearest even).
 * Per element |y - y_ref| <= 1e-2 |y_ref| + 1e-4 sum_k |w_hat x| against an
 * fp64 reference, for every X whose rows keep each nonzero element within
 * 2^57 of the row's largest magnitude. The tensor-core variants take X as
 * f16: each token row is scaled by a power of two (largest magnitude at
 * 2^14) and split into a hi plane and a lo plane (scaled by 2^29), which
 * together hold every such element exactly. An element further below its
 * row maximum keeps only the lo plane's subnormal step (absolute error at
 * most 2^-68 max_k |x[m][k]|), so for rows that hold one the bound above
 * gains the term 2^-67 max_k |x[m][k]| sum_k |w_hat[n][k]|. The CUDA-core
 * variant (GEMV) has no such range condition.
 *
 * Conventions.
 *   - Every buffer is device memory owned by the caller; the library makes
 *     no device allocation at run time. It holds one fixed array of
 *     NVFP4_STATIC_SCRATCH_BYTES per device where its device code is loaded
 *     (a __device__ variable, reserved when the module loads), used only by
 *     nvfp4_linear_run_static. A plan holds only launch parameters and
 *     cached TMA descriptors.
 *   - Calls that take a stream are asynchronous on it (a cudaStream_t passed
 *     as void*; NULL = legacy default stream), except nvfp4_linear_status,
 *     which synchronises that stream.
 *   - Argument errors are returned before anything is launched. Device-side
 *     timeouts of bounded waits are reported through the workspace status word
 *     and read by nvfp4_linear_status.
 *   - Limits: 1 <= M <= 16, N >= 0, K >= 0 with K % 256 == 0, every pointer
 *     16-byte aligned (gs: 4-byte aligned). N need not be a multiple of any
 *     tile size.
 *   - Thread safety: a plan's launch parameters are fixed at creation; the
 *     TMA descriptors it caches per buffer are updated under a lock, so a
 *     plan may be shared by threads. Runs on different streams may proceed
 *     concurrently if they use different workspaces.
 */
#ifndef NVFP4_LINEAR_H
#define NVFP4_LINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1,   /* a size, pointer or handle is invalid */
  NVFP4_ERR_UNSUPPORTED = 2,   /* shape/variant combination not supported */
  NVFP4_ERR_MISALIGNED = 3,    /* a pointer breaks the alignment rule */
  NVFP4_ERR_CUDA = 4,          /* a CUDA runtime call failed */
  NVFP4_ERR_TIMEOUT = 5,       /* a bounded device wait gave up (status word) */
  NVFP4_ERR_BAD_SCALE = 6,     /* reserved, never returned: the scale checks report counts */
  NVFP4_ERR_WORKSPACE = 7      /* workspace missing or smaller than required */
} nvfp4_status;

typedef struct nvfp4_plan_s* nvfp4_plan_t;

/* Kernel variants (plan flags, bits 0..3). AUTO takes the variant measured
 * fastest on B200 for the plan's (M, N, K), and TC for a shape the chosen
 * variant cannot take. */
#define NVFP4_VARIANT_AUTO 0u
#define NVFP4_VARIANT_GEMV 1u  /* CUDA-core warp-per-row GEMV, fp32 FMA        */
#define NVFP4_VARIANT_MMA  2u  /* TMA ring + warp MMA (m16n8k16), stream-K    */
#define NVFP4_VARIANT_TC   3u  /* tcgen05 + TMA ring + TMEM accumulators       */
#define NVFP4_VARIANT_ROW  4u  /* M <= 2: 16-row units taken dynamically, warp
                                  MMA with a block-diagonal X operand          */
#define NVFP4_PLAN_VARIANT_MASK 0xFu
/* Fused epilogues (plan flags, bits 8..11; variant MMA, which AUTO takes).
 * Page "SparkInfer" README, section "Layout & scoring", names fused FFN
 * kernels; page "Qwen3.8-27B-NVFP4-RTX5090 API & Inference Endpoint",
 * section "Why lm_head is NVFP4, and why MTP is gone", has the 248,320-row
 * output projection read for every token, and the greedy decode of page
 * "SparkInfer" README, section "DSpark speculative decode", needs only each
 * token's top logit.
 *   NVFP4_PLAN_EPI_SWIGLU: W is a fused gate+up projection whose rows 2c and
 *     2c+1 are the gate and up rows of output column c (N even). y is bf16
 *     [M][N/2]: y[m][c] = silu(g) * u with g, u the complete fp32 values
 *     gs * acc of rows 2c, 2c+1 and silu(v) = v / (1 + exp(-v)), rounded once
 *     to bf16.
 *   NVFP4_PLAN_EPI_ARGMAX: no logits are written. y receives int32 index [M]
 *     followed by float value [M] (8 M bytes): per token the row n with the
 *     largest fp32 value gs * acc[n] (not rounded to bf16), equal values
 *     going to the lower n. The plan's workspace holds the running maxima;
 *     it is left cleared after the run, like the counters. */
/* FP8 weight tier (plan flag; variant MMA without an epilogue, or ROW if
 * forced or if MMA cannot take the shape, M <= 2): W is stored as E4M3
 * codes, one byte per element, with one fp32 scale per row, for comparison
 * with NVFP4 at the same shapes (page "Qwen3.8-27B-NVFP4-RTX5090 API &
 * Inference Endpoint", section "Measured against the other NVFP4 builds of
 * this model": a weight format one step wider than NVFP4 is reported 1.5 to
 * 2.1 times slower on these shapes; page "InventDB Sparkle", section "How it
 * answers quickly": 8-bit weights). With this flag w_packed is uint8 [N][K] (E4M3 codes), w_scales
 * is float [N] and w_hat[n][k] = e4m3(code[n][k]) * w_scales[n] * gs; X, Y,
 * the tolerance and the X range are as for NVFP4. nvfp4_quantize_fp8 makes
 * such weights. */
#define NVFP4_PLAN_WEIGHT_FP8 0x1000u
/* W4A4 tier (plan flag; variants MMA and TC, any M): X arrives as bf16 like
 * always and is quantised to NVFP4 on the device with the weights'
 * quantiser steps -- 16-element blocks of a token row, E4M3 block scales,
 * one per-tensor scale gs_x = amax(|X|) / (6 * 448) of the call's X (page
 * "Qwen3.8-27B-NVFP4-RTX5090 API & Inference Endpoint", section "Recipe
 * (NVIDIA ModelOpt)": weights and activations NVFP4). Y is then sum_k
 * w_hat[n][k] * x_hat[m][k] with x_hat = e2m1 * e4m3 * gs_x: a different
 * (quantised) result from the W4A16 linear; the same tolerance, against the
 * fp64 sum of w_hat * x_hat, applies.
 *   MMA: codes decoded to f16 for the warp MMA; for M <= 4 every CTA
 *     quantises the K-steps it stages, from M = 5 the X-conversion kernel
 *     quantises X once per call. Takes the fused epilogues.
 *   TC: the block-scaled FP4 tensor cores (tcgen05.mma kind::mxf4nvf4) read
 *     the packed codes as stored and apply the block scales themselves; two
 *     small kernels quantise X first (3 launches per call). The scale bytes
 *     are read as unsigned E4M3: their sign bit must be clear (nvfp4_quantize
 *     never sets it). No fused epilogue.
 * AUTO takes TC from M = 4 without an epilogue (its time is flat in M) and
 * MMA otherwise, or MMA when TC cannot take the plan. GEMV, ROW and the FP8
 * weight tier return UNSUPPORTED. */
#define NVFP4_PLAN_ACT_NVFP4  0x2000u
#define NVFP4_PLAN_EPI_MASK   0xF00u
#define NVFP4_PLAN_EPI_SWIGLU 0x100u
#define NVFP4_PLAN_EPI_ARGMAX 0x200u
/* Programmatic dependent launch (MMA and ROW variants and W4A4 on TC;
 * ignored by the others). The launch may start while the previous kernel in the stream is
 * still running:
 * it begins streaming W at once and touches X, Y, w_global and the workspace
 * only after that kernel has completed. So W (codes and scales) must not be
 * written by the kernel launched just before it on the same stream. Back to
 * back calls then overlap one call's tail with the next call's weight stream. */
#define NVFP4_PLAN_PDL 0x10000u
/* Test only: the variant's producer never signals, so every bounded device
 * wait runs out and the kernel reports NVFP4_ERR_TIMEOUT through the status
 * word instead of computing. Has no effect on variants without device waits. */
#define NVFP4_PLAN_TEST_STALL 0x40000000u

/* Create a plan for Y[M][N] = X[M][K] W^T on `device`. Chooses the kernel
 * variant (or takes the one forced in `flags`), the split of K and the grid.
 * Returns INVALID_ARG for M outside [1,16], negative N/K, K % 256 != 0, an
 * unknown epilogue, SWIGLU with N odd, or a null `out`; UNSUPPORTED if a
 * forced variant cannot run this shape or epilogue; CUDA if the device cannot
 * be queried. On success *out must be released with nvfp4_linear_destroy. */
nvfp4_status nvfp4_linear_plan(int M, int N, int K, int device, unsigned flags,
                               nvfp4_plan_t* out);

/* Device workspace bytes nvfp4_linear_run needs for this plan (status word,
 * per-tile counters and fp32 partials of tiles computed in several pieces;
 * for the mma variant with M >= 5 also X converted to two f16 planes), 0 if
 * none. Zero-fill it once before first use: after every successful run its
 * status word and counters are zero again, so it can be reused without
 * clearing (the partial and X areas never need clearing). Two runs in flight
 * at the same time must not share a workspace. */
size_t nvfp4_linear_workspace_bytes(nvfp4_plan_t plan);

/* Chosen variant (NVFP4_VARIANT_*) and split-K factor of a plan; -1 if null. */
int nvfp4_linear_variant(nvfp4_plan_t plan);
int nvfp4_linear_split_k(nvfp4_plan_t plan);

/* The variant an AUTO plan of this shape starts from: the fastest measured
 * variant of the nearest shape in the library's table of per-variant times
 * on B200 (nearest: smallest 2 |log2 M - log2 Mt| + |log2 NK - log2 NtKt|,
 * the first such row on a tie). nvfp4_linear_plan then falls back to the
 * MMA variant, and from there to TC, if that variant cannot take the shape,
 * the epilogue or the weight format. -1 for M outside [1,16], negative N/K
 * or K % 256 != 0. Host-only; touches no device. */
int nvfp4_auto_variant(int M, int N, int K);

/* Kernels one nvfp4_linear_run (or nvfp4_linear_run_static) of this plan
 * launches: 2 for the mma variant when X goes through its ring (M >= 5, or a
 * K so long that X does not fit next to the ring: X is converted to its two
 * f16 planes by a kernel of its own first), 3 for a W4A4 plan on the TC
 * variant (X amax, X quantisation, the linear), 1 otherwise, 0 when N == 0;
 * -1 if the plan is null. Host-only; touches no device. */
int nvfp4_linear_launches_per_run(nvfp4_plan_t plan);

/* Run the linear on `stream` (device pointers, see the layout above):
 *   w_packed  uint8 [N][K/2]     w_scales uint8 [N][K/16] (E4M3)
 *   w_global  fp32 [1]           x        bf16 [M][K]
 *   y         bf16 [M][N], or as the plan's epilogue defines it
 *   workspace >= nvfp4_linear_workspace_bytes(plan) bytes (NULL if 0).
 * Must run on the plan's device (the current device). Returns INVALID_ARG
 * for a null plan or pointer, MISALIGNED for a pointer off its alignment,
 * WORKSPACE for a short workspace, CUDA if the launch fails. Y may not alias
 * any input. K == 0 writes zeros to Y; N == 0 launches nothing. */
nvfp4_status nvfp4_linear_run(nvfp4_plan_t plan, const uint8_t* w_packed,
                              const uint8_t* w_scales, const float* w_global,
                              const void* x, void* y, void* workspace,
                              size_t ws_bytes, void* stream);

/* Size of the fixed device scratch area behind nvfp4_linear_run_static. */
#define NVFP4_STATIC_SCRATCH_BYTES (16u << 20)

/* nvfp4_linear_run without a caller workspace and without allocating. The
 * pages define only the linear itself (as for nvfp4_linear_run); this entry
 * point has no counterpart there. It serves callers that cannot allocate
 * device memory at the point of the call: an engine that reserved nearly
 * all of HBM up front (weights, KV cache) and forbids allocation while
 * serving, a plain C host with no device allocator of its own, or a latency
 * path where cudaMalloc/cudaFree would stall (cudaFree synchronises the
 * device). The split-K scratch (status word, per-tile counters, partial
 * sums) lives instead in one fixed array of NVFP4_STATIC_SCRATCH_BYTES
 * inside the library, one per device.
 *   - Same arguments, layout and errors as nvfp4_linear_run, minus the
 *     workspace. Returns WORKSPACE, launching nothing, if the plan needs more
 *     than NVFP4_STATIC_SCRATCH_BYTES (nvfp4_linear_workspace_bytes).
 *   - status_out: optional device pointer (uint32, 4-byte aligned). After
 *     the kernel, the run's status word is copied there on `stream`: 0 if
 *     every device wait completed, nonzero if one timed out (then Y is
 *     unspecified). NULL skips the copy.
 *   - The first call on a device looks up the array's address with that
 *     device current, which may load the library's device code there; make
 *     that first call before any stream capture. The address is kept for
 *     the life of the process: after a cudaDeviceReset (or anything else
 *     that destroys the device's primary context) it is stale, and this
 *     entry point must not be called again on that device.
 *   - Every call on a device shares the one array and leaves the last call's
 *     contents in it; each call clears, on `stream`, the part that must start
 *     at zero (status word and counters). Calls on one stream are therefore
 *     ordered and safe; two calls that overlap in time on one device (other
 *     streams, other host threads) race on the array and give wrong results.
 *   - Allocates no memory: no cudaMalloc/cudaFree, no library allocator. */
nvfp4_status nvfp4_linear_run_static(nvfp4_plan_t plan, const uint8_t* w_packed,
                                     const uint8_t* w_scales, const float* w_global,
                                     const void* x, void* y, unsigned* status_out,
                                     void* stream);

/* Synchronise `stream`, then report: CUDA if the stream holds an error,
 * TIMEOUT if a kernel of this plan recorded a device-wait timeout in the
 * workspace status word (the word is cleared), else OK. workspace may be NULL
 * for plans whose workspace size is 0. */
nvfp4_status nvfp4_linear_status(nvfp4_plan_t plan, void* workspace, void* stream);

/* Release a plan (NULL is ignored). */
void nvfp4_linear_destroy(nvfp4_plan_t plan);

/* Unpack and scale-decode check. For every element writes the exact product
 * e2m1(code) * e4m3(scale) -- without the global scale -- as bf16 to
 * w_bf16_out [N][K] (nullable: then only counting is done), and adds to the
 * device counter *d_bad (uint32, caller-zeroed) the number of NaN scale codes
 * (0x7F, 0xFF) plus 1 if *w_global is NaN, infinite or negative. Values
 * produced from NaN scales are unspecified. Same alignment rules as run;
 * K % 16 == 0 suffices here. Asynchronous on `stream`. */
nvfp4_status nvfp4_pack_check(const uint8_t* w_packed, const uint8_t* w_scales,
                              const float* w_global, int N, int K,
                              void* w_bf16_out, unsigned* d_bad, void* stream);

/* Quantise fp32 W [N][K] (device) to NVFP4 with the recipe:
 *   gs = amax|W| / (6*448); per 16-element block s = E4M3_RNE_sat((amax_b/6)/gs);
 *   code = E2M1_RNE_sat(w / (e4m3(s) * gs)), codes of magnitude 0 stored as 0x0;
 *   a block whose e4m3(s)*gs is 0 gets all-zero codes.
 * Every step is one fp32 operation, in that order. Writes w_packed, w_scales
 * and *w_global (device). *d_bad (nullable, caller-zeroed) receives the
 * number of non-finite elements of W (the outputs are then unspecified).
 * K % 16 == 0; pointers 16-byte aligned. Three kernels on `stream`. */
nvfp4_status nvfp4_quantize(const float* w, int N, int K, uint8_t* w_packed,
                            uint8_t* w_scales, float* w_global, unsigned* d_bad,
                            void* stream);

/* FP8 weight tier quantiser: fp32 W [N][K] (device) -> E4M3 codes uint8
 * [N][K] and fp32 row scales [N]: s_n = amax |W[n]| / 448, code =
 * E4M3_RNE_satfinite(w / s_n), each step one fp32 operation; a row with
 * s_n = 0 gets all-zero codes, and a negative value that rounds to zero keeps
 * its sign (0x80). *d_bad (nullable, caller-zeroed) receives the number of
 * non-finite elements (the outputs are then unspecified). K % 16 == 0;
 * pointers 16-byte aligned. One kernel on `stream`. */
nvfp4_status nvfp4_quantize_fp8(const float* w, int N, int K, uint8_t* codes, float* row_scales,
                                unsigned* d_bad, void* stream);

/* Static text for a status code. */
const char* nvfp4_status_string(nvfp4_status s);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_LINEAR_H */
