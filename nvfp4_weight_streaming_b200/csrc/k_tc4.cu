// k_tc4.cu -- W4A4 linear on the block-scaled FP4 tensor cores (sm_100a).
//
// Y[M][N] = gs_w * gs_x * sum_k (e2m1_w * s_w) * (e2m1_x * s_x) with W and X
// both in NVFP4: E2M1 codes, one E4M3 scale per 16 consecutive K elements,
// one fp32 scale per tensor (page "Qwen3.8-27B-NVFP4-RTX5090 API & Inference
// Endpoint", section "Recipe (NVIDIA ModelOpt)": W4A4, group size 16, a
// per-layer input scale). X is quantised per call: gs_x = amax(|X|) / (6 *
// 448), blocks by the weights' quantiser steps.
//
// tcgen05.mma kind::mxf4nvf4 multiplies packed E2M1 operands read straight
// from shared memory and applies the 16-element E4M3 block scales from tensor
// memory, so nothing is decoded: the weight stream goes from HBM to the
// tensor core as stored. Swap-AB: the MMA's 128-row dimension is weight rows,
// its N dimension the tokens (1 + drafted tokens, padded to 16; page
// "InventDB Sparkle", section "How it answers quickly").
//
// Per call three launches, chained by programmatic dependent launch:
//   k_x4_amax   amax(|X|) over the whole call's X (atomic max of bit patterns).
//   k_x4_quant  one CTA per 256-element K-step: the 16 token rows quantised to
//               E2M1 codes in the MMA's 128-byte-swizzled K-major layout and
//               their E4M3 scales in the tensor-memory copy layout (below); a
//               K-step block is 4 KB of the workspace.
//   k_tc4       the weight stream, one CTA per SM:
//     warp 0    TMA producer: per stage a 256-row x 256-element tile of W codes
//               (32 KB, 128-byte swizzle, L2 evict-first), its scales (4 KB)
//               and the K-step's X block (4 KB, one bulk copy), 5 stages.
//     warps 3-4 scale warps, one per 128-row half: regroup the half's W scales
//               into the copy layout (all lanes), copy them to tensor memory
//               (tcgen05.cp, 4 per stage; warp 3 also the 4 X-scale copies)
//               and commit to the stage's scales-ready barrier.
//     warps 1-2 MMA warps, one per half: 4 MMAs per stage (K-blocks of 64)
//               into the half's fp32 accumulator in tensor memory, then
//               commit the stage back to the producer.
//     warps 5-12 epilogue: tcgen05.ld of a finished tile (double-buffered
//               accumulators), gs_w * gs_x, bf16 rounding, store; or fp32
//               partials and a deterministic in-order sum when K is split.
//
// Scale layout in tensor memory. For an M = 128 MMA the scales of row
// m = 32 * m1 + m0 (four bytes, one per 16-element block of the MMA's 64 K)
// sit in column base + m1 at lane m0 of every 32-lane quadrant. A copy of
// 32 x 128 bits broadcast to the four quadrants writes exactly that from a
// 512-byte shared-memory atom whose byte 16 * m0 + 4 * m1 + b is block b of
// row 32 * m1 + m0. The token scales use the same atom (tokens < 16: m1 = 0).
// So each MMA's scales take 4 columns, and every scale address an MMA is
// given is a multiple of 4 columns.
//
// Work split: units are (256-row tile, K-slice) pairs. When the tiles fill
// the SMs a unit is a whole tile and CTAs loop over tiles; otherwise K is cut
// into S slices so that tiles * S CTAs stream, each writes fp32 partials,
// and the last slice to finish (atomic counter) sums all S in slice order
// (results repeat bit for bit) and resets the counter.
//
// Every wait is bounded (clock64); on expiry the kernel records an error in
// the workspace status word, stops, waits for its own TMA loads and MMAs,
// frees tensor memory and returns.
#include "kernels.h"
#include "nvfp4_device.cuh"

#include <cuda.h>

namespace nvfp4 {
namespace tc4 {

constexpr int KS = 256;                      // K elements per stage
constexpr int TROWS = 256;                   // weight rows per tile (two M = 128 MMAs)
constexpr int NTOK = 16;                     // MMA N: tokens, zero-padded
constexpr int W_BYTES = TROWS * KS / 2;      // 32768
constexpr int S_BYTES = TROWS * KS / 16;     // 4096
constexpr int XC_BYTES = NTOK * KS / 2;      // 2048: X codes, 16 rows of 128 bytes
// W scales: one replicated 32 x 128-bit copy per MMA
constexpr int XB_BYTES = XC_BYTES + 4 * 512; // X codes + the 4 MMAs' scale atoms
constexpr int SA_BYTES = 8 * 512;            // W scale atoms: 2 halves x 4 MMAs
constexpr int NST = 5;
constexpr int SF_COLS = 48;                  // per stage: W 2 x 4 x 4, X 4 x 4
constexpr int align1k(int v) { return (v + 1023) / 1024 * 1024; }
// stage: [W codes][X block][W scales][W scales as copied], 1024-aligned parts
constexpr int OFF_XB = W_BYTES;
constexpr int OFF_S = align1k(OFF_XB + XB_BYTES);
constexpr int OFF_SA = OFF_S + S_BYTES;
constexpr int STAGE = align1k(OFF_SA + SA_BYTES);
constexpr int NUM_EPI = 8;
// warp 0 producer, then NMW MMA warps, NSFW scale warps, 8 epilogue warps (any
// 8 consecutive warps cover each 32-lane quadrant of tensor memory twice).
// Each tcgen05 instruction holds its issuing thread for ~100+ cycles, so the
// 12 scale copies and 8 MMAs of a stage are spread over four issuing warps
// (one row half each); measured on lm_head M = 1: one warp for everything
// 162 us, scale copies on their own warp 132 us, two of each 123 us.
constexpr int NMW = 2, NSFW = 2;
constexpr int WARP_MMA0 = 1, WARP_SF0 = WARP_MMA0 + NMW, WARP_EPI0 = WARP_SF0 + NSFW;
constexpr int NUM_THREADS = (WARP_EPI0 + NUM_EPI) * 32;
constexpr int TMEM_COLS = 512;
constexpr int ACC_COLS = 2 * NTOK;           // per accumulator buffer (two row halves)
constexpr int SF_BASE = 2 * ACC_COLS;        // after the two accumulator buffers
constexpr int SMEM_BYTES = NST * STAGE + 512 + 1024;
constexpr int BAR_EPI = 1;                   // named barrier of the epilogue warps
static_assert(SF_BASE + NST * SF_COLS <= TMEM_COLS, "tensor memory budget");
static_assert(STAGE % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");

constexpr uint32_t ST_TIMEOUT_PRODUCER = 1u, ST_TIMEOUT_MMA = 4u, ST_TIMEOUT_EPI = 8u,
                   ST_TIMEOUT_DRAIN = 16u;

struct Params {
  int M, N, K, tiles, S, ks_base, ks_rem, units;
  const float* gs;          // weights' per-tensor scale
  const float* gsx;         // X per-tensor scale (workspace, written by k_x4_quant)
  const uint8_t* xblk;      // X K-step blocks (workspace)
  uint16_t* y;
  uint32_t* status;
  uint32_t* amax;           // amax bits of X (workspace; reset here for the next call)
  uint32_t* counters;
  float* partials;
  long long timeout;
  int stall;
};

// ---- PTX wrappers -----------------------------------------------------------

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// K-major operand with the 128-byte swizzle: rows of 128 bytes, 8-row atoms
// of 1024 bytes (stride-byte offset), version 1, layout type 2.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
  return uint64_t((addr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}
// Source of a 32 x 128-bit scale copy: 32 rows of 16 bytes, no swizzle,
// 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t desc_sf(uint32_t addr) {
  return uint64_t((addr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) | (uint64_t(128 >> 4) << 32) |
         (uint64_t(1) << 46);
}
// Instruction descriptor: A and B E2M1 (format 1), K-major, N = 16, M = 128,
// UE4M3 scales (format 0), dense K = 64.
constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | (uint32_t(NTOK >> 3) << 17) | (uint32_t(128 >> 4) << 24);

__device__ __forceinline__ void sf_copy(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void mma_fp4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t sfa,
                                        uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(IDESC), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, "
      "%10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr) : "memory");
}

// Bounded wait on an mbarrier phase by one thread. Returns false if the CTA is
// aborting or the wait ran out (then the CTA starts aborting and the status
// word says who).
// hint_ns > 0: the thread may sleep in hardware between probes (until the
// phase completes or about hint_ns pass), leaving issue slots to the warps
// that issue tensor-core work.
__device__ __forceinline__ bool wait_bar(uint32_t b, uint32_t parity, volatile int* abort_flag,
                                         const Params& p, uint32_t who, uint32_t hint_ns = 0) {
  if (mbar_test(b, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (hint_ns ? mbar_wait_hint(b, parity, hint_ns) : mbar_test(b, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > p.timeout) {
      *abort_flag = 1;
      atomicOr(p.status, who);
      return false;
    }
  }
}
// The same for a whole warp: lane 0 waits, the others take its answer and,
// on success, observe the completed phase themselves.
__device__ __forceinline__ bool warp_wait(uint32_t b, uint32_t parity, volatile int* abort_flag,
                                          const Params& p, uint32_t who, int lane, uint32_t hint_ns = 0) {
  bool ok = true;
  if (lane == 0) ok = wait_bar(b, parity, abort_flag, p, who, hint_ns);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (ok && lane != 0) (void)mbar_test(b, parity);
  return ok;
}
__device__ __forceinline__ void drain_bar(uint32_t b, uint32_t parity, const Params& p) {
  const long long t0 = clock64();
  while (!mbar_test(b, parity)) {
    if (clock64() - t0 > p.timeout) {
      atomicOr(p.status, ST_TIMEOUT_DRAIN);
      return;
    }
  }
}

// Sum of the S slices' fp32 partials of row r for tokens m < M, each token's
// sum in slice order: G slices x MT tokens of loads in flight per round (the
// loads of a thread would otherwise wait on one another through the adds).
template <int MT, int G>
__device__ __forceinline__ void sum_slices(const float* base, int S, int M, int r, float* sum) {
  for (int s0 = 0; s0 < S; s0 += G) {
    float v[G][MT];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int m = 0; m < MT; ++m)
        v[g][m] = (s0 + g < S && m < M) ? __ldcg(base + (size_t(s0 + g) * M + m) * TROWS + r) : 0.0f;
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int m = 0; m < MT; ++m)
        if (s0 + g < S) sum[m] += v[g][m];
  }
}

struct Unit {
  int tile, slice, ks0, cnt;
};
__device__ __forceinline__ Unit unit_of(const Params& p, int u) {
  Unit q;
  q.tile = u / p.S;
  q.slice = u % p.S;
  q.cnt = p.ks_base + (q.slice < p.ks_rem ? 1 : 0);
  q.ks0 = q.slice * p.ks_base + min(q.slice, p.ks_rem);
  return q;
}

// ---- X preparation ------------------------------------------------------------

// amax(|X|) over all M * K elements as the largest bf16 magnitude bit pattern.
__global__ void __launch_bounds__(256)
k_x4_amax(const uint16_t* __restrict__ x, int n8, uint32_t* __restrict__ amax) {
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ uint32_t s_max[8];
  const uint4* x4 = reinterpret_cast<const uint4*>(x);
  uint32_t mg = 0u;
  for (int u = blockIdx.x * 256 + threadIdx.x; u < n8; u += gridDim.x * 256) mg = max(mg, bf16_mag_max8(x4[u]));
  mg = __reduce_max_sync(0xffffffffu, mg);
  if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = mg;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t m = 0u;
#pragma unroll
    for (int w = 0; w < 8; ++w) m = max(m, s_max[w]);
    if (m) atomicMax(amax, m);
  }
}

// One CTA per K-step: thread (n, b) quantises block b (16 elements) of token
// n by the weights' quantiser steps under gs_x = amax / 2688. Codes go to row
// n of the block's 128-byte-swizzled code tile (16-byte chunk c of row n at
// position c ^ (n & 7), as a TMA 128-byte swizzle would place it), scales to
// the copy-layout atom of MMA b / 4 (byte 16 n + b % 4). Tokens >= M and the
// atoms' unused bytes are zero.
__global__ void __launch_bounds__(256)
k_x4_quant(const uint16_t* __restrict__ x, int M, int K, const uint32_t* __restrict__ amax,
           uint8_t* __restrict__ xblk, float* __restrict__ gsx_out) {
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ uint32_t s_sc[NTOK][4];
  const float gsx = __fdiv_rn(__uint_as_float(*amax << 16), 2688.0f);   // 6 * 448
  const int n = threadIdx.x >> 4, b = threadIdx.x & 15;
  uint8_t* blk = xblk + size_t(blockIdx.x) * XB_BYTES;
  uint32_t s_code = 0u, q[2] = {0u, 0u};
  if (n < M) {
    const uint4* src = reinterpret_cast<const uint4*>(x + size_t(n) * K + size_t(blockIdx.x) * KS + 16 * b);
    const uint4 xa = src[0], xb = src[1];
    const uint32_t wv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
    float v[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = __uint_as_float(wv[i] << 16);
      v[2 * i + 1] = __uint_as_float(wv[i] & 0xFFFF0000u);
    }
    quantize_block16(v, gsx, s_code, q);
  }
  *reinterpret_cast<uint2*>(blk + n * 128 + (((b >> 1) ^ (n & 7)) << 4) + 8 * (b & 1)) = make_uint2(q[0], q[1]);
  reinterpret_cast<uint8_t*>(&s_sc[n][b >> 2])[b & 3] = uint8_t(s_code);
  __syncthreads();
  if (threadIdx.x < 128) {
    const int m0 = threadIdx.x >> 2, j = threadIdx.x & 3;
    const uint32_t w0 = m0 < NTOK ? s_sc[m0][j] : 0u;
    *reinterpret_cast<uint4*>(blk + XC_BYTES + j * 512 + 16 * m0) = make_uint4(w0, 0u, 0u, 0u);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) *gsx_out = gsx;
}

// ---- the kernel -------------------------------------------------------------

// At most 96 registers: 4 warps of one SM sub-partition then leave 4096 of
// its 16384 registers to the next call's X kernels (2 warps of <= 40), which
// start on these SMs while this grid runs (programmatic dependent launch).
__global__ void __maxnreg__(96)
k_tc4(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_s, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NST * STAGE);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + NST * STAGE + 256);
  // misc: [0] tensor memory base, [1] abort flag, [2] last-slice flag
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  const uint32_t b_full = smem_u32(bars), b_empty = b_full + 8 * NST, b_accf = b_empty + 8 * NST,
                 b_acce = b_accf + 16, b_sfr = b_acce + 16, b_done = b_sfr + 8 * NST;   // b_done: one per issuing warp
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(b_full + 8 * i, 1);
      mbar_init(b_empty + 8 * i, NMW);      // one commit per MMA warp
      mbar_init(b_sfr + 8 * i, NSFW);       // one commit per scale warp
    }
    for (int i = 0; i < 2; ++i) { mbar_init(b_accf + 8 * i, NMW); mbar_init(b_acce + 8 * i, NUM_EPI); }
    for (int i = 0; i < NMW + NSFW; ++i) mbar_init(b_done + 8 * i, 1);
    misc[1] = 0; misc[2] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(misc)), "r"(TMEM_COLS) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = misc[0];

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy();
      long long n_issued = 0, n_x = 0;
      // the X block of a step is issued after the wait for the X kernels;
      // the steps before it already stream their weights
      auto issue_x = [&](long long i, int ks) {
        bulk_load(smem_u32(smem + int(i % NST) * STAGE + OFF_XB), p.xblk + size_t(ks) * XB_BYTES, XB_BYTES,
                  b_full + 8 * int(i % NST));
      };
      bool waited = false;
      int pend_ks[NST];
      if (!p.stall) {
        for (int u = blockIdx.x; u < p.units && !*abort_flag; u += gridDim.x) {
          const Unit q = unit_of(p, u);
          bool stop = false;
          for (int j = 0; j < q.cnt; ++j, ++n_issued) {
            const int st = int(n_issued % NST);
            const uint32_t ph = uint32_t(n_issued / NST) & 1u;
            if (!wait_bar(b_empty + 8 * st, ph ^ 1u, abort_flag, p, ST_TIMEOUT_PRODUCER, 1000)) { stop = true; break; }
            uint8_t* sb = smem + st * STAGE;
            mbar_expect_tx(b_full + 8 * st, W_BYTES + S_BYTES + XB_BYTES);
            tma_load_2d_hint(smem_u32(sb), &tm_w, (q.ks0 + j) * (KS / 2), q.tile * TROWS, b_full + 8 * st, pol);
            tma_load_2d_hint(smem_u32(sb + OFF_S), &tm_s, (q.ks0 + j) * (KS / 16), q.tile * TROWS,
                             b_full + 8 * st, pol);
            if (waited) {
              issue_x(n_issued, q.ks0 + j);
              ++n_x;
            } else {
              pend_ks[st] = q.ks0 + j;
              if (n_issued + 1 == NST) {
                asm volatile("griddepcontrol.wait;" ::: "memory");
                waited = true;
                for (; n_x <= n_issued; ++n_x) issue_x(n_x, pend_ks[int(n_x % NST)]);
              }
            }
          }
          if (stop) break;
        }
        if (!waited) {
          // fewer steps than stages
          asm volatile("griddepcontrol.wait;" ::: "memory");
          waited = true;
          for (; n_x < n_issued; ++n_x) issue_x(n_x, pend_ks[int(n_x % NST)]);
        }
      }
      if (*abort_flag) {
        // wait for the loads still in flight before the CTA may exit
        const long long first = n_issued > NST ? n_issued - NST : 0;
        for (long long i = first; i < n_issued; ++i)
          drain_bar(b_full + 8 * int(i % NST), uint32_t(i / NST) & 1u, p);
      }
    }
    __syncwarp();
  } else if (warp < WARP_SF0) {
    // ------------------------------------------------------------ MMA issuers
    // warp mw issues the MMAs of the row halves h with h % NMW == mw
    const int mw = warp - WARP_MMA0;
    long long n = 0;
    int tcount = 0;
    bool issued = false;
    for (int u = blockIdx.x; u < p.units; u += gridDim.x, ++tcount) {
      const Unit q = unit_of(p, u);
      const int ab = tcount & 1;
      if (tcount >= 2 &&
          !warp_wait(b_acce + 8 * ab, uint32_t((tcount >> 1) - 1) & 1u, abort_flag, p, ST_TIMEOUT_MMA, lane))
        break;
      fence_after();
      bool stop = false;
      for (int j = 0; j < q.cnt; ++j, ++n) {
        const int st = int(n % NST);
        const uint32_t ph = uint32_t(n / NST) & 1u;
        if (!warp_wait(b_full + 8 * st, ph, abort_flag, p, ST_TIMEOUT_MMA, lane) ||
            !warp_wait(b_sfr + 8 * st, ph, abort_flag, p, ST_TIMEOUT_MMA, lane)) {
          stop = true;
          break;
        }
        if (lane == 0) {
          fence_after();
          uint8_t* sb = smem + st * STAGE;
          const uint32_t sf = tmem + uint32_t(SF_BASE + st * SF_COLS);
          const uint32_t a_w = smem_u32(sb), a_xc = smem_u32(sb + OFF_XB);
          const uint32_t d = tmem + uint32_t(ab * ACC_COLS);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const uint64_t bdesc = desc_sw128(a_xc + 32 * jj);
            for (int h = mw; h < 2; h += NMW)
              mma_fp4(d + uint32_t(h * NTOK), desc_sw128(a_w + h * (128 * 128) + 32 * jj), bdesc,
                      sf + uint32_t(4 * (h * 4 + jj)), sf + uint32_t(32 + 4 * jj), (j > 0 || jj > 0) ? 1u : 0u);
          }
          mma_commit(b_empty + 8 * st);
        }
        issued = true;
        __syncwarp();
      }
      if (stop) break;
      if (lane == 0) mma_commit(b_accf + 8 * ab);
    }
    if (lane == 0 && issued) {
      // every MMA of this thread has completed before tensor memory is freed
      mma_commit(b_done + 8 * (warp - WARP_MMA0));
      drain_bar(b_done + 8 * (warp - WARP_MMA0), 0, p);
    }
    __syncwarp();
  } else if (warp < WARP_EPI0) {
    // ------------------------------------------------------------ scale warps
    // warp sw regroups and copies the W scales of the row halves h with
    // h % NSFW == sw; warp 0 of them also copies the X scales
    const int sw = warp - WARP_SF0;
    long long n = 0;
    bool issued = false;
    for (int u = blockIdx.x; u < p.units; u += gridDim.x) {
      const Unit q = unit_of(p, u);
      bool stop = false;
      for (int j = 0; j < q.cnt; ++j, ++n) {
        const int st = int(n % NST);
        if (!warp_wait(b_full + 8 * st, uint32_t(n / NST) & 1u, abort_flag, p, ST_TIMEOUT_MMA, lane)) {
          stop = true;
          break;
        }
        uint8_t* sb = smem + st * STAGE;
        // W scales [256 rows][16 bytes] -> atoms (half h, MMA jj): lane m0 takes
        // rows 128h + 32 m1 + m0 (m1 = 0..3) and writes their jj-th words
        for (int h = sw; h < 2; h += NSFW) {
          uint4 r[4];
#pragma unroll
          for (int m1 = 0; m1 < 4; ++m1)
            r[m1] = *reinterpret_cast<const uint4*>(sb + OFF_S + (128 * h + 32 * m1 + lane) * 16);
          uint8_t* at = sb + OFF_SA + h * 4 * 512 + 16 * lane;
          *reinterpret_cast<uint4*>(at + 0 * 512) = make_uint4(r[0].x, r[1].x, r[2].x, r[3].x);
          *reinterpret_cast<uint4*>(at + 1 * 512) = make_uint4(r[0].y, r[1].y, r[2].y, r[3].y);
          *reinterpret_cast<uint4*>(at + 2 * 512) = make_uint4(r[0].z, r[1].z, r[2].z, r[3].z);
          *reinterpret_cast<uint4*>(at + 3 * 512) = make_uint4(r[0].w, r[1].w, r[2].w, r[3].w);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          fence_after();
          const uint32_t sf = tmem + uint32_t(SF_BASE + st * SF_COLS);
          const uint32_t a_sa = smem_u32(sb + OFF_SA), a_xs = smem_u32(sb + OFF_XB + XC_BYTES);
          for (int h = sw; h < 2; h += NSFW)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) sf_copy(sf + 4 * (h * 4 + jj), desc_sf(a_sa + 512 * (h * 4 + jj)));
          if (sw == 0)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) sf_copy(sf + 32 + 4 * jj, desc_sf(a_xs + 512 * jj));
          mma_commit(b_sfr + 8 * st);
        }
        issued = true;
        __syncwarp();
      }
      if (stop) break;
    }
    if (lane == 0 && issued) {
      mma_commit(b_done + 8 * (warp - WARP_MMA0));
      drain_bar(b_done + 8 * (warp - WARP_MMA0), 0, p);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int e = warp - WARP_EPI0, qd = warp & 3, h = e >> 2;
    if (blockIdx.x == 0 && e == 0 && lane == 0) *p.amax = 0u;   // the X kernels of this call are done
    const float scale = __fmul_rn(*p.gs, *p.gsx);
    int tcount = 0;
    for (int u = blockIdx.x; u < p.units; u += gridDim.x, ++tcount) {
      const Unit q = unit_of(p, u);
      const int ab = tcount & 1;
      // the eight warps agree on every outcome, so none waits alone at a barrier below
      const bool ok =
          warp_wait(b_accf + 8 * ab, uint32_t(tcount >> 1) & 1u, abort_flag, p, ST_TIMEOUT_EPI, lane, 20000);
      if (!named_bar_and(BAR_EPI, NUM_EPI * 32, ok)) break;
      fence_after();
      uint32_t v[16];
      tmem_ld16(tmem + (uint32_t(32 * qd) << 16) + uint32_t(ab * ACC_COLS + h * NTOK), v);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      float acc[16];
#pragma unroll
      for (int m = 0; m < 16; ++m) acc[m] = __uint_as_float(v[m]);
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_acce + 8 * ab);
      const int r = 128 * h + 32 * qd + lane;           // row within the tile
      const int row = q.tile * TROWS + r;
      if (p.S == 1) {
        if (row < p.N)
          for (int m = 0; m < p.M; ++m)
            p.y[size_t(m) * p.N + row] = float_to_bf16_bits(__fmul_rn(scale, acc[m]));
      } else {
        float* part = p.partials + (size_t(q.tile) * p.S + q.slice) * size_t(p.M) * TROWS;
        for (int m = 0; m < p.M; ++m) __stcg(part + m * TROWS + r, acc[m]);
        __threadfence();
        named_bar(BAR_EPI, NUM_EPI * 32);
        if (e == 0 && lane == 0) {
          const uint32_t old = atomicAdd(p.counters + q.tile, 1u);
          const bool last = old == uint32_t(p.S - 1);
          if (last) p.counters[q.tile] = 0u;
          misc[2] = last ? 1u : 0u;
        }
        named_bar(BAR_EPI, NUM_EPI * 32);
        if (misc[2]) {
          __threadfence();
          if (row < p.N) {
            const float* base = p.partials + size_t(q.tile) * p.S * size_t(p.M) * TROWS;
            float sum[NTOK];
#pragma unroll
            for (int m = 0; m < NTOK; ++m) sum[m] = 0.0f;
            if (p.M <= 4) sum_slices<4, 8>(base, p.S, p.M, r, sum);
            else sum_slices<NTOK, 2>(base, p.S, p.M, r, sum);
#pragma unroll
            for (int m = 0; m < NTOK; ++m)
              if (m < p.M) p.y[size_t(m) * p.N + row] = float_to_bf16_bits(__fmul_rn(scale, sum[m]));
          }
        }
        named_bar(BAR_EPI, NUM_EPI * 32);
      }
    }
  }
  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS)
                 : "memory");
  }
}

}  // namespace tc4

cudaError_t tc4_configure(Tc4Config& c, int num_sms) {
  using namespace tc4;
  if (c.M < 1 || c.M > 16 || c.K % KS != 0 || c.K <= 0 || c.N <= 0) return cudaErrorInvalidValue;
  c.tiles = (c.N + TROWS - 1) / TROWS;
  const int ksteps = c.K / KS;
  int S = 1;
  if (c.tiles * 100 < num_sms * 85) {
    S = num_sms / c.tiles;
    if (S > ksteps) S = ksteps;
    if (S < 1) S = 1;
  }
  c.S = S;
  c.ks_base = ksteps / S;
  c.ks_rem = ksteps % S;
  c.units = c.tiles * S;
  c.grid = c.units < num_sms ? c.units : num_sms;
  c.smem = SMEM_BYTES;
  // workspace: [0] status word, [64] X amax bits, [68] gs_x; counters from
  // 256; X K-step blocks 1024-aligned; fp32 partials when K is split
  c.ws_amax_off = 64;
  c.ws_gsx_off = 68;
  c.ws_counters_off = 256;
  c.ws_x_off = (c.ws_counters_off + size_t(c.tiles) * 4 + 1023) / 1024 * 1024;
  c.ws_partials_off = c.ws_x_off + size_t(ksteps) * XB_BYTES;
  c.ws_bytes = c.ws_partials_off + (S > 1 ? size_t(c.tiles) * S * c.M * TROWS * 4 : 0);
  int dev = 0, optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  if (c.smem > size_t(optin)) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(k_tc4, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e != cudaSuccess) return e;
  if (!tensor_maps_supported()) return cudaErrorNotSupported;
  return cudaSuccess;
}

cudaError_t launch_tc4(const Tc4Config& c, const void* map_w, const void* map_s, const float* gs,
                       const uint16_t* x, uint16_t* y, void* workspace, long long timeout_cycles, bool stall,
                       bool pdl, cudaStream_t st) {
  using namespace tc4;
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  uint32_t* amax = reinterpret_cast<uint32_t*>(wsb + c.ws_amax_off);
  float* gsx = reinterpret_cast<float*>(wsb + c.ws_gsx_off);
  uint8_t* xblk = wsb + c.ws_x_off;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;

  const int n8 = c.M * c.K / 8;
  int ga = (n8 + 1023) / 1024;
  if (ga < 1) ga = 1;
  if (ga > 148) ga = 148;
  cudaLaunchConfig_t pa = {};
  pa.gridDim = dim3(ga);
  pa.blockDim = dim3(256);
  pa.stream = st;
  pa.attrs = attr;
  pa.numAttrs = pdl ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&pa, k_x4_amax, x, n8, amax);
  if (e != cudaSuccess) return e;

  // the next two wait for their predecessor in-kernel
  cudaLaunchConfig_t pq = {};
  pq.gridDim = dim3(c.K / KS);
  pq.blockDim = dim3(256);
  pq.stream = st;
  pq.attrs = attr;
  pq.numAttrs = 1;
  e = cudaLaunchKernelEx(&pq, k_x4_quant, x, c.M, c.K, static_cast<const uint32_t*>(amax), xblk, gsx);
  if (e != cudaSuccess) return e;

  Params p;
  p.M = c.M; p.N = c.N; p.K = c.K; p.tiles = c.tiles; p.S = c.S;
  p.ks_base = c.ks_base; p.ks_rem = c.ks_rem; p.units = c.units;
  p.gs = gs; p.gsx = gsx; p.xblk = xblk; p.y = y;
  p.status = reinterpret_cast<uint32_t*>(wsb);
  p.amax = amax;
  p.counters = reinterpret_cast<uint32_t*>(wsb + c.ws_counters_off);
  p.partials = c.S > 1 ? reinterpret_cast<float*>(wsb + c.ws_partials_off) : nullptr;
  p.timeout = timeout_cycles;
  p.stall = stall ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(c.grid);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = c.smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const CUtensorMap mw = *static_cast<const CUtensorMap*>(map_w);
  const CUtensorMap ms = *static_cast<const CUtensorMap*>(map_s);
  return cudaLaunchKernelEx(&cfg, k_tc4, mw, ms, p);
}

}  // namespace nvfp4
