// k_mma.cu -- TMA-fed warp-MMA variant of the NVFP4 linear (sm_100a).
//
// Y[M][N] = X[M][K] W^T, swap-AB on mma.sync.m16n8k16 (f16 x f16 -> f32):
// the 16-row MMA dimension is weight rows, the 8-column dimension is tokens
// (1 + drafted tokens checked in one pass; page "InventDB Sparkle", section
// "How it answers quickly"). The weight read is the whole cost (page
// "Qwen3.8-27B-NVFP4-RTX5090 API & Inference Endpoint", section "Why lm_head
// is NVFP4, and why MTP is gone"), so the kernel is a weight stream, one CTA
// per SM:
//
//   warp 0       TMA producer: 256-row x 256-element tiles of packed codes
//                (32 KB, 128-byte swizzle) and their E4M3 scales (4 KB), with
//                an L2 evict-first policy, into a ring of 3..8 shared-memory
//                stages (mbarrier full/empty pairs).
//   warps 1..16  consumers: warp w owns rows 16(w-1)..16(w-1)+15 of every tile.
//                Lane (g, t) reads rows g and g+8, 64 consecutive K elements
//                each (two swizzled 16-byte chunks and 4 scale bytes per row),
//                converts codes and scales with the hardware e2m1x2 / e4m3x2 ->
//                f16x2 conversions and multiplies them (exact: at most 6
//                significant bits, magnitude in [2^-10, 2688]) straight into
//                the A fragment registers, then issues the MMAs. MMA i of a
//                step maps its K slots to physical K as (2t, 2t+1) <-> 64t + 4i
//                + {0, 1} and (2t+8, 2t+9) <-> 64t + 4i + {2, 3}, so every
//                fragment is four consecutive elements of one lane. A warp
//                releases a stage after its MMAs. For M = 1 (and M = 2 without
//                a lo plane) the A fragments are the raw E2M1 values and the
//                block scale is applied per 16-element block in fp32 instead
//                (block-diagonal B, compute_step_bd). FP8 weights: the same K
//                mapping on E4M3 codes, row scales applied to the sums.
//   warp 17      settler: completes tiles split between CTAs (below).
//
// B is X in f16, scaled per token by a power of two (largest magnitude at
// 2^14) in a hi plane (exact within 2^28 of that maximum) and a lo plane
// scaled by 2^29 (exact for the next 29 binades); elements further below keep
// only the lo plane's subnormal step (within 2^-68 of the maximum).
// Columns are groups of 64 elements padded to 136 bytes, so B fragments are
// bank-conflict-free 8-byte shared loads at immediate offsets. Every product
// is exact; only the fp32 accumulation rounds. When no element needs the lo
// plane, only hi tiles are issued. M <= 4: each CTA stages the K-steps of X
// its units touch in shared memory (W4A4: quantising them to NVFP4 on the
// way). M >= 5 ("X in the ring"): k_xprep writes both planes once per call
// into the workspace and every ring stage also carries one K-step box of
// them, so these classes need no K-slices.
//
// Why not tcgen05 here: for N = 8..32 token columns a tcgen05.mma of M = 128
// weight rows costs hundreds of cycles per instruction once its A operand
// has to be decoded and stored by the warps (the variant TC kernel measures
// ~400 SM cycles per MMA, tensor pipe 3% busy), while this warp MMA takes the
// decoded fragments straight from registers at ~1000 MAC per clock per SM.
// For this skinny contraction the warp MMA is the faster tensor path.
//
// Work split: with at most as many 256-row tiles as SMs (and at least 85% of
// them busy) every CTA takes one whole tile over all of K and stores it
// directly: nothing crosses CTAs. Otherwise K is cut into S slices (S = 1
// unless a staged X slice would not fit next to the ring) and the CTAs of a
// slice share its (256-row tile, 256-k step) units evenly (stream-K). Tiles a
// CTA covers entirely are stored directly. A split tile is completed per
// 16-row group: the pieces write fp32 partials and count themselves on the
// group's counter; the last sums all pieces in k order (results repeat bit
// for bit) and resets the counter. The piece at the end of a CTA's range
// usually finds the tile's other piece already counted and finishes the tile
// from its registers. Every mbarrier wait is bounded; on expiry the CTA
// records the timeout in the workspace status word, stops, drains its
// in-flight TMA loads and returns.
#include "kernels.h"
#include "nvfp4_device.cuh"

#include <cuda.h>
#include <algorithm>
#include <climits>
#include <vector>

namespace nvfp4 {
namespace mm {

constexpr int KS = 256;                    // K elements per step
constexpr int XP_STEPS = 8;                // K-steps one X-conversion block converts
constexpr int TROWS = 256;                 // weight rows per tile
constexpr int NCW = 16;                    // consumer warps (16 rows each)
constexpr int WARP_SETTLE = NCW + 1;       // warp 0 producer, 1..16 consumers, 17 settler
constexpr int NUM_THREADS = (NCW + 2) * 32;
constexpr int QN = 8;                      // split-tile queue slots (consumers -> settler)
constexpr int MAX_PIECES = 62;             // pieces of one tile that can be listed
constexpr int FAST_MAX = 3;                // other pieces the in-loop finish can add
constexpr int LIST_MAX = 32;               // row groups whose sum waits for the end phase
constexpr int NSTAGE_MIN = 3;             // ring depth the X budget is planned with
constexpr int NSTAGE_MAX = 8;             // deeper rings use what X leaves free
constexpr int W_BYTES = TROWS * KS / 2;    // 32768
constexpr int S_BYTES = TROWS * KS / 16;   // 4096
// FP8 weight tier: E4M3 codes [N][K], one fp32 scale per row; a stage holds
// 256 rows x 256 codes as two 128-byte-wide swizzled halves (K 0..127, 128..255)
constexpr int FMT_NVFP4 = 0, FMT_FP8 = 1;
constexpr int W_BYTES_FP8 = TROWS * KS;    // 65536
__host__ __device__ constexpr int w_bytes_of(int fmt) { return fmt == FMT_FP8 ? W_BYTES_FP8 : W_BYTES; }
__host__ __device__ constexpr int s_bytes_of(int fmt) { return fmt == FMT_FP8 ? 0 : S_BYTES; }
constexpr int MISC_BASE = 1024;            // barriers, flags, lists
// misc area size: for M <= 4 plus the prefetched piece [M][TROWS] floats
inline int misc_bytes(int M) { return MISC_BASE + (M <= 4 ? M * TROWS * 4 : 0); }
// misc area: barriers [0,256) (full, empty, qfull, qempty: 8 each), emax [256,320),
// flags [320,336) (need_lo, abort, list count), skip masks [336,368),
// prefetch flag [368,372), W4A4 amax and gs_x [372,380), piece slots
// [384,640), end-phase list [640,896)
constexpr int MISC_EMAX = 256, MISC_FLAGS = 320, MISC_SKIP = 336, MISC_PREFLAG = 368, MISC_PIECES = 384,
              MISC_LIST = 640, MISC_PREBUF = 1024,   // prefetched piece: [M <= 4][TROWS] floats
              MISC_XAMAX = 372, MISC_XGS = 376;      // W4A4: largest |x| (bf16 bits), gs_x
constexpr int LO_SHIFT = X_LO_SHIFT;
constexpr int BAR_CONSUMERS = 1;           // named barrier of the consumer warps
constexpr int XR_MIN_M = 5;                // token counts from which X goes through the ring

constexpr uint32_t ST_TIMEOUT_PRODUCER = 1u, ST_TIMEOUT_CONSUMER = 2u, ST_TIMEOUT_SETTLER = 4u,
                   ST_TIMEOUT_DRAIN = 16u;

struct Params {
  int M, N, K, tiles, S, P, ks_base, ks_rem, ncols, xk_max, xstride, pmax, nstage;
  int tpc;                                   // whole tiles per CTA (no split tiles), 0: stream-K
  int act4;                                  // W4A4: X quantised to NVFP4 in the kernel
  const float* row_scale;                    // FP8 tier: fp32 scale of each weight row [N]
  const float* xgs;                          // W4A4 with X in the ring: gs_x written by k_xprep
  int xbytes, xbox_words, xbox_bytes;        // X in the ring: stage area, words per column, box bytes
  const int* xemax;                          // X in the ring: per-token exponent maximum
  const uint32_t* xlo;                       // X in the ring: "lo plane used" [xchunks][16]
  int xchunks;                               // X in the ring: conversion blocks per token
  const float* gs;
  const uint16_t* x;
  uint16_t* y;
  uint32_t* status;
  uint32_t* counters;
  float* partials;
  unsigned long long* keys;                  // argmax epilogue: per-token best (value, index) key
  uint32_t* done;                            // argmax epilogue: CTAs finished
  long long timeout;
  int stall;
};

// ---- epilogues --------------------------------------------------------------
// EPI_NONE: y[m][n] = bf16(gs * acc). EPI_SWIGLU (fused gate+up projection,
// rows 2c and 2c+1 are the gate and up rows of output column c): y[m][c] =
// bf16(silu(gs * acc_2c) * gs * acc_2c+1), computed in fp32 from the complete
// sums. EPI_ARGMAX (greedy choice over the output vocabulary): per token the
// largest fp32 logit gs * acc and its row, equal values going to the lower
// row; no logits are written. The candidates meet as 64-bit keys (order-
// preserving bits of the value above the complemented row index) in one
// atomic maximum per token and warp; the last CTA to finish writes
// int32 index [M] then float value [M] to y and clears the keys.
constexpr int EPI_NONE = 0, EPI_SWIGLU = 1, EPI_ARGMAX = 2;

__device__ __forceinline__ float silu(float v) { return v / (1.0f + expf(-v)); }

__device__ __forceinline__ unsigned long long argmax_key(float v, int n) {
  const uint32_t b = __float_as_uint(v);
  const uint32_t ord = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return (static_cast<unsigned long long>(ord) << 32) | (0xFFFFFFFFu - uint32_t(n));
}
__device__ __forceinline__ unsigned long long shfl_xor_u64(unsigned mask, unsigned long long v, int o) {
  const uint32_t lo = __shfl_xor_sync(mask, uint32_t(v), o), hi = __shfl_xor_sync(mask, uint32_t(v >> 32), o);
  return (static_cast<unsigned long long>(hi) << 32) | lo;
}

// Token of accumulator value e of a lane in quad position t, or -1: the
// columns 2t, 2t+1 of the first token tile (e = 0, 1) and of the second
// (e = 2, 3; M > 8). The block-diagonal class (MC 0) leaves its tokens where
// class 1 has them.
template <int MC>
__device__ __forceinline__ int tok_of(int t, int e) {
  if (MC <= 1) return (t < 2 && e < 2) ? 2 * t + e : -1;
  if (e < 2) return 2 * t + e;
  return MC == 3 ? 8 + 2 * t + (e - 2) : -1;
}

// Complete sums (before the global scale) of a lane's rows row0 and row0 + 8
// for its tokens, stored as the plan's epilogue asks. All 32 lanes of the
// warp call it together (the epilogues exchange values across lanes).
template <int MC, int EPI>
__device__ __forceinline__ void emit_rows(const Params& p, int row0, const float (&val)[4][2], float gs,
                                          int lane) {
  const int t = lane & 3, g = lane >> 2;
  if constexpr (EPI == EPI_NONE) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int m = tok_of<MC>(t, e);
      if (m >= 0 && m < p.M) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int n = row0 + 8 * h;
          if (n < p.N) p.y[size_t(m) * p.N + n] = float_to_bf16_bits(gs * val[e][h]);
        }
      }
    }
  } else if constexpr (EPI == EPI_SWIGLU) {
    // rows row0 and row0 + 8 pair with the rows of the lane g ^ 1
    float up[4][2];
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
      for (int h = 0; h < 2; ++h) up[e][h] = __shfl_xor_sync(0xffffffffu, val[e][h], 4);
    if ((g & 1) == 0) {
      const int half = p.N >> 1;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int m = tok_of<MC>(t, e);
        if (m >= 0 && m < p.M) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int n = row0 + 8 * h;
            if (n < p.N) p.y[size_t(m) * half + (n >> 1)] = float_to_bf16_bits(silu(gs * val[e][h]) * (gs * up[e][h]));
          }
        }
      }
    }
  } else {
    // the eight lanes g = 0..7 of a quad position hold the same tokens
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int m = tok_of<MC>(t, e);
      unsigned long long key = 0ull;
      if (m >= 0 && m < p.M) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int n = row0 + 8 * h;
          if (n < p.N) key = max(key, argmax_key(gs * val[e][h], n));
        }
      }
      key = max(key, shfl_xor_u64(0xffffffffu, key, 4));
      key = max(key, shfl_xor_u64(0xffffffffu, key, 8));
      key = max(key, shfl_xor_u64(0xffffffffu, key, 16));
      if (g == 0 && m >= 0 && m < p.M) atomicMax(p.keys + m, key);
    }
  }
}

// Byte offset of X element k (local to the slice) inside a column: groups of
// 64 elements take 136 bytes (8 bytes of padding), so the four lanes t of an
// MMA, which read groups 4s+t of step s, start on different banks and the
// offsets of the sixteen MMAs of a step are immediates.
constexpr int XGROUP_BYTES = 136;
__device__ __forceinline__ uint32_t x_off(int k) {
  return uint32_t(XGROUP_BYTES * (k >> 6) + 2 * (k & 63));
}

__device__ __forceinline__ void mma16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Same, accumulator starting from zero.
__device__ __forceinline__ void mma16816_z(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%10, %10, %10, %10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// Bounded mbarrier wait. Between checks of the abort flag and the clock the
// thread sleeps in try_wait (up to `hint_ns`) rather than spinning, so
// waiting warps leave the issue slots to the ones computing.
__device__ __forceinline__ bool wait_bar(uint32_t b, uint32_t parity, volatile int* abort_flag,
                                         const Params& p, uint32_t who, uint32_t hint_ns = 2000) {
  if (mbar_test(b, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_wait_hint(b, parity, hint_ns)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > p.timeout) {
      *abort_flag = 1;
      atomicOr(p.status, who);
      return false;
    }
  }
}

// Number of CTA range boundaries floor(c * L / W), c in [1, W), in (lo, hi];
// 32-bit (configure() checks that L * W fits).
__device__ __forceinline__ int bnd_in(int lo, int hi, int L, int W) {
  if (hi <= lo) return 0;
  int cmin = int((unsigned(lo + 1) * unsigned(W) + unsigned(L) - 1u) / unsigned(L));
  int cmax = int((unsigned(hi + 1) * unsigned(W) + unsigned(L) - 1u) / unsigned(L)) - 1;
  if (cmin < 1) cmin = 1;
  if (cmax > W - 1) cmax = W - 1;
  return cmax >= cmin ? cmax - cmin + 1 : 0;
}

// Tile whose first k-range is this CTA's last segment and whose only other
// piece is the next CTA's first segment (one slice), else -1: the settler
// fetches that piece into shared memory while the consumers work, so the
// tile is finished from registers at the end.
__device__ __forceinline__ int prefetch_tile(const Params& p, int a, int b, int cnt, int L) {
  if (p.S != 1 || b <= a || p.M > 4) return -1;
  const int tf = (b - 1) / cnt;
  if (tf * cnt < a || b >= (tf + 1) * cnt) return -1;
  return bnd_in(tf * cnt, (tf + 1) * cnt - 1, L, p.P) == 1 ? tf : -1;
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* a) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t* a) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// Slots of the pieces of `tile` in k order (slice, then ordinal); returns
// their number (at most MAX_PIECES are listed).
__device__ __forceinline__ int list_pieces(const Params& p, int tile, uint32_t* out) {
  int n = 0;
  for (int s2 = 0; s2 < p.S; ++s2) {
    const int cnt2 = p.ks_base + (s2 < p.ks_rem ? 1 : 0);
    const int L2 = p.tiles * cnt2;
    const int np = 1 + bnd_in(tile * cnt2, (tile + 1) * cnt2 - 1, L2, p.P);
    for (int o = 0; o < np && n < MAX_PIECES; ++o)
      out[n++] = uint32_t(((long long)tile * p.S + s2) * p.pmax + o);
  }
  return n;
}

// Y rows of the row groups in `gmask` of `tile` = sum of all pieces in k
// order (first piece first), for threads tid, tid + nth, ...
template <int EPI>
__device__ __forceinline__ void sum_pieces(const Params& p, int tile, uint32_t gmask,
                                           const uint32_t* pieces, int np, int tid, int nth) {
  const float gs = *p.gs;
  const int MT = p.M * TROWS;
  const int nval = __popc(gmask) * 16 * p.M;
  for (int u = tid; u < nval; u += nth) {
    const int rr = u & 15, rest = u >> 4;
    const int m = rest % p.M, gi = rest / p.M;
    const int grp = __fns(gmask, 0, gi + 1);
    const int row = grp * 16 + rr;
    const float* base = p.partials + size_t(m) * TROWS + row;
    float sum = __ldcg(base + size_t(pieces[0]) * MT);
    int o = 1;
    for (; o + 3 < np; o += 4) {
      const float v1 = __ldcg(base + size_t(pieces[o]) * MT), v2 = __ldcg(base + size_t(pieces[o + 1]) * MT);
      const float v3 = __ldcg(base + size_t(pieces[o + 2]) * MT), v4 = __ldcg(base + size_t(pieces[o + 3]) * MT);
      sum += v1; sum += v2; sum += v3; sum += v4;
    }
    for (; o < np; ++o) sum += __ldcg(base + size_t(pieces[o]) * MT);
    const int n = tile * TROWS + row;
    if constexpr (EPI == EPI_NONE) {
      if (n < p.N) p.y[size_t(m) * p.N + n] = float_to_bf16_bits(gs * sum);
    } else if constexpr (EPI == EPI_SWIGLU) {
      // consecutive u are consecutive rows of one token: the partner is u ^ 1
      const float up = __shfl_xor_sync(__activemask(), sum, 1);
      if ((rr & 1) == 0 && n < p.N) p.y[size_t(m) * (p.N >> 1) + (n >> 1)] = float_to_bf16_bits(silu(gs * sum) * (gs * up));
    } else {
      // the 16 consecutive u of a row group share the token
      const unsigned mask = __activemask();
      unsigned long long key = n < p.N ? argmax_key(gs * sum, n) : 0ull;
      key = max(key, shfl_xor_u64(mask, key, 1));
      key = max(key, shfl_xor_u64(mask, key, 2));
      key = max(key, shfl_xor_u64(mask, key, 4));
      key = max(key, shfl_xor_u64(mask, key, 8));
      if (rr == 0) atomicMax(p.keys + m, key);
    }
  }
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

// X in the ring: one CTA per token converts its row of X into the hi and lo
// planes (columns m and M + m, `pitch` bytes each, the shared-memory group
// layout of x_off) and records the token's exponent maximum and whether its
// lo plane is used. The main kernel then loads one K-step of all planes per
// ring stage.
//
// Both conversion kernels are held to 32 registers a thread: the main kernel
// triggers its launch at the top of theirs, and with 18 warps of 82-88
// registers it leaves 2304 registers in an SM sub-partition of 16384, two
// warps of up to 32 each. Above that a conversion block cannot share an SM
// with a main CTA; with a main grid on every SM each call then waits for SMs
// to drain (measured: +9 us a call on the down projection at M = 8 and 16
// with 43 registers, none at 32).
//
// Block (m, c) of the grid (M, C) takes the maximum over the whole row but
// converts only K-steps [csteps c, csteps (c + 1)), so a long row is
// converted by several SMs at once; it records its lo-plane use in its own
// slot lo_out[16 c + m] (the main kernel ORs the slots of a token).
__global__ void __launch_bounds__(256, 8)
k_xprep(const uint16_t* __restrict__ x, int M, int K, uint8_t* __restrict__ planes, int pitch,
        int* __restrict__ emax_out, uint32_t* __restrict__ lo_out, int csteps) {
  // The main kernel may launch now (it waits for this grid before it reads
  // the planes, and meanwhile streams weights); X may be the previous grid's
  // output.
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ int s_max[8];
  const int m = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint4* row = reinterpret_cast<const uint4*>(x + size_t(m) * K);
  const int chunks = K / 8;
  uint32_t mag = 0u;
  for (int kc = threadIdx.x; kc < chunks; kc += 256) mag = max(mag, bf16_mag_max8(row[kc]));
  int mx = bf16_mag_exp(__reduce_max_sync(0xffffffffu, mag));
  if (lane == 0) s_max[warp] = mx;
  __syncthreads();
  int emax = s_max[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) emax = max(emax, s_max[w]);
  const int sh = emax == INT_MIN ? 0 : 14 - emax;
  bool lo_used = false;
  uint8_t* ch = planes + size_t(m) * pitch;
  uint8_t* cl = planes + size_t(M + m) * pitch;
  const int kc_end = min(chunks, int(blockIdx.y + 1) * (csteps * KS / 8));
  for (int kc = int(blockIdx.y) * (csteps * KS / 8) + threadIdx.x; kc < kc_end; kc += 256) {
    const uint4 v = row[kc];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t hi[4], lo[4];
    lo_used |= x_split8(w, sh, hi, lo);
    *reinterpret_cast<uint2*>(ch + x_off(8 * kc)) = make_uint2(hi[0], hi[1]);
    *reinterpret_cast<uint2*>(ch + x_off(8 * kc + 4)) = make_uint2(hi[2], hi[3]);
    *reinterpret_cast<uint2*>(cl + x_off(8 * kc)) = make_uint2(lo[0], lo[1]);
    *reinterpret_cast<uint2*>(cl + x_off(8 * kc + 4)) = make_uint2(lo[2], lo[3]);
  }
  lo_used = __syncthreads_or(lo_used);
  if (threadIdx.x == 0) {
    emax_out[m] = emax;                        // the same value from every block of the row
    lo_out[16 * blockIdx.y + m] = lo_used ? 1u : 0u;
  }
}

// W4A4 with X in the ring: the token's row quantised to NVFP4 by the weights'
// quantiser steps under gs_x = amax(|X|) / 2688 over all of X (every CTA takes
// the maximum over all tokens, so all agree); the hi plane holds the exact f16
// products e2m1 * e4m3, the lo plane zeros, the per-token factor is 1, and
// CTA 0 stores gs_x for the main kernel's epilogue.
__global__ void __launch_bounds__(256, 8)
k_xprep_act4(const uint16_t* __restrict__ x, int M, int K, uint8_t* __restrict__ planes, int pitch,
             int* __restrict__ emax_out, uint32_t* __restrict__ lo_out, float* __restrict__ gsx_out) {
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ uint32_t s_max[8];
  const int m = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint4* row = reinterpret_cast<const uint4*>(x + size_t(m) * K);
  const uint4* all = reinterpret_cast<const uint4*>(x);
  uint32_t mg = 0u;
  for (int u = threadIdx.x; u < M * (K / 8); u += 256) mg = max(mg, bf16_mag_max8(all[u]));
  mg = __reduce_max_sync(0xffffffffu, mg);
  if (lane == 0) s_max[warp] = mg;
  __syncthreads();
  uint32_t amax_bits = 0u;
#pragma unroll
  for (int w = 0; w < 8; ++w) amax_bits = max(amax_bits, s_max[w]);
  const float gsx = __fdiv_rn(__uint_as_float(amax_bits << 16), 2688.0f);   // 6 * 448
  uint8_t* ch = planes + size_t(m) * pitch;
  uint8_t* cl = planes + size_t(M + m) * pitch;
  for (int b = threadIdx.x; b < K / 16; b += 256) {
    const uint4 xa = row[2 * b], xb = row[2 * b + 1];
    const uint32_t wv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
    float v[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = __uint_as_float(wv[i] << 16);
      v[2 * i + 1] = __uint_as_float(wv[i] & 0xFFFF0000u);
    }
    uint32_t s_code, q[2];
    quantize_block16(v, gsx, s_code, q);
    const uint32_t sc = bcast_lo(e4m3x2_to_f16x2(s_code));
    uint32_t h[8];
    e2m1x8_to_f16x2x4(q[0], h);
    e2m1x8_to_f16x2x4(q[1], h + 4);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      *reinterpret_cast<uint2*>(ch + x_off(16 * b + 4 * c)) = make_uint2(hmul2(h[2 * c], sc), hmul2(h[2 * c + 1], sc));
      *reinterpret_cast<uint2*>(cl + x_off(16 * b + 4 * c)) = make_uint2(0u, 0u);
    }
  }
  if (threadIdx.x == 0) {
    emax_out[m] = 14;
    lo_out[m] = 0u;
    if (m == 0) *gsx_out = gsx;
  }
}

// One step of one lane: decode rows r and r+8 of the stage (64 elements each)
// and issue the MMAs for NTILE 8-column token tiles. MMA i of the step adds
// into accumulator set i % (4 / NTILE): four independent chains per warp,
// instead of sixteen MMAs serialised on one accumulator. PRED: token tiles
// flagged off in `xon` read a zero B fragment instead of shared memory.
// EARLY: after loading its share of the stage into registers the warp
// releases the slot (lane 0 arrives on `empty`), so the refill overlaps the
// decode and the MMAs.
template <int NTILE, bool EARLY, bool PRED>
__device__ __forceinline__ void compute_step(const uint8_t* sw, const uint8_t* ss, int r, float (*acc)[4],
                                             const uint8_t* sx, const uint32_t* xcol, const bool* xon,
                                             uint32_t xg, int t, uint32_t empty_bar, int lane) {
  const int r1 = r + 8;
  // chunks 2t, 2t+1 of each row; the TMA 128-byte swizzle puts chunk c of row
  // r at position c ^ (r & 7)
  const uint4 c00 = *reinterpret_cast<const uint4*>(sw + r * 128 + (((2 * t) ^ (r & 7)) << 4));
  const uint4 c01 = *reinterpret_cast<const uint4*>(sw + r * 128 + (((2 * t + 1) ^ (r & 7)) << 4));
  const uint4 c10 = *reinterpret_cast<const uint4*>(sw + r1 * 128 + (((2 * t) ^ (r1 & 7)) << 4));
  const uint4 c11 = *reinterpret_cast<const uint4*>(sw + r1 * 128 + (((2 * t + 1) ^ (r1 & 7)) << 4));
  const uint32_t s0 = *reinterpret_cast<const uint32_t*>(ss + r * 16 + 4 * t);
  const uint32_t s1 = *reinterpret_cast<const uint32_t*>(ss + r1 * 16 + 4 * t);
  if (EARLY) {
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar);
  }
  const uint32_t w0[8] = {c00.x, c00.y, c00.z, c00.w, c01.x, c01.y, c01.z, c01.w};
  const uint32_t w1[8] = {c10.x, c10.y, c10.z, c10.w, c11.x, c11.y, c11.z, c11.w};
  // each scale byte duplicated, then converted: f16x2 {s, s}
  const uint32_t d0a = __byte_perm(s0, 0, 0x1100), d0b = __byte_perm(s0, 0, 0x3322);
  const uint32_t d1a = __byte_perm(s1, 0, 0x1100), d1b = __byte_perm(s1, 0, 0x3322);
  const uint32_t sc0[4] = {e4m3x2_to_f16x2(d0a), e4m3x2_to_f16x2(d0a >> 16), e4m3x2_to_f16x2(d0b),
                           e4m3x2_to_f16x2(d0b >> 16)};
  const uint32_t sc1[4] = {e4m3x2_to_f16x2(d1a), e4m3x2_to_f16x2(d1a >> 16), e4m3x2_to_f16x2(d1b),
                           e4m3x2_to_f16x2(d1b >> 16)};
#pragma unroll
  for (int wd = 0; wd < 8; ++wd) {
    uint32_t h0[4], h1[4];
    e2m1x8_to_f16x2x4(w0[wd], h0);
    e2m1x8_to_f16x2x4(w1[wd], h1);
    const uint32_t cc0 = sc0[wd >> 1], cc1 = sc1[wd >> 1];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int i = 2 * wd + hh;
      const uint32_t a0 = hmul2(h0[2 * hh], cc0);      // row g,   k = 4i, 4i+1
      const uint32_t a1 = hmul2(h1[2 * hh], cc1);      // row g+8, k = 4i, 4i+1
      const uint32_t a2 = hmul2(h0[2 * hh + 1], cc0);  // row g,   k = 4i+2, 4i+3
      const uint32_t a3 = hmul2(h1[2 * hh + 1], cc1);  // row g+8, k = 4i+2, 4i+3
      constexpr int NSET = 4 / NTILE;
#pragma unroll
      for (int nt = 0; nt < NTILE; ++nt) {
        uint2 bb = make_uint2(0u, 0u);
        if (!PRED || xon[nt]) bb = *reinterpret_cast<const uint2*>(sx + (xcol[nt] + xg) + 8 * i);
        mma16816(acc[(i % NSET) * NTILE + nt], a0, a1, a2, a3, bb.x, bb.y);
      }
    }
  }
}

// Block-diagonal step (class MC 0: two B streams -- hi and lo plane of one
// token, or the hi planes of two tokens). The lanes read the same 64
// elements of rows r and r+8 as in compute_step and MMA i covers the same K
// slots, but the A fragments are the raw E2M1 values (no scale multiply):
// B column g is (lane quad g >> 1, stream g & 1) and is nonzero only in that
// quad's K slots, so after the four MMAs of one scale block per quad (MMA
// 4j..4j+3 hold elements 16j..16j+15 of lane quad t's 64, i.e. scale block
// 4t + j of the step), column (t, s) of the product is the exact dot product
// of one 16-element block of codes with stream s; it is multiplied by that
// block's E4M3 scale in fp32 and added to the lane's accumulator (set j & 1).
// bon: this lane supplies B (g >> 1 == t); sxc: its stream's column.
__device__ __forceinline__ void compute_step_bd(const uint8_t* sw, const uint8_t* ss, int r, float (*acc)[4],
                                                const uint8_t* sxc, bool bon, uint32_t xg, int t) {
  const int r1 = r + 8;
  const uint4 c00 = *reinterpret_cast<const uint4*>(sw + r * 128 + (((2 * t) ^ (r & 7)) << 4));
  const uint4 c01 = *reinterpret_cast<const uint4*>(sw + r * 128 + (((2 * t + 1) ^ (r & 7)) << 4));
  const uint4 c10 = *reinterpret_cast<const uint4*>(sw + r1 * 128 + (((2 * t) ^ (r1 & 7)) << 4));
  const uint4 c11 = *reinterpret_cast<const uint4*>(sw + r1 * 128 + (((2 * t + 1) ^ (r1 & 7)) << 4));
  const uint32_t s0 = *reinterpret_cast<const uint32_t*>(ss + r * 16 + 4 * t);
  const uint32_t s1 = *reinterpret_cast<const uint32_t*>(ss + r1 * 16 + 4 * t);
  const uint32_t w0[8] = {c00.x, c00.y, c00.z, c00.w, c01.x, c01.y, c01.z, c01.w};
  const uint32_t w1[8] = {c10.x, c10.y, c10.z, c10.w, c11.x, c11.y, c11.z, c11.w};
  // the four block scales of each row, exactly, in fp32
  const float2 fa = f16x2_to_float2(e4m3x2_to_f16x2(s0)), fb = f16x2_to_float2(e4m3x2_to_f16x2(s0 >> 16));
  const float2 fc = f16x2_to_float2(e4m3x2_to_f16x2(s1)), fd = f16x2_to_float2(e4m3x2_to_f16x2(s1 >> 16));
  const float f0[4] = {fa.x, fa.y, fb.x, fb.y}, f1[4] = {fc.x, fc.y, fd.x, fd.y};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float d[4];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int wd = 2 * j + q;
      uint32_t h0[4], h1[4];
      e2m1x8_to_f16x2x4(w0[wd], h0);
      e2m1x8_to_f16x2x4(w1[wd], h1);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int i = 2 * wd + hh;
        uint2 bb = make_uint2(0u, 0u);
        if (bon) bb = *reinterpret_cast<const uint2*>(sxc + xg + 8 * i);
        if (i % 4 == 0) mma16816_z(d, h0[2 * hh], h1[2 * hh], h0[2 * hh + 1], h1[2 * hh + 1], bb.x, bb.y);
        else mma16816(d, h0[2 * hh], h1[2 * hh], h0[2 * hh + 1], h1[2 * hh + 1], bb.x, bb.y);
      }
    }
    float* a = acc[j & 1];
    a[0] = fmaf(f0[j], d[0], a[0]);
    a[1] = fmaf(f0[j], d[1], a[1]);
    a[2] = fmaf(f1[j], d[2], a[2]);
    a[3] = fmaf(f1[j], d[3], a[3]);
  }
}

// FP8 step: the same K mapping as compute_step (lane quad t holds elements
// 64t..64t+63 of rows r and r+8, MMA i takes 64t + 4i + {0..3}), on E4M3
// codes: one cvt.rn.f16x2.e4m3x2 per pair of codes is the exact A fragment
// (the row scale is applied to the finished sums). Elements 64t.. sit in
// half t >> 1 of the stage, 16-byte chunks 4 (t & 1) .. 4 (t & 1) + 3.
template <int NTILE, bool PRED>
__device__ __forceinline__ void compute_step_fp8(const uint8_t* sw, int r, float (*acc)[4], const uint8_t* sx,
                                                 const uint32_t* xcol, const bool* xon, uint32_t xg, int t) {
  const int r1 = r + 8;
  const uint8_t* hb = sw + (t >> 1) * (TROWS * 128);
  const int cb = 4 * (t & 1);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 c0 = *reinterpret_cast<const uint4*>(hb + r * 128 + (((cb + j) ^ (r & 7)) << 4));
    const uint4 c1 = *reinterpret_cast<const uint4*>(hb + r1 * 128 + (((cb + j) ^ (r1 & 7)) << 4));
    const uint32_t w0[4] = {c0.x, c0.y, c0.z, c0.w}, w1[4] = {c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = 4 * j + q;
      const uint32_t a0 = e4m3x2_to_f16x2(w0[q]);         // row r,   k = 4i, 4i+1
      const uint32_t a1 = e4m3x2_to_f16x2(w1[q]);         // row r+8, k = 4i, 4i+1
      const uint32_t a2 = e4m3x2_to_f16x2(w0[q] >> 16);   // row r,   k = 4i+2, 4i+3
      const uint32_t a3 = e4m3x2_to_f16x2(w1[q] >> 16);   // row r+8, k = 4i+2, 4i+3
      constexpr int NSET = 4 / NTILE;
#pragma unroll
      for (int nt = 0; nt < NTILE; ++nt) {
        uint2 bb = make_uint2(0u, 0u);
        if (!PRED || xon[nt]) bb = *reinterpret_cast<const uint2*>(sx + (xcol[nt] + xg) + 8 * i);
        mma16816(acc[(i % NSET) * NTILE + nt], a0, a1, a2, a3, bb.x, bb.y);
      }
    }
  }
}

// Consumer warp's walk over the CTA's units. MC = token class (1: M <= 4,
// 2: M <= 8, 3: M <= 16); NTILE token tiles per A fragment (1: hi and lo in
// one tile; 2: hi + lo tiles, or two hi tiles; 4: two hi + two lo tiles).
// Pieces of split tiles are written to the workspace and handed to the
// settler warp through the queue (mbarriers q_full / q_empty).
template <int MC, int NTILE, bool LO, bool XR, int EPI, int FMT>
__device__ __forceinline__ void consume(const Params& p, uint8_t* sW, uint8_t* sS, const uint8_t* sX,
                                        const int* emax, uint32_t b_full, uint32_t b_empty,
                                        uint32_t b_qfull, uint32_t b_qempty,
                                        volatile int* abort_flag, uint32_t* skip,
                                        const volatile uint32_t* pre_flag, const float* pre_buf, int s,
                                        int cnt, int a, int b, int L, int cw, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const int r = 16 * cw + g;                           // row of the tile (and r + 8)
  // tokens of this lane's accumulator values (columns 2t, 2t+1 of a tile):
  // e = 0, 1 from the first token tile, e = 2, 3 from the second (M > 8)
  auto tok = [t](int e) { return tok_of<MC>(t, e); };
  // X column of each token tile for this lane (B column g); shared memory
  // holds only the 2M used columns: hi plane tokens 0..M-1, then lo plane.
  // LO: some lo element is nonzero, lanes of absent tokens skip their loads
  // (B = 0); otherwise the lo plane is all zero, the M <= 8 and M <= 16
  // classes issue hi tiles only, and absent tokens read lo column 0 (zeros)
  // so no load is predicated.
  uint32_t xcol[NTILE];
  bool xon[NTILE];
#pragma unroll
  for (int nt = 0; nt < NTILE; ++nt) {
    int plane, tk;
    if (MC == 0) { plane = 0; tk = 0; }               // set below
    else if (MC == 1) { plane = g >> 2; tk = g & 3; }
    else if (MC == 2) { plane = LO ? nt : 0; tk = g; }
    else if (LO) { plane = nt >> 1; tk = 8 * (nt & 1) + g; }
    else { plane = 0; tk = 8 * nt + g; }
    const bool valid = tk < p.M;
    xon[nt] = valid;
    // column stride: the slice's column (staged X) or one K-step box (X in the ring)
    const uint32_t cstride = XR ? uint32_t(p.xbox_words * 4) : uint32_t(p.xstride);
    if (LO) xcol[nt] = uint32_t(plane * p.M + (valid ? tk : 0)) * cstride;
    else xcol[nt] = uint32_t(valid ? plane * p.M + tk : p.M) * cstride;
    if (MC == 0) {
      // stream g & 1 is column g & 1: hi and lo of token 0 (M = 1) or the hi
      // planes of tokens 0 and 1 (M = 2, no lo plane)
      xcol[nt] = uint32_t(g & 1) * cstride;
      xon[nt] = (g >> 1) == t;
    }
  }
  float acc[4][4];
#pragma unroll
  for (int q = 0; q < 4; ++q) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0.0f;
  int st = 0;                                          // ring stage and its phase
  uint32_t ph = 0;
  int seg_start = a;
  int nsplit = 0;                                      // split segments handed to the settler
  int tile = a / cnt, j = a - tile * cnt;
  const int pre_tile = MC <= 1 ? prefetch_tile(p, a, b, cnt, L) : -1;
  for (int idx = a; idx < b; ++idx) {
    const bool ok = wait_bar(b_full + 8 * st, ph, abort_flag, p, ST_TIMEOUT_CONSUMER);
    if (!__all_sync(0xffffffffu, ok)) break;
    // The slot is released after the MMAs. (Releasing it as soon as the
    // weights are in registers measured ~2% slower at M = 1, and is not
    // possible with X in the ring, which is read during the MMAs.)
    constexpr bool EARLY = false;
    // lane t reads 64-element group t of this step (staged X: of the slice)
    const uint32_t xg = uint32_t(XGROUP_BYTES * (XR ? t : 4 * j + t));
    if constexpr (FMT == FMT_FP8)
      compute_step_fp8<NTILE, LO>(sW + st * W_BYTES_FP8, r, acc, XR ? sX + st * p.xbytes : sX, xcol, xon, xg, t);
    else if constexpr (MC == 0)
      compute_step_bd(sW + st * W_BYTES, sS + st * S_BYTES, r, acc, (XR ? sX + st * p.xbytes : sX) + xcol[0],
                      xon[0], xg, t);
    else
      compute_step<NTILE, EARLY, LO>(sW + st * W_BYTES, sS + st * S_BYTES, r, acc,
                                     XR ? sX + st * p.xbytes : sX, xcol, xon, xg, t,
                                     b_empty + 8 * st, lane);
    if (!EARLY) {
      __syncwarp();
      if (lane == 0) mbar_arrive(b_empty + 8 * st);
    }
    if (++st == p.nstage) { st = 0; ph ^= 1u; }
    const int jcur = j;
    const int tcur = tile;
    if (++j == cnt) { j = 0; ++tile; }
    const bool seg_last = (idx + 1 == b) || (jcur + 1 == cnt);
    if (!seg_last) continue;

    // ------------------------------------------------------ segment epilogue
    // add the accumulator sets of each tile (fixed order)
    constexpr int NSET = 4 / NTILE;
    float at[4][4];
#pragma unroll
    for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float sum = acc[nt][e];
#pragma unroll
        for (int q = 1; q < NSET; ++q) sum += acc[q * NTILE + nt][e];
        at[nt][e] = sum;
      }
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0.0f;
    // per-token values of this lane: v[e][0] row r, v[e][1] row r+8; the
    // planes' scales 2^-sh (hi) and 2^-(sh + LO_SHIFT) (lo) undone here
    float fh[4], fl[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int m = tok(e);
      fh[e] = fl[e] = 0.0f;
      if (m >= 0 && m < p.M && emax[m] != INT_MIN) {
        const int sh = 14 - emax[m];
        fh[e] = ldexpf(1.0f, -sh);
        fl[e] = ldexpf(1.0f, -(sh + LO_SHIFT));
      }
    }
    const float gs = *p.gs;
    float v[4][2];
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e][0] = v[e][1] = 0.0f;
    if (MC == 0) {
      // block-diagonal: the lanes of a quad hold disjoint blocks of the same
      // rows; add them (fixed order), then undo the planes' scales
      float bt[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        bt[e] = at[0][e];
        bt[e] += __shfl_xor_sync(0xffffffffu, bt[e], 1);
        bt[e] += __shfl_xor_sync(0xffffffffu, bt[e], 2);
      }
      const float h0 = emax[0] == INT_MIN ? 0.0f : ldexpf(1.0f, emax[0] - 14);
      if (p.M == 1) {
        const float l0 = h0 * (1.0f / 536870912.0f);          // 2^-LO_SHIFT
        v[0][0] = bt[0] * h0 + bt[1] * l0;
        v[0][1] = bt[2] * h0 + bt[3] * l0;
      } else {
        const float h1 = emax[1] == INT_MIN ? 0.0f : ldexpf(1.0f, emax[1] - 14);
        v[0][0] = bt[0] * h0; v[1][0] = bt[1] * h1;
        v[0][1] = bt[2] * h0; v[1][1] = bt[3] * h1;
      }
    } else if (MC == 1) {
      // one tile: columns 0..3 hi tokens 0..3, 4..7 lo tokens 0..3; lo partner lane t^2
      float o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] = __shfl_xor_sync(0xffffffffu, at[0][e], 2);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        v[e][0] = at[0][e] * fh[e] + o[e] * fl[e];
        v[e][1] = at[0][2 + e] * fh[e] + o[2 + e] * fl[e];
      }
    } else if (MC == 2) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float l0 = NTILE == 2 ? at[1 % NTILE][e] : 0.0f, l1 = NTILE == 2 ? at[1 % NTILE][2 + e] : 0.0f;
        v[e][0] = at[0][e] * fh[e] + l0 * fl[e];
        v[e][1] = at[0][2 + e] * fh[e] + l1 * fl[e];
      }
    } else {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float l0 = NTILE == 4 ? at[2 % NTILE][e] : 0.0f, l1 = NTILE == 4 ? at[2 % NTILE][2 + e] : 0.0f;
        const float l2 = NTILE == 4 ? at[3 % NTILE][e] : 0.0f, l3 = NTILE == 4 ? at[3 % NTILE][2 + e] : 0.0f;
        v[e][0] = at[0][e] * fh[e] + l0 * fl[e];
        v[e][1] = at[0][2 + e] * fh[e] + l1 * fl[e];
        v[2 + e][0] = at[1 % NTILE][e] * fh[2 + e] + l2 * fl[2 + e];
        v[2 + e][1] = at[1 % NTILE][2 + e] * fh[2 + e] + l3 * fl[2 + e];
      }
    }
    if constexpr (FMT == FMT_FP8) {
      // the rows' fp32 scales (rows past N read nothing)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int n = tcur * TROWS + r + 8 * h;
        const float rs = n < p.N ? __ldg(p.row_scale + n) : 0.0f;
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e][h] *= rs;
      }
    }
    if (p.act4) {
      // W4A4: the per-tensor scale of the quantised X (X in the ring: from
      // k_xprep in the workspace; staged X: in the CTA's misc area, next to emax)
      const float gsx = XR ? *p.xgs
                           : *reinterpret_cast<const float*>(reinterpret_cast<const uint8_t*>(emax) - MISC_EMAX + MISC_XGS);
#pragma unroll
      for (int e = 0; e < 4; ++e) { v[e][0] *= gsx; v[e][1] *= gsx; }
    }
    const int this_start = seg_start;
    seg_start = idx + 1;
    const bool whole = (p.S == 1) && (this_start == tcur * cnt) && (jcur + 1 == cnt);
    const int row0 = tcur * TROWS + r;
    if (whole) {
      emit_rows<MC, EPI>(p, row0, v, gs, lane);
      continue;
    }
    // piece of a split tile
    const int qs = nsplit % QN;
    if (nsplit >= QN) {
      const bool okq = wait_bar(b_qempty + 8 * qs, uint32_t((nsplit / QN) - 1) & 1u, abort_flag, p,
                                ST_TIMEOUT_CONSUMER);
      if (!__all_sync(0xffffffffu, okq)) break;
    }
    const int ord = bnd_in(tcur * cnt, this_start, L, p.P);
    bool done_here = false;
    if (MC <= 1 && tcur == pre_tile && ord == 0 && idx + 1 == b &&
        __all_sync(0xffffffffu, *pre_flag != 0u)) {
      // the settler has copied the other piece into shared memory
      __threadfence_block();
      float sum[4][2];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int m = tok(e);
        const bool ok_m = m >= 0 && m < p.M;
        sum[e][0] = v[e][0] + (ok_m ? pre_buf[m * TROWS + r] : 0.0f);
        sum[e][1] = v[e][1] + (ok_m ? pre_buf[m * TROWS + r + 8] : 0.0f);
      }
      emit_rows<MC, EPI>(p, row0, sum, gs, lane);
      __syncwarp();
      if (lane == 0) *reinterpret_cast<volatile uint32_t*>(p.counters + tcur * NCW + cw) = 0u;
      done_here = true;
    } else if (p.S == 1 && ord == 0 && idx + 1 == b) {
      // The CTA's last segment holds the tile's first k-range. The other
      // pieces were the first segments of the next CTAs and are usually
      // counted by now: then this warp adds them to its registers and stores
      // its rows without writing a partial.
      const int np = 1 + bnd_in(tcur * cnt, (tcur + 1) * cnt - 1, L, p.P);
      if (np - 1 <= FAST_MAX) {
        uint32_t* ctr = p.counters + tcur * NCW + cw;
        const uint32_t seen = ld_relaxed_gpu(ctr);
        if (__all_sync(0xffffffffu, seen == uint32_t(np - 1))) {
          fence_acq_rel_gpu();                       // with the relaxed load: acquire
          float sum[4][2];
#pragma unroll
          for (int e = 0; e < 4; ++e) { sum[e][0] = v[e][0]; sum[e][1] = v[e][1]; }
#pragma unroll
          for (int o = 1; o <= FAST_MAX; ++o) {
            if (o < np) {
              const float* part = p.partials + ((long long)tcur * p.pmax + o) * p.M * TROWS;
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int m = tok(e);
                if (m >= 0 && m < p.M) {
                  sum[e][0] += __ldcg(part + m * TROWS + r);
                  sum[e][1] += __ldcg(part + m * TROWS + r + 8);
                }
              }
            }
          }
          emit_rows<MC, EPI>(p, row0, sum, gs, lane);
          __syncwarp();
          if (lane == 0) *reinterpret_cast<volatile uint32_t*>(ctr) = 0u;
          done_here = true;
        }
      }
    }
    if (!done_here) {
      const long long slot = ((long long)tcur * p.S + s) * p.pmax + ord;
      float* part = p.partials + slot * p.M * TROWS;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int m = tok(e);
        if (m >= 0 && m < p.M) {
          part[m * TROWS + r] = v[e][0];
          part[m * TROWS + r + 8] = v[e][1];
        }
      }
    }
    __syncwarp();
    if (lane == 0) {
      if (done_here) atomicOr(&skip[qs], 1u << cw);
      mbar_arrive(b_qfull + 8 * qs);
    }
    ++nsplit;
  }
}

// Settler warp: walks the same segments as the consumers. For each split
// piece, once all consumer warps have written their rows (or finished them
// in place, see the skip mask), it counts the piece on each row group's
// counter (a gpu-scope fence first: the mbarrier wait ordered the consumers'
// partial stores before it, and fences are cumulative). Row groups for which
// this CTA brought the last piece are listed for the end phase, where all
// warps of the CTA add the pieces; if the list is full the settler adds them
// itself.
template <int EPI>
__device__ __forceinline__ void settle(const Params& p, uint32_t b_qfull, uint32_t b_qempty,
                                       volatile int* abort_flag, uint32_t* skip, uint32_t* list,
                                       uint32_t* nlist, uint32_t* pieces, volatile uint32_t* pre_flag,
                                       float* pre_buf, int cnt, int a, int b, int L, int lane) {
  const int pre_tile = prefetch_tile(p, a, b, cnt, L);
  int nsplit = 0;
  int seg_start = a;
  int tile = a / cnt, j = a - tile * cnt;
  for (int idx = a; idx < b; ++idx) {
    const int tcur = tile, jcur = j;
    if (++j == cnt) { j = 0; ++tile; }
    if (!((idx + 1 == b) || (jcur + 1 == cnt))) continue;
    const int this_start = seg_start;
    seg_start = idx + 1;
    const bool whole = (p.S == 1) && (this_start == tcur * cnt) && (jcur + 1 == cnt);
    if (whole) continue;
    const int qs = nsplit % QN;
    const uint32_t qpar = uint32_t(nsplit / QN) & 1u;
    if (tcur == pre_tile && idx + 1 == b) {
      // While the consumers work on the last piece: if the other piece of
      // this tile (the next CTA's first segment) gets counted on every row
      // group first, copy it into shared memory for the consumers.
      bool copied = false;
      const long long t0 = clock64();
      while (!__any_sync(0xffffffffu, mbar_test(b_qfull + 8 * qs, qpar))) {
        if (!copied) {
          const bool ready = lane >= NCW || ld_acquire_gpu(p.counters + tcur * NCW + lane) == 1u;
          if (__all_sync(0xffffffffu, ready)) {
            const float* part = p.partials + ((long long)tcur * p.pmax + 1) * p.M * TROWS;
            for (int u = lane; u < p.M * TROWS; u += 32) pre_buf[u] = __ldcg(part + u);
            __syncwarp();
            __threadfence_block();
            if (lane == 0) *pre_flag = 1u;
            copied = true;
          }
        }
        if (*abort_flag || clock64() - t0 > p.timeout) break;   // wait_bar below reports it
        __nanosleep(200);
      }
    }
    const bool ok = wait_bar(b_qfull + 8 * qs, qpar, abort_flag, p, ST_TIMEOUT_SETTLER, 20000);
    if (!__all_sync(0xffffffffu, ok)) return;
    // total pieces of the tile over all slices
    int npieces = 0;
    for (int s2 = 0; s2 < p.S; ++s2) {
      const int cnt2 = p.ks_base + (s2 < p.ks_rem ? 1 : 0);
      const int L2 = p.tiles * cnt2;
      npieces += 1 + bnd_in(tcur * cnt2, (tcur + 1) * cnt2 - 1, L2, p.P);
    }
    const uint32_t sk = skip[qs];
    bool last = false;
    if (lane < NCW && !((sk >> lane) & 1u)) {
      __threadfence();
      const uint32_t old = atomicAdd(&p.counters[tcur * NCW + lane], 1u);
      last = old == uint32_t(npieces - 1);
      if (last) __threadfence();                 // with the atomic: acquire the other pieces
    }
    const uint32_t lastmask = __ballot_sync(0xffffffffu, last);
    if (lastmask) {
      if (*nlist < uint32_t(LIST_MAX)) {
        if (lane == 0) {
          list[2 * *nlist] = uint32_t(tcur);
          list[2 * *nlist + 1] = lastmask;
          *nlist += 1;
        }
      } else {
        if (lane == 0) pieces[MAX_PIECES] = uint32_t(list_pieces(p, tcur, pieces));
        __syncwarp();
        __threadfence();
        sum_pieces<EPI>(p, tcur, lastmask, pieces, int(pieces[MAX_PIECES]), lane, 32);
        if ((lastmask >> lane) & 1u) p.counters[tcur * NCW + lane] = 0u;
      }
    }
    __syncwarp();
    if (lane == 0) {
      skip[qs] = 0u;
      mbar_arrive(b_qempty + 8 * qs);
    }
    ++nsplit;
  }
}

// XR: X in the ring. Each stage also carries one K-step of the X planes
// (prepared by k_xprep in the workspace), there are no K-slices and no
// staging; otherwise the CTA stages its K-slice of X in shared memory.
template <int MC, bool XR, int EPI, int FMT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
k_mma(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_s,
      const __grid_constant__ CUtensorMap tm_x, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment (128-byte swizzled TMA destinations) by an offset, so
  // every derived pointer stays visibly in the shared window (32-bit shared
  // addressing instead of generic loads)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int nst = p.nstage;
  uint8_t* sW = smem;                                     // nst x 32 KB (1024-aligned)
  uint8_t* sS = smem + nst * w_bytes_of(FMT);             // nst x 4 KB (NVFP4; none for FP8)
  uint8_t* sX = sS + nst * s_bytes_of(FMT);               // staged slice, or nst X boxes
  uint8_t* misc = sX + (XR ? size_t(nst) * p.xbytes : size_t(p.ncols) * p.xstride);
  uint64_t* bars = reinterpret_cast<uint64_t*>(misc);     // full[8] empty[8] qfull[8] qempty[8]
  int* emax = reinterpret_cast<int*>(misc + MISC_EMAX);   // [16]
  uint32_t* flags = reinterpret_cast<uint32_t*>(misc + MISC_FLAGS);  // [0] need_lo [1] abort [2] list count
  uint32_t* skip = reinterpret_cast<uint32_t*>(misc + MISC_SKIP);    // [QN]
  uint32_t* pieces = reinterpret_cast<uint32_t*>(misc + MISC_PIECES);  // [MAX_PIECES + 1]
  uint32_t* list = reinterpret_cast<uint32_t*>(misc + MISC_LIST);    // [LIST_MAX][2]
  volatile uint32_t* pre_flag = reinterpret_cast<volatile uint32_t*>(misc + MISC_PREFLAG);
  float* pre_buf = reinterpret_cast<float*>(misc + MISC_PREBUF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(flags + 1);
  const uint32_t b_full = smem_u32(bars), b_empty = b_full + 8 * NSTAGE_MAX;
  const uint32_t b_qfull = b_empty + 8 * NSTAGE_MAX, b_qempty = b_qfull + 8 * QN;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = blockIdx.x / p.P, c = blockIdx.x % p.P;
  const int cnt = p.ks_base + (s < p.ks_rem ? 1 : 0);
  const int ks0 = s * p.ks_base + min(s, p.ks_rem);
  const int klen = cnt * KS, k0e = ks0 * KS;
  const int L = p.tiles * cnt;
  // whole tiles per CTA (tpc > 0), else an even share of the units (stream-K)
  const int a = p.tpc > 0 ? min(c * p.tpc, p.tiles) * cnt : int((long long)c * L / p.P);
  const int b = p.tpc > 0 ? min((c + 1) * p.tpc, p.tiles) * cnt : int((long long)(c + 1) * L / p.P);

  // Dependent launches (PDL) may start now: they only stream weights until
  // this grid has completed.
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) {
    for (int i = 0; i < nst; ++i) { mbar_init(b_full + 8 * i, 1); mbar_init(b_empty + 8 * i, NCW); }
    for (int i = 0; i < QN; ++i) { mbar_init(b_qfull + 8 * i, NCW); mbar_init(b_qempty + 8 * i, 1); }
    for (int m = 0; m < 16; ++m) emax[m] = INT_MIN;
    flags[0] = 0u; flags[1] = 0u; flags[2] = 0u;
    *pre_flag = 0u;
    *reinterpret_cast<uint32_t*>(misc + MISC_XAMAX) = 0u;
    for (int i = 0; i < QN; ++i) skip[i] = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();

  if (warp == 0) {
    // -------------------------------------------------------------- producer
    // Weights do not depend on the previous grid: stream them at once.
    if (lane == 0) {
      int n_issued = 0;
      const uint64_t pol = l2_evict_first_policy();
      // XR: the first stages' weights go out before the previous grid has
      // completed; their X boxes (written by k_xprep) only after it
      const int pre_n = XR ? min(nst, b - a) : 0;
      bool x_first = !XR;
      if (!p.stall) {
        int tile = a / cnt, j = a - tile * cnt, st = 0;
        uint32_t ph = 0;
        for (int idx = a; idx < b; ++idx, ++n_issued) {
          if (!x_first && n_issued == pre_n) {
            asm volatile("griddepcontrol.wait;" ::: "memory");
            int j2 = a % cnt;
            for (int n = 0; n < pre_n; ++n) {
              tma_load_2d(smem_u32(sX + n * p.xbytes), &tm_x, (ks0 + j2) * p.xbox_words, 0, b_full + 8 * n);
              if (++j2 == cnt) j2 = 0;
            }
            x_first = true;
          }
          if (!wait_bar(b_empty + 8 * st, ph ^ 1u, abort_flag, p, ST_TIMEOUT_PRODUCER)) break;
          // the X box delivers exactly xbox_bytes (2M columns of one K-step)
          mbar_expect_tx(b_full + 8 * st, w_bytes_of(FMT) + s_bytes_of(FMT) + (XR ? p.xbox_bytes : 0));
          if constexpr (FMT == FMT_FP8) {
            // two 128-byte-wide halves of the 256 codes of each row
            tma_load_2d_hint(smem_u32(sW + st * W_BYTES_FP8), &tm_w, (ks0 + j) * KS, tile * TROWS,
                             b_full + 8 * st, pol);
            tma_load_2d_hint(smem_u32(sW + st * W_BYTES_FP8 + TROWS * 128), &tm_w, (ks0 + j) * KS + 128,
                             tile * TROWS, b_full + 8 * st, pol);
          } else {
            tma_load_2d_hint(smem_u32(sW + st * W_BYTES), &tm_w, (ks0 + j) * (KS / 2), tile * TROWS,
                             b_full + 8 * st, pol);
            tma_load_2d_hint(smem_u32(sS + st * S_BYTES), &tm_s, (ks0 + j) * (KS / 16), tile * TROWS,
                             b_full + 8 * st, pol);
          }
          if (XR && x_first)
            tma_load_2d(smem_u32(sX + st * p.xbytes), &tm_x, (ks0 + j) * p.xbox_words, 0, b_full + 8 * st);
          if (++j == cnt) { j = 0; ++tile; }
          if (++st == nst) { st = 0; ph ^= 1u; }
        }
        if (!x_first && n_issued == pre_n) {
          asm volatile("griddepcontrol.wait;" ::: "memory");
          int j2 = a % cnt;
          for (int n = 0; n < pre_n; ++n) {
            tma_load_2d(smem_u32(sX + n * p.xbytes), &tm_x, (ks0 + j2) * p.xbox_words, 0, b_full + 8 * n);
            if (++j2 == cnt) j2 = 0;
          }
          x_first = true;
        }
      }
      if (*abort_flag) {
        // wait (bounded) for the loads still in flight before leaving
        const int first = n_issued > nst ? n_issued - nst : 0;
        for (int i = first; i < n_issued; ++i)
          drain_bar(b_full + 8 * (i % nst), uint32_t(i / nst) & 1u, p);
      }
    }
    __syncwarp();
    asm volatile("griddepcontrol.wait;" ::: "memory");   // before the end phase
  } else if (warp == WARP_SETTLE) {
    // ---------------------------------------------------------------- settler
    asm volatile("griddepcontrol.wait;" ::: "memory");   // counters of the previous grid
    settle<EPI>(p, b_qfull, b_qempty, abort_flag, skip, list, flags + 2, pieces, pre_flag, pre_buf, cnt, a, b, L, lane);
  } else {
    // ------------------------------------------------ consumers: stage X first
    // X, the global scale, Y and the workspace may belong to the previous grid
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int cw = warp - 1;
#define NVFP4_CONSUME(MC_, NT_, LO_, XR_, EMAX_) \
  consume<MC_, NT_, LO_, XR_, EPI, FMT>(p, sW, sS, sX, EMAX_, b_full, b_empty, b_qfull, b_qempty, abort_flag, skip, pre_flag, pre_buf, s, cnt, a, b, L, cw, lane)
    if constexpr (XR) {
      // X arrives with the weights; exponents and lo flags come from k_xprep
      bool need_lo = false;
      for (int c = 0; c < p.xchunks; ++c)
        for (int m = 0; m < p.M; ++m) need_lo |= p.xlo[16 * c + m] != 0u;
      if constexpr (MC == 1) {
        if (FMT == FMT_NVFP4 && (p.M == 1 || (p.M == 2 && !need_lo))) NVFP4_CONSUME(0, 1, false, true, p.xemax);
        else if (need_lo) NVFP4_CONSUME(1, 1, true, true, p.xemax); else NVFP4_CONSUME(1, 1, false, true, p.xemax);
      } else if constexpr (MC == 2) {
        if (need_lo) NVFP4_CONSUME(2, 2, true, true, p.xemax); else NVFP4_CONSUME(2, 1, false, true, p.xemax);
      } else if constexpr (MC == 3) {
        if (need_lo) NVFP4_CONSUME(3, 4, true, true, p.xemax); else NVFP4_CONSUME(3, 2, false, true, p.xemax);
      }
    } else {
    const int ctid = threadIdx.x - 32;                    // 0 .. NCW*32-1
    constexpr int NCT = NCW * 32;
    // Only the K-steps of the slice that this CTA's units touch are staged:
    // nx_steps of them, circularly from step j0x (a range shorter than a
    // tile's K either lies in one tile or wraps from the end of one tile to
    // the start of the next). The exponent maximum is taken over them too:
    // the planes' scales are undone before any sum leaves the CTA.
    const int nx_steps = min(cnt, b - a), j0x = a % cnt;
    const int nx = nx_steps * (KS / 8);                  // 16-byte chunks per token
    auto chunk_of = [&](int rem) {
      int st = j0x + (rem >> 5);
      if (st >= cnt) st -= cnt;
      return st * (KS / 8) + (rem & 31);
    };
    static_assert(KS / 8 == 32, "chunk_of: 32 chunks of 8 elements per K-step");
    const int nreal = p.M * nx;
    if (!p.act4) {
    // 1. X slice -> shared memory as raw bf16, in the hi plane's places, and
    //    the per-token exponent maximum (lanes holding the same token reduce
    //    in the warp: one shared-memory atomic per token and warp)
    for (int base = ctid & ~31; base < nreal; base += 2 * NCT) {   // warp-uniform bound
      uint4 xv[2];
      int mm[2], kk[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int u = base + (ctid & 31) + h * NCT;
        mm[h] = -1;
        if (u < nreal) {
          mm[h] = u / nx;
          kk[h] = chunk_of(u - mm[h] * nx);
          xv[h] = *reinterpret_cast<const uint4*>(p.x + size_t(mm[h]) * p.K + k0e + 8 * kk[h]);
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t mag = 0u;
        if (mm[h] >= 0) {
          uint8_t* ch = sX + size_t(mm[h]) * p.xstride;
          *reinterpret_cast<uint2*>(ch + x_off(8 * kk[h])) = make_uint2(xv[h].x, xv[h].y);
          *reinterpret_cast<uint2*>(ch + x_off(8 * kk[h] + 4)) = make_uint2(xv[h].z, xv[h].w);
          mag = bf16_mag_max8(xv[h]);
        }
        const unsigned grp = __match_any_sync(0xffffffffu, mm[h]);
        const int gmx = bf16_mag_exp(__reduce_max_sync(grp, mag));
        if (mm[h] >= 0 && gmx != INT_MIN && (threadIdx.x & 31) == __ffs(grp) - 1) atomicMax(&emax[mm[h]], gmx);
      }
    }
    named_bar(BAR_CONSUMERS, NCT);
    // 2. in place: raw bf16 -> hi plane, and the lo plane next to it
    bool lo_used = false;
#pragma unroll 1
    for (int u = ctid; u < nreal; u += NCT) {
      const int m = u / nx, kc = chunk_of(u - m * nx);
      const int sh = (emax[m] == INT_MIN) ? 0 : 14 - emax[m];
      const uint32_t o0 = x_off(8 * kc), o1 = x_off(8 * kc + 4);
      uint8_t* ch = sX + size_t(m) * p.xstride;
      uint8_t* cl = sX + size_t(p.M + m) * p.xstride;
      const uint2 r0 = *reinterpret_cast<const uint2*>(ch + o0), r1 = *reinterpret_cast<const uint2*>(ch + o1);
      const uint32_t w[4] = {r0.x, r0.y, r1.x, r1.y};
      uint32_t hi[4], lo[4];
      lo_used |= x_split8(w, sh, hi, lo);
      *reinterpret_cast<uint2*>(ch + o0) = make_uint2(hi[0], hi[1]);
      *reinterpret_cast<uint2*>(ch + o1) = make_uint2(hi[2], hi[3]);
      *reinterpret_cast<uint2*>(cl + o0) = make_uint2(lo[0], lo[1]);
      *reinterpret_cast<uint2*>(cl + o1) = make_uint2(lo[2], lo[3]);
    }
    if (lo_used) atomicOr(&flags[0], 1u);
    named_bar(BAR_CONSUMERS, NCT);
    } else {
      // W4A4: X is quantised to NVFP4 here by the weights' quantiser steps,
      // under the per-tensor scale gs_x = amax(|X|) / 2688 of this X (every
      // CTA reads all of X for it, so all CTAs agree). B is the exact f16
      // product e2m1(code) * e4m3(scale) of each element (the lo plane stays
      // zero, the per-token factor is 1) and gs_x multiplies the sums.
      uint32_t* amax_s = reinterpret_cast<uint32_t*>(misc + MISC_XAMAX);
      const int per_tok = p.K / 8;
      uint32_t mag = 0u;
      for (int u = ctid; u < p.M * per_tok; u += NCT) {
        const int m = u / per_tok;
        mag = max(mag, bf16_mag_max8(*reinterpret_cast<const uint4*>(p.x + size_t(m) * p.K + 8 * (u - m * per_tok))));
      }
      mag = __reduce_max_sync(0xffffffffu, mag);
      if ((ctid & 31) == 0) atomicMax(amax_s, mag);
      named_bar(BAR_CONSUMERS, NCT);
      const float gsx = __fdiv_rn(__uint_as_float(*amax_s << 16), 2688.0f);   // 6 * 448
      // 16-element blocks of the staged K-steps: chunk pairs (2i, 2i+1) of a token
      const int nbt = nx / 2;
      for (int u = ctid; u < p.M * nbt; u += NCT) {
        const int m = u / nbt, kc = chunk_of(2 * (u - m * nbt));
        const uint16_t* src = p.x + size_t(m) * p.K + k0e + 8 * kc;
        const uint4 xa = *reinterpret_cast<const uint4*>(src), xb = *reinterpret_cast<const uint4*>(src + 8);
        const uint32_t wv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
        float v[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          v[2 * i] = __uint_as_float(wv[i] << 16);
          v[2 * i + 1] = __uint_as_float(wv[i] & 0xFFFF0000u);
        }
        uint32_t s_code, q[2];
        quantize_block16(v, gsx, s_code, q);
        const uint32_t sc = bcast_lo(e4m3x2_to_f16x2(s_code));
        uint32_t h[8];
        e2m1x8_to_f16x2x4(q[0], h);
        e2m1x8_to_f16x2x4(q[1], h + 4);
#pragma unroll
        for (int i = 0; i < 8; ++i) h[i] = hmul2(h[i], sc);   // exact products
        uint8_t* ch = sX + size_t(m) * p.xstride;
        uint8_t* cl = sX + size_t(p.M + m) * p.xstride;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          *reinterpret_cast<uint2*>(ch + x_off(8 * kc + 4 * c)) = make_uint2(h[2 * c], h[2 * c + 1]);
          *reinterpret_cast<uint2*>(cl + x_off(8 * kc + 4 * c)) = make_uint2(0u, 0u);
        }
      }
      if (ctid == 0) {
        *reinterpret_cast<float*>(misc + MISC_XGS) = gsx;
        for (int m = 0; m < p.M; ++m) emax[m] = 14;
      }
      named_bar(BAR_CONSUMERS, NCT);
    }
    const bool need_lo = flags[0] != 0u;

    if constexpr (MC == 1) {
      if (FMT == FMT_NVFP4 && (p.M == 1 || (p.M == 2 && !need_lo))) NVFP4_CONSUME(0, 1, false, false, emax);
      else if (need_lo) NVFP4_CONSUME(1, 1, true, false, emax); else NVFP4_CONSUME(1, 1, false, false, emax);
    } else if constexpr (MC == 2) {
      if (need_lo) NVFP4_CONSUME(2, 2, true, false, emax); else NVFP4_CONSUME(2, 1, false, false, emax);
    } else {
      if (need_lo) NVFP4_CONSUME(3, 4, true, false, emax); else NVFP4_CONSUME(3, 2, false, false, emax);
    }
    }
#undef NVFP4_CONSUME
  }
  __syncthreads();
  // ------------------------------------------------------------- end phase
  // every warp adds the pieces of the row groups this CTA completed last
  if (!*abort_flag) {
    const int nl = int(flags[2]);
    for (int e = 0; e < nl; ++e) {
      const int tile = int(list[2 * e]);
      const uint32_t gmask = list[2 * e + 1];
      if (threadIdx.x == 0) pieces[MAX_PIECES] = uint32_t(list_pieces(p, tile, pieces));
      __syncthreads();
      sum_pieces<EPI>(p, tile, gmask, pieces, int(pieces[MAX_PIECES]), threadIdx.x, NUM_THREADS);
      if (threadIdx.x < NCW && ((gmask >> threadIdx.x) & 1u)) p.counters[tile * NCW + threadIdx.x] = 0u;
      __syncthreads();
    }
  }
  if constexpr (EPI == EPI_ARGMAX) {
    // the last CTA to finish turns the per-token keys into (index, value)
    __syncthreads();
    if (threadIdx.x == 0 && !*abort_flag) {
      __threadfence();
      if (atomicAdd(p.done, 1u) == gridDim.x - 1) {
        __threadfence();
        int* out_idx = reinterpret_cast<int*>(p.y);
        float* out_val = reinterpret_cast<float*>(out_idx + p.M);
        for (int m = 0; m < p.M; ++m) {
          const unsigned long long key = atomicExch(p.keys + m, 0ull);
          const uint32_t ord = uint32_t(key >> 32);
          out_idx[m] = int(0xFFFFFFFFu - uint32_t(key));
          out_val[m] = __uint_as_float((ord & 0x80000000u) ? (ord & 0x7FFFFFFFu) : ~ord);
        }
        *p.done = 0u;
      }
    }
  }
}

}  // namespace mm

// The kernels' opt-in shared memory (every instantiation the launcher uses).
template <int EPI>
cudaError_t set_smem_attrs(int optin) {
  using namespace mm;
  cudaError_t e = cudaFuncSetAttribute(k_mma<1, false, EPI, FMT_NVFP4>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_mma<1, true, EPI, FMT_NVFP4>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_mma<2, true, EPI, FMT_NVFP4>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_mma<3, true, EPI, FMT_NVFP4>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e == cudaSuccess && EPI == EPI_NONE)
    e = cudaFuncSetAttribute(k_mma<1, false, EPI_NONE, FMT_FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e == cudaSuccess && EPI == EPI_NONE)
    e = cudaFuncSetAttribute(k_mma<2, true, EPI_NONE, FMT_FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e == cudaSuccess && EPI == EPI_NONE)
    e = cudaFuncSetAttribute(k_mma<3, true, EPI_NONE, FMT_FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  return e;
}

// Launch of the main kernel for one epilogue.
template <int EPI>
cudaError_t launch_main(const MmaConfig& c, cudaLaunchConfig_t* cfg, const CUtensorMap& mw, const CUtensorMap& ms,
                        const CUtensorMap& mx, const mm::Params& p) {
  using namespace mm;
  if (c.fmt == FMT_FP8) {
    if (c.M <= 4 && !c.xr) return cudaLaunchKernelEx(cfg, k_mma<1, false, EPI_NONE, FMT_FP8>, mw, ms, mx, p);
    if (c.M >= XR_MIN_M && c.M <= 8) return cudaLaunchKernelEx(cfg, k_mma<2, true, EPI_NONE, FMT_FP8>, mw, ms, mx, p);
    if (c.M > 8) return cudaLaunchKernelEx(cfg, k_mma<3, true, EPI_NONE, FMT_FP8>, mw, ms, mx, p);
    return cudaErrorInvalidConfiguration;
  }
  if (c.M <= 4) {
    if (c.xr) return cudaLaunchKernelEx(cfg, k_mma<1, true, EPI, FMT_NVFP4>, mw, ms, mx, p);
    return cudaLaunchKernelEx(cfg, k_mma<1, false, EPI, FMT_NVFP4>, mw, ms, mx, p);
  }
  if (c.M <= 8) return cudaLaunchKernelEx(cfg, k_mma<2, true, EPI, FMT_NVFP4>, mw, ms, mx, p);
  return cudaLaunchKernelEx(cfg, k_mma<3, true, EPI, FMT_NVFP4>, mw, ms, mx, p);
}

cudaError_t mma_configure(MmaConfig& c, int num_sms) {
  using namespace mm;
  if (c.M < 1 || c.M > 16 || c.K % KS != 0 || c.K <= 0 || c.N <= 0) return cudaErrorInvalidValue;
  if (c.epi < EPI_NONE || c.epi > EPI_ARGMAX || (c.epi == EPI_SWIGLU && c.N % 2 != 0))
    return cudaErrorInvalidConfiguration;
  int dev = 0, optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  c.ncols = 2 * c.M;                        // hi and lo plane of each token
  c.tiles = (c.N + TROWS - 1) / TROWS;
  const int ksteps = c.K / KS;
  // Column stride of a staged X slice: the padded groups, rounded to 32 mod
  // 128 bytes so that columns g and g+1 start 8 banks apart. A K-step box of
  // the X planes (X in the ring) is 4 groups = 544 bytes, also 32 mod 128.
  auto stride_for = [](int ks) {
    const int base = XGROUP_BYTES * (ks * KS / 64);
    return ((base - 32 + 127) / 128) * 128 + 32;
  };
  // Small M: the CTA stages its K-slice of X (2M columns) next to the ring.
  // From XR_MIN_M: 2M columns would force several K-slices; X goes through
  // the ring.
  c.xr = c.M >= XR_MIN_M;
  // FP8 weights: no epilogue, no W4A4. With X in the ring a 64 KB stage and
  // its X box leave room for two stages (still double-buffered).
  if (c.fmt == FMT_FP8 && (c.epi != EPI_NONE || c.act4)) return cudaErrorInvalidConfiguration;
  const int stage_bytes = w_bytes_of(c.fmt) + s_bytes_of(c.fmt);
  const int nstage_min = (c.fmt == FMT_FP8 && c.xr) ? 2 : NSTAGE_MIN;
  int S = 1;
  if (c.xr) {
    c.x_box = 4 * XGROUP_BYTES;
    c.x_pitch = (c.K / 64) * XGROUP_BYTES;
    c.xbytes = ((c.ncols * c.x_box + 127) / 128) * 128;
  } else {
    const long long x_budget = (long long)optin - 1024 - (long long)NSTAGE_MIN * stage_bytes - misc_bytes(c.M);
    auto fits = [&](int ks) { return (long long)c.ncols * stride_for(ks) <= x_budget; };
    if (!fits(1)) return cudaErrorInvalidConfiguration;
    int max_ks = 1;
    while (max_ks < ksteps && fits(max_ks + 1)) ++max_ks;
    S = (ksteps + max_ks - 1) / max_ks;
    c.x_box = 0; c.x_pitch = 0; c.xbytes = 0;
  }
  int P = num_sms / S;
  if (P < 1) return cudaErrorInvalidConfiguration;
  const int ks_base = ksteps / S, ks_rem = ksteps % S;
  const long long min_units = (long long)c.tiles * ks_base;
  if (P > min_units) P = int(min_units);
  // One whole tile per CTA when there are at most as many tiles as SMs and
  // they keep at least 85% of the SMs busy: a split tile costs its pieces a
  // round trip through the workspace and the CTA holding the last piece a
  // wait at the end of the call, which measured more than the idle SMs
  // (decode projection, N = 34816: 136 tiles on 136 SMs, 20 us per call
  // against 23 with stream-K on 148; M = 16: 29 against 36). With several
  // tiles per CTA (lm_head) stream-K over all SMs measured faster.
  c.tpc = 0;
  if (S == 1 && c.tiles <= num_sms && c.tiles * 100 >= num_sms * 85) {
    c.tpc = 1;
    P = c.tiles;
  }
  c.S = S; c.P = P; c.ks_base = ks_base; c.ks_rem = ks_rem;
  c.grid = S * P;
  c.xk_max = (ks_base + (ks_rem ? 1 : 0)) * KS;
  c.xstride = c.xr ? c.x_box : stride_for(c.xk_max / KS);
  int pmax = 1;
  bool split = S > 1;
  for (int s = 0; s < S && c.tpc == 0; ++s) {
    const int cnt = ks_base + (s < ks_rem ? 1 : 0);
    const long long L = (long long)c.tiles * cnt;
    std::vector<int> pieces(c.tiles, 1);
    for (long long w = 1; w < P; ++w) {
      const long long bnd = w * L / P;
      if (bnd % cnt != 0) { pieces[bnd / cnt] += 1; split = true; }
    }
    for (int r = 0; r < c.tiles; ++r) pmax = pieces[r] > pmax ? pieces[r] : pmax;
  }
  c.pmax = pmax;
  c.split = split;
  // device-side piece arithmetic is 32-bit: (units + 1) * P must fit
  if (((long long)c.tiles * (ks_base + 1) + 1) * P >= (1LL << 31)) return cudaErrorInvalidConfiguration;
  if ((long long)S * pmax > MAX_PIECES) return cudaErrorInvalidConfiguration;
  {
    const long long x_smem = c.xr ? 0 : (long long)c.ncols * c.xstride;
    const long long left = (long long)optin - 1024 - x_smem - misc_bytes(c.M);
    int nst = int(left / (stage_bytes + c.xbytes));
    c.nstage = nst < NSTAGE_MAX ? nst : NSTAGE_MAX;
  }
  if (c.nstage < nstage_min) return cudaErrorInvalidConfiguration;
  c.smem = 1024 + size_t(c.nstage) * (stage_bytes + c.xbytes) +
           (c.xr ? 0 : size_t(c.ncols) * c.xstride) + misc_bytes(c.M);
  if (c.smem > size_t(optin)) return cudaErrorInvalidConfiguration;
  // workspace: status word, per-(tile, row group) counters, partial sums,
  // and for X in the ring the X planes plus per-token exponent and lo flag
  c.ws_counters_off = 256;
  // argmax epilogue state (per-token keys, finished-CTA counter) after the counters
  c.ws_epi_off = c.ws_counters_off + ((size_t(c.tiles) * NCW * 4 + 255) / 256) * 256;
  c.ws_partials_off = c.ws_epi_off + 256;
  const size_t partials_end = split ? c.ws_partials_off + size_t(c.tiles) * S * pmax * c.M * TROWS * 4
                                    : ((c.xr || c.epi == EPI_ARGMAX) ? c.ws_partials_off : 256);
  if (c.xr) {
    c.ws_x_off = ((partials_end + 255) / 256) * 256;
    c.ws_xmeta_off = c.ws_x_off + ((size_t(c.ncols) * c.x_pitch + 255) / 256) * 256;
    // exponents [16], W4A4 gs_x, lo flags [xchunks][16]
    c.xchunks = c.act4 ? 1 : std::min(16, (c.K / KS + XP_STEPS - 1) / XP_STEPS);
    c.ws_bytes = c.ws_xmeta_off + 128 + size_t(c.xchunks) * 64;
  } else {
    c.ws_x_off = c.ws_xmeta_off = 0;
    c.ws_bytes = partials_end;
  }
  e = set_smem_attrs<EPI_NONE>(optin);
  if (e == cudaSuccess) e = set_smem_attrs<EPI_SWIGLU>(optin);
  if (e == cudaSuccess) e = set_smem_attrs<EPI_ARGMAX>(optin);
  return e;
}

// FP8 weight tier: the E4M3 codes [N][K] as boxes of 128 bytes x 256 rows
// with the 128-byte swizzle (two per 256-code K-step).
bool encode_fp8_codes_map(int N, int K, const uint8_t* wp, void* map_w) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dim[2] = {cuuint64_t(K), cuuint64_t(N)};
  const cuuint64_t str[1] = {cuuint64_t(K)};
  const cuuint32_t box[2] = {128, cuuint32_t(mm::TROWS)};
  const cuuint32_t one[2] = {1, 1};
  return fn(static_cast<CUtensorMap*>(map_w), CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(wp), dim, str,
            box, one, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_mma(const MmaConfig& c, const void* map_w, const void* map_s, const void* map_x,
                       const float* gs, const float* row_scale, const uint16_t* x, uint16_t* y,
                       void* workspace, long long timeout_cycles, bool stall, bool pdl, cudaStream_t st) {
  using namespace mm;
  Params p;
  p.M = c.M; p.N = c.N; p.K = c.K; p.tiles = c.tiles; p.S = c.S; p.P = c.P;
  p.ks_base = c.ks_base; p.ks_rem = c.ks_rem; p.ncols = c.ncols; p.xk_max = c.xk_max;
  p.xstride = c.xstride; p.pmax = c.pmax; p.nstage = c.nstage; p.tpc = c.tpc; p.act4 = c.act4;
  p.xbytes = c.xbytes; p.xbox_words = c.x_box / 4; p.xbox_bytes = c.ncols * c.x_box;
  p.gs = gs; p.x = x; p.y = y; p.row_scale = row_scale;
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  p.status = reinterpret_cast<uint32_t*>(wsb);
  p.counters = reinterpret_cast<uint32_t*>(wsb + c.ws_counters_off);
  p.partials = c.split ? reinterpret_cast<float*>(wsb + c.ws_partials_off) : nullptr;
  p.xemax = c.xr ? reinterpret_cast<const int*>(wsb + c.ws_xmeta_off) : nullptr;
  p.xlo = c.xr ? reinterpret_cast<const uint32_t*>(wsb + c.ws_xmeta_off + 128) : nullptr;
  p.xgs = c.xr ? reinterpret_cast<const float*>(wsb + c.ws_xmeta_off + 64) : nullptr;
  p.xchunks = c.xr ? c.xchunks : 0;
  p.keys = reinterpret_cast<unsigned long long*>(wsb + c.ws_epi_off);
  p.done = reinterpret_cast<uint32_t*>(wsb + c.ws_epi_off + 128);
  p.timeout = timeout_cycles;
  p.stall = stall ? 1 : 0;
  const CUtensorMap& mw = *static_cast<const CUtensorMap*>(map_w);
  const CUtensorMap& ms = *static_cast<const CUtensorMap*>(map_s);
  const CUtensorMap& mx = c.xr ? *static_cast<const CUtensorMap*>(map_x) : mw;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  if (c.xr) {
    cudaLaunchConfig_t pc = {};
    pc.gridDim = dim3(c.M, c.xchunks);
    pc.blockDim = dim3(256);
    pc.stream = st;
    pc.attrs = attr;
    pc.numAttrs = pdl ? 1 : 0;
    int* emax = reinterpret_cast<int*>(wsb + c.ws_xmeta_off);
    uint32_t* lo = reinterpret_cast<uint32_t*>(wsb + c.ws_xmeta_off + 128);
    cudaError_t e =
        c.act4 ? cudaLaunchKernelEx(&pc, k_xprep_act4, x, c.M, c.K, wsb + c.ws_x_off, c.x_pitch, emax, lo,
                                    reinterpret_cast<float*>(wsb + c.ws_xmeta_off + 64))
               : cudaLaunchKernelEx(&pc, k_xprep, x, c.M, c.K, wsb + c.ws_x_off, c.x_pitch, emax, lo,
                                    (c.K / KS + c.xchunks - 1) / c.xchunks);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(c.grid);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = c.smem;
  cfg.stream = st;
  cfg.attrs = attr;
  // after k_xprep the dependency is always programmatic: k_mma waits for it in-kernel
  cfg.numAttrs = (pdl || c.xr) ? 1 : 0;
  if (c.epi == EPI_SWIGLU) return launch_main<EPI_SWIGLU>(c, &cfg, mw, ms, mx, p);
  if (c.epi == EPI_ARGMAX) return launch_main<EPI_ARGMAX>(c, &cfg, mw, ms, mx, p);
  return launch_main<EPI_NONE>(c, &cfg, mw, ms, mx, p);
}

}  // namespace nvfp4
