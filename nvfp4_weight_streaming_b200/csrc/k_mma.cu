// k_mma.cu -- TMA-fed warp-MMA variant of the NVFP4 linear (sm_100a).
//
// Y[M][N] = X[M][K] W^T, swap-AB on mma.sync.m16n8k16 (f16 x f16 -> f32):
// the 16-row MMA dimension is weight rows, the 8-column dimension is tokens
// (1 + drafted tokens checked in one pass; page "InventDB Sparkle", section
// "How it answers quickly"). The weight read is the whole cost (page
// "Qwen3.8-27B-NVFP4-RTX5090 API & Inference Endpoint", section "Why lm_head
// is NVFP4, and why MTP is gone"), so the kernel is a weight stream:
//
//   warp 0       TMA producer: 256-row x 256-element tiles of packed codes
//                (32 KB, 128-byte swizzle) and their E4M3 scales (4 KB) into a
//                4-stage shared-memory ring (mbarrier full/empty pairs): about
//                144 KB in flight per SM, what the ~2.6 us loaded DRAM latency
//                of B200 needs at full bandwidth.
//   warps 1..16  consumers: warp w owns rows 16(w-1)..16(w-1)+15 of every tile.
//                Lane (g, t) reads rows g and g+8, 64 consecutive K elements
//                each (two swizzled 16-byte chunks and 4 scale bytes per row),
//                converts codes and scales with the hardware e2m1x2 / e4m3x2 ->
//                f16x2 conversions and multiplies them (exact: at most 6
//                significant bits, magnitude in [2^-10, 2688]) straight into
//                the A fragment registers, then issues the MMAs. MMA i of a
//                step maps its K slots to physical K as (2t, 2t+1) <-> 64t + 4i
//                + {0, 1} and (2t+8, 2t+9) <-> 64t + 4i + {2, 3}, so every
//                fragment is four consecutive elements of one lane.
//
// B is X, kept for the CTA's K-slice in shared memory as f16, scaled per token
// by a power of two (largest magnitude at 2^14) in a hi plane (exact within
// 2^28 of that maximum) and a lo plane scaled by 2^29 (the next 29 binades);
// elements further below are dropped. B fragments are 8-byte shared loads,
// XOR-swizzled so a half warp touches 16 distinct bank pairs. Every product is
// exact; only the fp32 accumulation rounds. For M > 8 the lo tiles are issued
// only when some element of the slice needs them.
//
// Why not tcgen05 here: on B200 a tcgen05.mma kind::f16 with M = 128 costs ~85
// cycles whatever N <= 128 is, i.e. at most 24 weight elements per clock per
// SM, while this warp MMA sustains ~1000 MAC per clock per SM, i.e. 128
// weight elements per clock at N = 8. For this skinny contraction the warp
// MMA is the faster tensor path (the tcgen05 kernel is kept as variant TC).
//
// Work split: K is cut into S slices (an X slice fits in shared memory next
// to the ring); the CTAs of a slice share its (256-row tile, 256-k step) units
// evenly (stream-K). Tiles a CTA covers entirely are stored directly; a tile
// split between CTAs writes fp32 partials, and after its last unit each CTA
// settles its split tiles: the last piece to arrive (atomic counter per tile)
// sums all pieces in k order, so results repeat bit for bit, and resets the
// counter. Every mbarrier wait is bounded; on expiry the CTA records the
// timeout in the workspace status word, stops, drains its in-flight TMA loads
// and returns.
#include "kernels.h"
#include "nvfp4_device.cuh"

#include <cuda.h>
#include <climits>
#include <vector>

namespace nvfp4 {
namespace mm {

constexpr int KS = 256;                    // K elements per step
constexpr int TROWS = 256;                 // weight rows per tile
constexpr int NCW = 16;                    // consumer warps (16 rows each)
constexpr int WARP_SETTLE = NCW + 1;       // warp 0 producer, 1..16 consumers, 17 settler
constexpr int NUM_THREADS = (NCW + 2) * 32;
constexpr int QN = 8;                      // split-tile queue slots (consumers -> settler)
constexpr int MAX_PIECES = 62;             // pieces of one tile the settler can list
constexpr int NSTAGE = 4;
constexpr int W_BYTES = TROWS * KS / 2;    // 32768
constexpr int S_BYTES = TROWS * KS / 16;   // 4096
constexpr int RING_BYTES = NSTAGE * (W_BYTES + S_BYTES);
constexpr int MISC_BYTES = 640;
constexpr int BAR_XISSUED = 2;             // producer waits until X loads are issued
constexpr int MAXC = 6;                    // X chunks (8 elements) per consumer thread
constexpr int LO_SHIFT = 29;
constexpr int BAR_CONSUMERS = 1;           // named barrier of the consumer warps

constexpr uint32_t ST_TIMEOUT_PRODUCER = 1u, ST_TIMEOUT_CONSUMER = 2u, ST_TIMEOUT_SETTLER = 4u,
                   ST_TIMEOUT_DRAIN = 16u;

struct Params {
  int M, N, K, tiles, S, P, ks_base, ks_rem, ncols, xk_max, xstride, pmax;
  const float* gs;
  const uint16_t* x;
  uint16_t* y;
  uint32_t* status;
  uint32_t* counters;
  float* partials;
  long long timeout;
  int stall;
};

// Byte offset of X element k (local to the slice) inside a column: 8-byte
// granules q = k/4 are XOR-swizzled by bits 4..5 of q.
__device__ __forceinline__ uint32_t x_off(int k) {
  const int q = k >> 2;
  return uint32_t(((q ^ ((q >> 4) & 3)) << 3) | ((k & 3) << 1));
}

__device__ __forceinline__ void mma16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ bool wait_bar(uint32_t b, uint32_t parity, volatile int* abort_flag,
                                         const Params& p, uint32_t who) {
  if (mbar_test(b, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_test(b, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > p.timeout) {
      *abort_flag = 1;
      atomicOr(p.status, who);
      return false;
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

// One step of one lane: decode rows r and r+8 of the stage (64 elements each)
// and issue the MMAs for NTILE 8-column token tiles. MMA i of the step adds
// into accumulator set i % (4 / NTILE): four independent chains per warp,
// instead of sixteen MMAs serialised on one accumulator.
template <int NTILE>
__device__ __forceinline__ void compute_step(const uint8_t* sw, const uint8_t* ss, int r, float (*acc)[4],
                                             const uint8_t* xcol, uint32_t xstride, int kloc, int t) {
  const int r1 = r + 8;
  // chunks 2t, 2t+1 of each row; the TMA 128-byte swizzle puts chunk c of row
  // r at position c ^ (r & 7)
  const uint4 c00 = *reinterpret_cast<const uint4*>(sw + r * 128 + (((2 * t) ^ (r & 7)) << 4));
  const uint4 c01 = *reinterpret_cast<const uint4*>(sw + r * 128 + (((2 * t + 1) ^ (r & 7)) << 4));
  const uint4 c10 = *reinterpret_cast<const uint4*>(sw + r1 * 128 + (((2 * t) ^ (r1 & 7)) << 4));
  const uint4 c11 = *reinterpret_cast<const uint4*>(sw + r1 * 128 + (((2 * t + 1) ^ (r1 & 7)) << 4));
  const uint32_t s0 = *reinterpret_cast<const uint32_t*>(ss + r * 16 + 4 * t);
  const uint32_t s1 = *reinterpret_cast<const uint32_t*>(ss + r1 * 16 + 4 * t);
  const uint32_t w0[8] = {c00.x, c00.y, c00.z, c00.w, c01.x, c01.y, c01.z, c01.w};
  const uint32_t w1[8] = {c10.x, c10.y, c10.z, c10.w, c11.x, c11.y, c11.z, c11.w};
  const uint32_t s0lo = e4m3x2_to_f16x2(s0), s0hi = e4m3x2_to_f16x2(s0 >> 16);
  const uint32_t s1lo = e4m3x2_to_f16x2(s1), s1hi = e4m3x2_to_f16x2(s1 >> 16);
  const uint32_t sc0[4] = {bcast_lo(s0lo), bcast_hi(s0lo), bcast_lo(s0hi), bcast_hi(s0hi)};
  const uint32_t sc1[4] = {bcast_lo(s1lo), bcast_hi(s1lo), bcast_lo(s1hi), bcast_hi(s1hi)};
  const int qbase = (kloc >> 2) + 16 * t;
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
      const uint32_t off = uint32_t(((qbase + i) ^ t) << 3);
      constexpr int NSET = 4 / NTILE;
#pragma unroll
      for (int nt = 0; nt < NTILE; ++nt) {
        const uint2 bb = *reinterpret_cast<const uint2*>(xcol + nt * 8 * xstride + off);
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
template <int MC, int NTILE>
__device__ __forceinline__ void consume(const Params& p, uint8_t* sW, uint8_t* sS, const uint8_t* sX,
                                        const int* emax, uint32_t b_full, uint32_t b_empty,
                                        uint32_t b_qfull, uint32_t b_qempty,
                                        volatile int* abort_flag, int s, int cnt, long long a,
                                        long long b, long long L, int cw, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const int r = 16 * cw + g;                           // row of the tile (and r + 8)
  int tok[4];
  float fh[4], fl[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) { tok[e] = -1; fh[e] = fl[e] = 0.0f; }
  if (MC == 1) {
    if (t < 2) { tok[0] = 2 * t; tok[1] = 2 * t + 1; }
  } else {
    tok[0] = 2 * t; tok[1] = 2 * t + 1;
    if (MC == 3) { tok[2] = 8 + 2 * t; tok[3] = 9 + 2 * t; }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int m = tok[e];
    if (m >= 0 && m < p.M && emax[m] != INT_MIN) {
      const int sh = 14 - emax[m];
      fh[e] = ldexpf(1.0f, -sh);
      fl[e] = ldexpf(1.0f, -(sh + LO_SHIFT));
    }
  }
  const float gs = *p.gs;
  const uint8_t* xcol = sX + size_t(g) * p.xstride;
  float acc[4][4];
#pragma unroll
  for (int q = 0; q < 4; ++q) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0.0f;
  long long i = 0;                                     // stage counter
  long long seg_start = a;
  int nsplit = 0;                                      // split segments handed to the settler
  for (long long idx = a; idx < b; ++idx, ++i) {
    const int st = int(i % NSTAGE);
    const bool ok = wait_bar(b_full + 8 * st, uint32_t(i / NSTAGE) & 1u, abort_flag, p, ST_TIMEOUT_CONSUMER);
    if (!__all_sync(0xffffffffu, ok)) break;
    const int tile = int(idx / cnt), j = int(idx % cnt);
    compute_step<NTILE>(sW + st * W_BYTES, sS + st * S_BYTES, r, acc, xcol, p.xstride, j * KS, t);
    __syncwarp();
    if (lane == 0) mbar_arrive(b_empty + 8 * st);
    const bool seg_last = (idx + 1 == b) || (j + 1 == cnt);
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
    // per-token values of this lane: v[e][0] row r, v[e][1] row r+8
    float v[4][2];
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e][0] = v[e][1] = 0.0f;
    if (MC == 1) {
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
        v[e][0] = at[0][e] * fh[e] + at[1][e] * fl[e];
        v[e][1] = at[0][2 + e] * fh[e] + at[1][2 + e] * fl[e];
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
    const long long this_start = seg_start;
    seg_start = idx + 1;
    const bool whole = (p.S == 1) && (this_start == (long long)tile * cnt) && (j + 1 == cnt);
    const int row0 = tile * TROWS + r, row1 = row0 + 8;
    if (whole) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int m = tok[e];
        if (m >= 0 && m < p.M) {
          if (row0 < p.N) p.y[size_t(m) * p.N + row0] = float_to_bf16_bits(gs * v[e][0]);
          if (row1 < p.N) p.y[size_t(m) * p.N + row1] = float_to_bf16_bits(gs * v[e][1]);
        }
      }
      continue;
    }
    // piece of a split tile: write the partial, then queue it for the settler
    const int qs = nsplit % QN;
    if (nsplit >= QN) {
      const bool okq = wait_bar(b_qempty + 8 * qs, uint32_t((nsplit / QN) - 1) & 1u, abort_flag, p,
                                ST_TIMEOUT_CONSUMER);
      if (!__all_sync(0xffffffffu, okq)) break;
    }
    const int ord = int(boundaries_in((long long)tile * cnt, this_start, L, p.P));
    const long long slot = ((long long)tile * p.S + s) * p.pmax + ord;
    float* part = p.partials + slot * p.M * TROWS;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int m = tok[e];
      if (m >= 0 && m < p.M) {
        part[m * TROWS + r] = v[e][0];
        part[m * TROWS + r + 8] = v[e][1];
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(b_qfull + 8 * qs);
    ++nsplit;
  }
}

// Settler warp: walks the same segments as the consumers; for each split
// tile, once all consumer warps have written its piece, it bumps the tile's
// counter; if this CTA brought the last piece it adds all pieces in k order
// (slice, then ordinal) and stores Y, and resets the counter.
__device__ __forceinline__ void settle(const Params& p, uint32_t b_qfull, uint32_t b_qempty,
                                       volatile int* abort_flag, int cnt, long long a, long long b,
                                       int lane, uint32_t* pieces) {
  const float gs = *p.gs;
  int nsplit = 0;
  long long seg_start = a;
  for (long long idx = a; idx < b; ++idx) {
    const int tile = int(idx / cnt), j = int(idx % cnt);
    if (!((idx + 1 == b) || (j + 1 == cnt))) continue;
    const long long this_start = seg_start;
    seg_start = idx + 1;
    const bool whole = (p.S == 1) && (this_start == (long long)tile * cnt) && (j + 1 == cnt);
    if (whole) continue;
    const int qs = nsplit % QN;
    const bool ok = wait_bar(b_qfull + 8 * qs, uint32_t(nsplit / QN) & 1u, abort_flag, p, ST_TIMEOUT_SETTLER);
    if (!__all_sync(0xffffffffu, ok)) return;
    unsigned last = 0;
    if (lane == 0) {
      // the tile's pieces in k order (slice, then ordinal) as partial slots
      int npieces = 0;
      for (int s2 = 0; s2 < p.S; ++s2) {
        const int cnt2 = p.ks_base + (s2 < p.ks_rem ? 1 : 0);
        const long long L2 = (long long)p.tiles * cnt2;
        const int np = 1 + int(boundaries_in((long long)tile * cnt2, (long long)(tile + 1) * cnt2 - 1, L2, p.P));
        for (int o = 0; o < np && npieces < MAX_PIECES; ++o)
          pieces[npieces++] = uint32_t(((long long)tile * p.S + s2) * p.pmax + o);
      }
      pieces[MAX_PIECES] = uint32_t(npieces);
      // the mbarrier wait orders the consumers' partial stores before this
      // gpu-scope fence (fences are cumulative); then the counter
      __threadfence();
      const unsigned old = atomicAdd(&p.counters[tile], 1u);
      __threadfence();
      last = (old == unsigned(npieces - 1)) ? 1u : 0u;
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    __syncwarp();
    if (last) {
      const int npieces = int(pieces[MAX_PIECES]);
      const int MT = p.M * TROWS;
      for (int u = lane; u < MT; u += 32) {
        float sum = 0.0f;
        for (int o = 0; o < npieces; ++o) sum += __ldcg(p.partials + size_t(pieces[o]) * MT + u);
        const int m = u / TROWS, row = tile * TROWS + (u - m * TROWS);
        if (row < p.N) p.y[size_t(m) * p.N + row] = float_to_bf16_bits(gs * sum);
      }
      __syncwarp();
      if (lane == 0) atomicExch(&p.counters[tile], 0u);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(b_qempty + 8 * qs);
    ++nsplit;
  }
}

template <int MC>
__global__ void __launch_bounds__(NUM_THREADS, 1)
k_mma(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_s, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sW = smem;                                     // NSTAGE x 32 KB (1024-aligned)
  uint8_t* sS = smem + NSTAGE * W_BYTES;                  // NSTAGE x 4 KB
  uint8_t* sX = sS + NSTAGE * S_BYTES;
  uint8_t* misc = sX + size_t(p.ncols) * p.xstride;
  uint64_t* bars = reinterpret_cast<uint64_t*>(misc);     // full[4] empty[4] qfull[8] qempty[8]
  int* emax = reinterpret_cast<int*>(misc + 256);          // [16]
  uint32_t* flags = reinterpret_cast<uint32_t*>(misc + 320);  // [0] need_lo [1] abort
  volatile int* abort_flag = reinterpret_cast<volatile int*>(flags + 1);
  const uint32_t b_full = smem_u32(bars), b_empty = b_full + 8 * NSTAGE;
  const uint32_t b_qfull = b_empty + 8 * NSTAGE, b_qempty = b_qfull + 8 * QN;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = blockIdx.x / p.P, c = blockIdx.x % p.P;
  const int cnt = p.ks_base + (s < p.ks_rem ? 1 : 0);
  const int ks0 = s * p.ks_base + min(s, p.ks_rem);
  const int klen = cnt * KS, k0e = ks0 * KS;
  const int mcols = MC == 1 ? 4 : (MC == 2 ? 8 : 16);    // columns per plane
  const long long L = (long long)p.tiles * cnt;
  const long long a = (long long)c * L / p.P, b = (long long)(c + 1) * L / p.P;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSTAGE; ++i) { mbar_init(b_full + 8 * i, 1); mbar_init(b_empty + 8 * i, NCW); }
    for (int i = 0; i < QN; ++i) { mbar_init(b_qfull + 8 * i, NCW); mbar_init(b_qempty + 8 * i, 1); }
    for (int m = 0; m < 16; ++m) emax[m] = INT_MIN;
    flags[0] = 0u; flags[1] = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();

  if (warp == 0) {
    // -------------------------------------------------------------- producer
    // X is read first: wait until every consumer has issued its X loads, so
    // they are not queued behind the weight stream
    named_bar(BAR_XISSUED, (NCW + 1) * 32);
    if (lane == 0) {
      long long n_issued = 0;
      if (!p.stall) {
        for (long long idx = a; idx < b; ++idx, ++n_issued) {
          const int tile = int(idx / cnt), j = int(idx % cnt);
          const int st = int(n_issued % NSTAGE);
          const uint32_t ph = uint32_t(n_issued / NSTAGE) & 1u;
          if (!wait_bar(b_empty + 8 * st, ph ^ 1u, abort_flag, p, ST_TIMEOUT_PRODUCER)) break;
          mbar_expect_tx(b_full + 8 * st, W_BYTES + S_BYTES);
          tma_load_2d(smem_u32(sW + st * W_BYTES), &tm_w, (ks0 + j) * (KS / 2), tile * TROWS, b_full + 8 * st);
          tma_load_2d(smem_u32(sS + st * S_BYTES), &tm_s, (ks0 + j) * (KS / 16), tile * TROWS, b_full + 8 * st);
        }
      }
      if (*abort_flag) {
        const long long first = n_issued > NSTAGE ? n_issued - NSTAGE : 0;
        for (long long i = first; i < n_issued; ++i)
          drain_bar(b_full + 8 * int(i % NSTAGE), uint32_t(i / NSTAGE) & 1u, p);
      }
    }
    __syncwarp();
  } else if (warp == WARP_SETTLE) {
    // ---------------------------------------------------------------- settler
    settle(p, b_qfull, b_qempty, abort_flag, cnt, a, b, lane, reinterpret_cast<uint32_t*>(misc + 384));
  } else {
    // ------------------------------------------------ consumers: stage X first
    const int ctid = threadIdx.x - 32;                    // 0 .. NCW*32-1
    constexpr int NCT = NCW * 32;
    const int chunks = klen / 8;
    const int nreal = p.M * chunks;
    uint4 xv[MAXC];
#pragma unroll
    for (int cc = 0; cc < MAXC; ++cc) {
      const int u = ctid + cc * NCT;
      if (u < nreal) {
        const int m = u / chunks, kc = u - m * chunks;
        xv[cc] = *reinterpret_cast<const uint4*>(p.x + size_t(m) * p.K + k0e + 8 * kc);
      }
    }
    asm volatile("bar.arrive %0, %1;" ::"r"(BAR_XISSUED), "r"((NCW + 1) * 32) : "memory");
#pragma unroll
    for (int cc = 0; cc < MAXC; ++cc) {
      const int u = ctid + cc * NCT;
      if (u < nreal) {
        const int m = u / chunks;
        const uint32_t w[4] = {xv[cc].x, xv[cc].y, xv[cc].z, xv[cc].w};
        int mx = INT_MIN;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint32_t bb = (w[q >> 1] >> (16 * (q & 1))) & 0xFFFFu;
          if (bb & 0x7FFFu) { uint32_t sg; mx = max(mx, bf16_exp(bb, sg)); }
        }
        if (mx != INT_MIN) atomicMax(&emax[m], mx);
      }
    }
    named_bar(BAR_CONSUMERS, NCT);
    bool lo_used = false;
#pragma unroll
    for (int cc = 0; cc < MAXC; ++cc) {
      const int u = ctid + cc * NCT;
      if (u < nreal) {
        const int m = u / chunks, kc = u - m * chunks;
        const int sh = (emax[m] == INT_MIN) ? 0 : 14 - emax[m];
        const uint32_t w[4] = {xv[cc].x, xv[cc].y, xv[cc].z, xv[cc].w};
        uint32_t hi[4] = {0u, 0u, 0u, 0u}, lo[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint32_t bb = (w[q >> 1] >> (16 * (q & 1))) & 0xFFFFu;
          if (bb & 0x7FFFu) {
            uint32_t sg;
            const int th = bf16_exp(bb, sg) + sh;
            if (th >= -14) hi[q >> 1] |= make_f16(bb >> 15, th, sg) << (16 * (q & 1));
            else lo[q >> 1] |= make_f16(bb >> 15, th + LO_SHIFT, sg) << (16 * (q & 1));
          }
        }
        lo_used |= (lo[0] | lo[1] | lo[2] | lo[3]) != 0u;
        const uint32_t o0 = x_off(8 * kc), o1 = x_off(8 * kc + 4);
        uint8_t* ch = sX + size_t(m) * p.xstride;
        uint8_t* cl = sX + size_t(mcols + m) * p.xstride;
        *reinterpret_cast<uint2*>(ch + o0) = make_uint2(hi[0], hi[1]);
        *reinterpret_cast<uint2*>(ch + o1) = make_uint2(hi[2], hi[3]);
        *reinterpret_cast<uint2*>(cl + o0) = make_uint2(lo[0], lo[1]);
        *reinterpret_cast<uint2*>(cl + o1) = make_uint2(lo[2], lo[3]);
      }
    }
    {
      const int npad = mcols - p.M;                       // token columns >= M are zero
      for (int u = ctid; u < 2 * npad * chunks; u += NCT) {
        const int pr = u / chunks, kc = u - pr * chunks;
        const int col = (pr < npad) ? (p.M + pr) : (mcols + p.M + pr - npad);
        *reinterpret_cast<uint4*>(sX + size_t(col) * p.xstride + 16 * kc) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    if (lo_used) atomicOr(&flags[0], 1u);
    named_bar(BAR_CONSUMERS, NCT);
    const bool need_lo = flags[0] != 0u;

    const int cw = warp - 1;
    if (MC == 1) {
      consume<1, 1>(p, sW, sS, sX, emax, b_full, b_empty, b_qfull, b_qempty, abort_flag, s, cnt, a, b, L, cw, lane);
    } else if (MC == 2) {
      consume<2, 2>(p, sW, sS, sX, emax, b_full, b_empty, b_qfull, b_qempty, abort_flag, s, cnt, a, b, L, cw, lane);
    } else {
      if (need_lo)
        consume<3, 4>(p, sW, sS, sX, emax, b_full, b_empty, b_qfull, b_qempty, abort_flag, s, cnt, a, b, L, cw, lane);
      else
        consume<3, 2>(p, sW, sS, sX, emax, b_full, b_empty, b_qfull, b_qempty, abort_flag, s, cnt, a, b, L, cw, lane);
    }
  }
  __syncthreads();
}

}  // namespace mm

cudaError_t mma_configure(MmaConfig& c, int num_sms) {
  using namespace mm;
  if (c.M < 1 || c.M > 16 || c.K % KS != 0 || c.K <= 0 || c.N <= 0) return cudaErrorInvalidValue;
  int dev = 0, optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  const int mcols = c.M <= 4 ? 4 : (c.M <= 8 ? 8 : 16);
  c.ncols = 2 * mcols;
  c.tiles = (c.N + TROWS - 1) / TROWS;
  const int ksteps = c.K / KS;
  const long long x_budget = (long long)optin - 1024 - RING_BYTES - MISC_BYTES;
  // largest slice (in steps) whose two X planes fit next to the ring and whose
  // chunks the consumers hold in registers (M * steps * KS / 8 <= MAXC * consumer threads)
  auto fits = [&](int ks) {
    return (long long)c.ncols * (ks * KS * 2 + 32) <= x_budget &&
           (long long)c.M * ks * KS / 8 <= (long long)MAXC * NCW * 32;
  };
  if (!fits(1)) return cudaErrorInvalidConfiguration;
  int max_ks = 1;
  while (max_ks < ksteps && fits(max_ks + 1)) ++max_ks;
  const int S = (ksteps + max_ks - 1) / max_ks;
  int P = num_sms / S;
  if (P < 1) return cudaErrorInvalidConfiguration;
  const int ks_base = ksteps / S, ks_rem = ksteps % S;
  const long long min_units = (long long)c.tiles * ks_base;
  if (P > min_units) P = int(min_units);
  c.S = S; c.P = P; c.ks_base = ks_base; c.ks_rem = ks_rem;
  c.grid = S * P;
  c.xk_max = (ks_base + (ks_rem ? 1 : 0)) * KS;
  c.xstride = c.xk_max * 2 + 32;
  int pmax = 1;
  bool split = S > 1;
  for (int s = 0; s < S; ++s) {
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
  if ((long long)S * pmax > MAX_PIECES) return cudaErrorInvalidConfiguration;
  c.smem = 1024 + size_t(RING_BYTES) + size_t(c.ncols) * c.xstride + MISC_BYTES;
  c.ws_counters_off = 256;
  c.ws_partials_off = c.ws_counters_off + ((size_t(c.tiles) * 4 + 255) / 256) * 256;
  c.ws_bytes = split ? c.ws_partials_off + size_t(c.tiles) * S * pmax * c.M * TROWS * 4 : 256;
  if (c.smem > size_t(optin)) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(k_mma<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_mma<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_mma<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  return e;
}

cudaError_t launch_mma(const MmaConfig& c, const void* map_w, const void* map_s, const float* gs,
                       const uint16_t* x, uint16_t* y, void* workspace, long long timeout_cycles,
                       bool stall, cudaStream_t st) {
  using namespace mm;
  Params p;
  p.M = c.M; p.N = c.N; p.K = c.K; p.tiles = c.tiles; p.S = c.S; p.P = c.P;
  p.ks_base = c.ks_base; p.ks_rem = c.ks_rem; p.ncols = c.ncols; p.xk_max = c.xk_max;
  p.xstride = c.xstride; p.pmax = c.pmax;
  p.gs = gs; p.x = x; p.y = y;
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  p.status = reinterpret_cast<uint32_t*>(wsb);
  p.counters = reinterpret_cast<uint32_t*>(wsb + c.ws_counters_off);
  p.partials = c.split ? reinterpret_cast<float*>(wsb + c.ws_partials_off) : nullptr;
  p.timeout = timeout_cycles;
  p.stall = stall ? 1 : 0;
  const CUtensorMap& mw = *static_cast<const CUtensorMap*>(map_w);
  const CUtensorMap& ms = *static_cast<const CUtensorMap*>(map_s);
  if (c.M <= 4) k_mma<1><<<c.grid, NUM_THREADS, c.smem, st>>>(mw, ms, p);
  else if (c.M <= 8) k_mma<2><<<c.grid, NUM_THREADS, c.smem, st>>>(mw, ms, p);
  else k_mma<3><<<c.grid, NUM_THREADS, c.smem, st>>>(mw, ms, p);
  return cudaGetLastError();
}

}  // namespace nvfp4
