// k_row.cu -- row-block streaming variant of the NVFP4 linear (sm_100a), M <= 2.
//
// Y[M][N] = X[M][K] W^T for one decode token or a token plus one drafted
// token (page "InventDB Sparkle", section "How it answers quickly"), where the
// whole cost is reading W once (page "Qwen3.8-27B-NVFP4-RTX5090 API &
// Inference Endpoint", section "Why lm_head is NVFP4, and why MTP is gone").
//
// Work. W is cut into units of 16 rows (one m16 MMA row group) by a K-slice
// of at most ten 512-element items (the whole of K = 5120; K is split further
// only when N is so small that the units would not keep every SM busy). One
// CTA per SM takes units: the first two statically, the rest from an atomic
// counter, so SMs that stream faster take more units and the grid ends
// nearly together. A unit is computed by one CTA alone, so Y is written
// without any cross-CTA completion; only a K-split unit adds its partial to
// the others of its row group, in slice order.
//
//   warp 0       producer: claims units and streams each into one slot of a
//                shared-memory ring with two 3D TMA loads and an L2
//                evict-first policy: the codes as 128-byte x 16-row x
//                (2 per item) boxes with the 128-byte swizzle, the E4M3 scales
//                as 16-byte x 16-row x (2 per item) boxes. (One TMA load per
//                16-row x 256-element piece would cost a load per 2 KB, and
//                loads that small cap the stream far below HBM bandwidth.)
//                The first nst units (a full ring) are static, so the ring
//                fills while the previous grid is still finishing.
//   warps 1..16  consumers: every warp passes every unit in order; warp w
//                computes the items w, w + 16, ... of the CTA's item sequence
//                (16 x M partial sums each, left in shared memory), and the
//                warp that completes a unit's last item adds the unit's
//                partials in item order. A slot is refilled once all 16
//                warps are past its unit.
//
// Block-diagonal B operand. An MMA m16n8k16 (f16 x f16 -> f32, swap-AB: rows
// = weights) covers four 16-element scale blocks, four elements of each:
// lane quad t owns block t of the step, so its k slots (2t, 2t+1, 2t+8, 2t+9)
// hold elements 4i..4i+3 of that block in MMA i. The eight B columns are
// (block t, stream s) pairs and the B operand is x only where the k slot's
// block equals the column's block, zero elsewhere. After the step's four
// MMAs, column (t, s) of the accumulator is the exact dot product of one
// block of codes with x; it is then multiplied by that block's E4M3 scale in
// fp32. So the decode is one cvt.rn.f16x2.e2m1x2 per code byte -- no per
// element scale multiply -- and the block scale costs one FFMA per block and
// stream. A stream is one token's hi or lo X plane (below); the two of a
// tile are (tokens 0, 1) or (hi, lo) of a single token.
//
// X. X is bf16, the MMA takes f16: once the previous grid has completed, the
// consumer warps of every CTA load X into registers, scale each token row by
// a power of two (largest magnitude at 2^14) and split it into an f16 hi
// plane and a lo plane scaled by 2^29, which together hold every element
// within 2^57 of the row maximum exactly; the planes stay in shared memory in
// the order the consumers read them. Every product is exact; only fp32 sums
// round.
//
// Every mbarrier wait is bounded by clock64; on expiry the CTA records the
// timeout in the workspace status word, stops, drains its in-flight copies
// and returns.
#include "kernels.h"
#include "nvfp4_device.cuh"

#include <cuda.h>
#include <climits>

namespace nvfp4 {
namespace rw {

constexpr int NCW = 16;                          // consumer warps
constexpr int NUM_THREADS = (NCW + 1) * 32;
constexpr int ROWS = 16;                         // weight rows per unit
constexpr int ITEM_K = 512;                      // K elements per item
constexpr int BOX_W = ROWS * 128;                // codes of 16 rows x 256 elements
constexpr int BOX_S = ROWS * 16;                 // scales of 16 rows x 256 elements
constexpr int XPIECE = ITEM_K * 2;               // f16 bytes of one stream per item
constexpr int XPAD = 64;                         // stream pitch: items * XPIECE + XPAD
constexpr int IPU_CAP = 10;                      // items per unit at most (NVFP4)
constexpr int IPU_CAP_FP8 = 5;                   // items per unit at most (FP8: 8 KB per item)
// Weight formats: NVFP4 (E2M1 codes, E4M3 scale per 16 elements) and the
// FP8 comparison tier (E4M3 codes [N][K], one fp32 scale per row).
constexpr int FMT_NVFP4 = 0, FMT_FP8 = 1;
__host__ __device__ constexpr int item_w_bytes(int fmt) { return fmt == FMT_FP8 ? ROWS * ITEM_K : 2 * ROWS * 128; }
__host__ __device__ constexpr int item_s_bytes(int fmt) { return fmt == FMT_FP8 ? 0 : 2 * ROWS * 16; }
constexpr int NST_MAX = 8;                       // ring slots (one unit each)
constexpr int NST_MIN = 2;
constexpr int MAX_M = 2;
constexpr int XCH_MAX = 8;                       // 16-byte X chunks per consumer thread
constexpr int BAR_CONSUMERS = 1;                 // named barrier of the consumer warps

// misc area (bytes): full[8], empty[8] mbarriers, slot metadata int4[8],
// per-slot item counters, flags (abort, lo plane used), per-token exponent
// maximum
constexpr int MISC_FULL = 0, MISC_EMPTY = 64, MISC_META = 128, MISC_CNT = 256,
              MISC_FLAGS = 288, MISC_EMAX = 296, MISC_BYTES = 320;

constexpr uint32_t ST_TIMEOUT_PRODUCER = 1u, ST_TIMEOUT_CONSUMER = 2u, ST_TIMEOUT_DRAIN = 16u;

struct Params {
  int M, N, K;
  int units16, KS, units, IT, ipu, nst, xstride, sp_row;
  const float* gs;
  const float* row_scale;     // FP8: per-row scale [N]
  const uint16_t* x;
  uint16_t* y;
  uint32_t* status;
  uint32_t* claim;            // [0] unit counter, [1] finished CTAs
  uint32_t* gcnt;             // K-split: per row group counters
  float* gpart;               // K-split: partials [units16][KS][M][16]
  long long timeout;
  int stall;
};

__device__ __forceinline__ bool wait_bar(uint32_t b, uint32_t parity, volatile int* abort_flag,
                                         const Params& p, uint32_t who) {
  if (mbar_test(b, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_wait_hint(b, parity, 2000)) return true;
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

// Byte offset, inside one stream of the prepared X, of the 16-byte piece
// (eight consecutive elements) holding element k: item, step q, half h and
// lane quad t, in the order the consumers read them.
__device__ __forceinline__ uint32_t xpiece_off(int k) {
  const int it = k >> 9, kk = k & 511;
  const int b = kk >> 4, q = b & 7, t = b >> 3, h = (kk >> 3) & 1;
  return uint32_t(it * XPIECE + ((q * 2 + h) * 4 + t) * 16);
}

// Adds the partials of a finished unit (its first `nit` items, in order) and
// writes its rows of Y, or, for a K-split unit, its partial and -- if it is
// the last slice of its row group to finish -- the row group's sum over
// slices in slice order.
template <int FMT>
__device__ __forceinline__ void finish_unit(const Params& p, const float* sPu, int u, int nit, int S,
                                            float fh0, float fh1, float gs, int lane) {
  const int rg = u / p.KS, sl = u - rg * p.KS;
  float v = 0.0f;
  const int r = lane & 15, m = lane >> 4;
  const bool mine = m < p.M;
  if (mine) {
    const float* base = sPu + r * p.sp_row;
    float vh = 0.0f, vl = 0.0f;
    for (int s = 0; s < nit; ++s) {
      const float* e = base + size_t(s) * ROWS * p.sp_row;
      vh += e[m];
      if (S > p.M) vl += e[p.M + m];
    }
    // the planes' scales 2^-sh (hi) and 2^-(sh + 29) (lo) undone: exact powers of two
    v = (vh + vl * (1.0f / 536870912.0f)) * (m == 0 ? fh0 : fh1);
  }
  const int n = rg * ROWS + r;
  // the output scale: the global scale, times the row's scale for FP8
  float os = gs;
  if (FMT == FMT_FP8 && mine && n < p.N) os *= __ldg(p.row_scale + n);
  if (p.KS == 1) {
    if (mine && n < p.N) p.y[size_t(m) * p.N + n] = float_to_bf16_bits(os * v);
    return;
  }
  float* gp = p.gpart + (size_t(rg) * p.KS) * p.M * ROWS;
  if (mine) gp[size_t(sl) * p.M * ROWS + m * ROWS + r] = v;
  __threadfence();
  __syncwarp();
  uint32_t last = 0;
  if (lane == 0) last = atomicAdd(p.gcnt + rg, 1u) == uint32_t(p.KS - 1) ? 1u : 0u;
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return;
  __threadfence();
  if (mine) {
    float sum = 0.0f;
    for (int s2 = 0; s2 < p.KS; ++s2) sum += __ldcg(gp + size_t(s2) * p.M * ROWS + m * ROWS + r);
    if (n < p.N) p.y[size_t(m) * p.N + n] = float_to_bf16_bits(os * sum);
  }
  if (lane == 0) p.gcnt[rg] = 0u;
}

// Consumer warp's walk over its items. NVFP4: NT token tiles (2 streams
// each) per A fragment, S <= 2 streams -> 1, S <= 4 -> 2. FP8: one tile
// whose column g is stream g (NT = 1).
template <int NT, int FMT>
__device__ __forceinline__ void consume(const Params& p, const uint8_t* sW, const uint8_t* sS,
                                        const uint8_t* sX, float* sP, const int4* meta,
                                        uint32_t* cnt, uint32_t b_full, uint32_t b_empty,
                                        volatile int* abort_flag, int S, float fh0, float fh1,
                                        float gs, int cw, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const int ipu = p.ipu;
  // this lane supplies B: column g is (block g >> 1, stream 2 tau + (g & 1))
  bool xon[NT];
#pragma unroll
  for (int tau = 0; tau < NT; ++tau) xon[tau] = ((g >> 1) == t) && (2 * tau + (g & 1) < S);
  // Every warp passes every unit in order (and arrives on its slot's empty
  // barrier), so no warp can run a ring phase ahead of a slot; it computes
  // the unit's items s with (j ipu + s) % NCW == cw.
  for (int j = 0;; ++j) {
    const int slot = j % p.nst;
    const bool ok = wait_bar(b_full + 8 * slot, uint32_t(j / p.nst) & 1u, abort_flag, p, ST_TIMEOUT_CONSUMER);
    if (!__all_sync(0xffffffffu, ok)) break;
    const int u = meta[slot].x;
    if (u < 0) break;
    float* sPu = sP + size_t(slot) * ipu * ROWS * p.sp_row;
    const int s0 = ((cw - (j * ipu) % NCW) + NCW) % NCW;
    for (int s_item = s0; s_item < ipu; s_item += NCW) {
      const int it = (u % p.KS) * ipu + s_item;         // item index along K
      float acc[NT][4];
#pragma unroll
      for (int tau = 0; tau < NT; ++tau) acc[tau][0] = acc[tau][1] = acc[tau][2] = acc[tau][3] = 0.0f;
      if (FMT == FMT_FP8 && it < p.IT) {
        // Lane quad t holds elements 16t .. 16t + 15 of each 64-element step:
        // k slots 2t, 2t+1 <- 4i, 4i+1 and 2t+8, 2t+9 <- 4i+2, 4i+3 of them in
        // MMA i. Column g of B is stream g; every lane supplies the x of its
        // quad's elements. The row scale is applied when the unit is done.
        const uint8_t* ubase = sW + size_t(slot) * ipu * item_w_bytes(FMT);
        const bool xo = g < S;
        const uint8_t* xbase = sX + g * p.xstride + it * XPIECE;
        float da[4] = {0.0f, 0.0f, 0.0f, 0.0f}, db[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          // 128-byte piece 4 s_item + q/2 of the unit; 16 bytes 4 (q & 1) + t of each row
          const uint8_t* cb = ubase + (4 * s_item + (q >> 1)) * BOX_W;
          const int sub = 4 * (q & 1) + t;
          const uint4 w0 = *reinterpret_cast<const uint4*>(cb + g * 128 + ((sub ^ g) << 4));
          const uint4 w1 = *reinterpret_cast<const uint4*>(cb + (g + 8) * 128 + ((sub ^ g) << 4));
          const uint32_t r0[4] = {w0.x, w0.y, w0.z, w0.w}, r1[4] = {w1.x, w1.y, w1.z, w1.w};
          uint32_t h0[8], h1[8];                        // f16x2 of elements (2j, 2j+1)
#pragma unroll
          for (int wd = 0; wd < 4; ++wd) {
            h0[2 * wd] = e4m3x2_to_f16x2(r0[wd]);
            h0[2 * wd + 1] = e4m3x2_to_f16x2(r0[wd] >> 16);
            h1[2 * wd] = e4m3x2_to_f16x2(r1[wd]);
            h1[2 * wd + 1] = e4m3x2_to_f16x2(r1[wd] >> 16);
          }
          // x of block 4q + t of the item (16 elements), in the prepared layout
          const int b = 4 * q + t;
          uint4 x0 = make_uint4(0u, 0u, 0u, 0u), x1 = x0;
          if (xo) {
            x0 = *reinterpret_cast<const uint4*>(xbase + (((b & 7) * 2) * 4 + (b >> 3)) * 16);
            x1 = *reinterpret_cast<const uint4*>(xbase + (((b & 7) * 2 + 1) * 4 + (b >> 3)) * 16);
          }
          const uint32_t xr[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (q & 1) mma16816(db, h0[2 * i], h1[2 * i], h0[2 * i + 1], h1[2 * i + 1], xr[2 * i], xr[2 * i + 1]);
            else mma16816(da, h0[2 * i], h1[2 * i], h0[2 * i + 1], h1[2 * i + 1], xr[2 * i], xr[2 * i + 1]);
          }
        }
        // columns 2t, 2t+1 (streams) of rows g and g + 8
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[0][e] = da[e] + db[e];
      }
      if (FMT == FMT_NVFP4 && it < p.IT) {              // past K: zeros, nothing to add
        const int chunk = 2 * s_item + (t >> 1);        // 256-element piece holding blocks 8t..8t+7
        const uint8_t* box = sW + size_t(slot) * ipu * item_w_bytes(FMT) + chunk * BOX_W;
        const uint8_t* srow = sS + size_t(slot) * ipu * item_s_bytes(FMT) + chunk * BOX_S + g * 16 + 8 * (t & 1);
        const uint2 sc0 = *reinterpret_cast<const uint2*>(srow);              // row g, blocks 8t..8t+7
        const uint2 sc1 = *reinterpret_cast<const uint2*>(srow + 8 * 16);     // row g + 8
        const uint8_t* xb[NT];
#pragma unroll
        for (int tau = 0; tau < NT; ++tau)
          xb[tau] = sX + (2 * tau + (g & 1)) * p.xstride + it * XPIECE + t * 16;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          // 16 bytes c of the lane quad's 64 per row (blocks 8t + 2c, 8t + 2c + 1),
          // at their 128-byte-swizzled place: rows g and g + 8 share the XOR g
          const int ch = 4 * (t & 1) + c;
          const uint4 w0 = *reinterpret_cast<const uint4*>(box + g * 128 + ((ch ^ g) << 4));
          const uint4 w1 = *reinterpret_cast<const uint4*>(box + (g + 8) * 128 + ((ch ^ g) << 4));
#pragma unroll
          for (int hq = 0; hq < 2; ++hq) {
            const int q = 2 * c + hq;                     // step: block 8t + q of the item
            uint32_t h0[8], h1[8];                        // f16x2 of bytes 0..7 of the block
            e2m1x8_to_f16x2x4(hq ? w0.z : w0.x, h0);
            e2m1x8_to_f16x2x4(hq ? w0.w : w0.y, h0 + 4);
            e2m1x8_to_f16x2x4(hq ? w1.z : w1.x, h1);
            e2m1x8_to_f16x2x4(hq ? w1.w : w1.y, h1 + 4);
            uint32_t xr[NT][8];
#pragma unroll
            for (int tau = 0; tau < NT; ++tau) {
              uint4 x0 = make_uint4(0u, 0u, 0u, 0u), x1 = x0;
              if (xon[tau]) {
                x0 = *reinterpret_cast<const uint4*>(xb[tau] + (q * 2) * 64);
                x1 = *reinterpret_cast<const uint4*>(xb[tau] + (q * 2 + 1) * 64);
              }
              xr[tau][0] = x0.x; xr[tau][1] = x0.y; xr[tau][2] = x0.z; xr[tau][3] = x0.w;
              xr[tau][4] = x1.x; xr[tau][5] = x1.y; xr[tau][6] = x1.z; xr[tau][7] = x1.w;
            }
            float d[NT][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              // k slots 2t, 2t+1 <- elements 4i, 4i+1 (byte 2i); 2t+8, 2t+9 <- 4i+2, 4i+3
#pragma unroll
              for (int tau = 0; tau < NT; ++tau) {
                if (i == 0) mma16816_z(d[tau], h0[0], h1[0], h0[1], h1[1], xr[tau][0], xr[tau][1]);
                else mma16816(d[tau], h0[2 * i], h1[2 * i], h0[2 * i + 1], h1[2 * i + 1], xr[tau][2 * i],
                              xr[tau][2 * i + 1]);
              }
            }
            // E4M3 scales of block 8t + q for rows g and g + 8, to fp32
            const uint32_t ra = (q < 4) ? sc0.x : sc0.y, rb = (q < 4) ? sc1.x : sc1.y;
            const uint32_t sb = __byte_perm(ra, rb, uint32_t((q & 3) | ((4 + (q & 3)) << 4)));
            const float2 sf = f16x2_to_float2(e4m3x2_to_f16x2(sb));
#pragma unroll
            for (int tau = 0; tau < NT; ++tau) {
              acc[tau][0] = fmaf(sf.x, d[tau][0], acc[tau][0]);
              acc[tau][1] = fmaf(sf.x, d[tau][1], acc[tau][1]);
              acc[tau][2] = fmaf(sf.y, d[tau][2], acc[tau][2]);
              acc[tau][3] = fmaf(sf.y, d[tau][3], acc[tau][3]);
            }
          }
        }
        // sum the four lane quads (blocks 8t..8t+7 each) in a fixed order
#pragma unroll
        for (int tau = 0; tau < NT; ++tau)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[tau][e] += __shfl_xor_sync(0xffffffffu, acc[tau][e], 1);
            acc[tau][e] += __shfl_xor_sync(0xffffffffu, acc[tau][e], 2);
          }
      }
      if (FMT == FMT_NVFP4 && t == 0) {
        float* e0 = sPu + (size_t(s_item) * ROWS + g) * p.sp_row;
        float* e1 = e0 + 8 * p.sp_row;
#pragma unroll
        for (int tau = 0; tau < NT; ++tau)
#pragma unroll
          for (int sg = 0; sg < 2; ++sg) {
            const int st = 2 * tau + sg;
            if (st < S) {
              e0[st] = acc[tau][sg];
              e1[st] = acc[tau][2 + sg];
            }
          }
      }
      if (FMT == FMT_FP8) {
        float* e0 = sPu + (size_t(s_item) * ROWS + g) * p.sp_row;
        float* e1 = e0 + 8 * p.sp_row;
#pragma unroll
        for (int sg = 0; sg < 2; ++sg) {
          const int st = 2 * t + sg;
          if (st < S) {
            e0[st] = acc[0][sg];
            e1[st] = acc[0][2 + sg];
          }
        }
      }
      __syncwarp();
      uint32_t last = 0;
      if (lane == 0) {
        __threadfence_block();
        last = atomicAdd(cnt + slot, 1u) == uint32_t(ipu - 1) ? 1u : 0u;
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        // every item of the unit is in: sum them (the slot is freed only
        // after this warp, like every other, has arrived on its empty barrier)
        __threadfence_block();
        const int nit = min(ipu, p.IT - (u % p.KS) * ipu);
        finish_unit<FMT>(p, sPu, u, nit, S, fh0, fh1, gs, lane);
        __syncwarp();
        if (lane == 0) cnt[slot] = 0u;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(b_empty + 8 * slot);
  }
}

// Consumers, once the previous grid has completed: X -> the hi and lo f16
// planes in shared memory (streams m and M + m, xstride bytes each, zero past
// K), with the per-token exponent maximum in emax[] and whether any lo
// element is nonzero in *lo_flag. Each thread keeps its (at most XCH_MAX)
// 16-byte chunks of X in registers between the two passes.
__device__ __forceinline__ void stage_x(const Params& p, uint8_t* sX, int* emax, uint32_t* lo_flag,
                                        int ctid) {
  constexpr int NCT = NCW * 32;
  const int per_tok = p.K / 8, nreal = p.M * per_tok;
  uint4 xv[XCH_MAX];
#pragma unroll
  for (int i = 0; i < XCH_MAX; ++i) {
    const int c = ctid + i * NCT;
    xv[i] = make_uint4(0u, 0u, 0u, 0u);
    if (c < nreal) xv[i] = *reinterpret_cast<const uint4*>(p.x + size_t(c) * 8);
  }
  // exponent maximum per token: lanes holding the same token reduce in the
  // warp, one shared-memory atomic per token and warp
#pragma unroll
  for (int i = 0; i < XCH_MAX; ++i) {
    const int c = ctid + i * NCT;
    if ((c & ~31) < nreal) {                          // warp-uniform: some lane of this warp has a chunk
      const int m = c < nreal ? c / per_tok : -1;
      const uint32_t mag = c < nreal ? bf16_mag_max8(xv[i]) : 0u;
      const unsigned grp = __match_any_sync(0xffffffffu, m);
      const int gmx = bf16_mag_exp(__reduce_max_sync(grp, mag));
      if (m >= 0 && gmx != INT_MIN && (ctid & 31) == __ffs(grp) - 1) atomicMax(&emax[m], gmx);
    }
  }
  named_bar(BAR_CONSUMERS, NCT);
  bool lo_used = false;
#pragma unroll
  for (int i = 0; i < XCH_MAX; ++i) {
    const int c = ctid + i * NCT;
    if (c < nreal) {
      const int m = c / per_tok, kc = c - m * per_tok;
      const int sh = emax[m] == INT_MIN ? 0 : 14 - emax[m];
      const uint32_t w[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
      uint32_t hi[4], lo[4];
      lo_used |= x_split8(w, sh, hi, lo);
      const uint32_t off = xpiece_off(8 * kc);
      *reinterpret_cast<uint4*>(sX + size_t(m) * p.xstride + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(sX + size_t(p.M + m) * p.xstride + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
  }
  // the half item past K (K % 512 == 256) reads zeros
  const int pad = p.IT * (ITEM_K / 8) - per_tok;         // chunks per stream, 0 or 32
  for (int c = ctid; c < 2 * p.M * pad; c += NCT) {
    const int st = c / pad, kc = per_tok + (c - st * pad);
    *reinterpret_cast<uint4*>(sX + size_t(st) * p.xstride + xpiece_off(8 * kc)) = make_uint4(0u, 0u, 0u, 0u);
  }
  if (lo_used) atomicOr(lo_flag, 1u);
  named_bar(BAR_CONSUMERS, NCT);
}

template <int FMT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
k_row(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_s, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int nst = p.nst, ipu = p.ipu;
  uint8_t* sW = smem;                                      // nst units of codes (1024-aligned)
  uint8_t* sS = sW + size_t(nst) * ipu * item_w_bytes(FMT);  // nst units of scales (NVFP4)
  uint8_t* sX = sS + size_t(nst) * ipu * item_s_bytes(FMT);   // 2M streams x xstride
  float* sP = reinterpret_cast<float*>(sX + size_t(2 * p.M) * p.xstride);
  uint8_t* misc = reinterpret_cast<uint8_t*>(sP) + size_t(nst) * ipu * ROWS * p.sp_row * 4;
  int4* meta = reinterpret_cast<int4*>(misc + MISC_META);
  uint32_t* cnt = reinterpret_cast<uint32_t*>(misc + MISC_CNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + MISC_FLAGS);
  uint32_t* lo_flag = reinterpret_cast<uint32_t*>(misc + MISC_FLAGS + 4);
  int* emax = reinterpret_cast<int*>(misc + MISC_EMAX);
  const uint32_t b_full = smem_u32(misc + MISC_FULL), b_empty = smem_u32(misc + MISC_EMPTY);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Dependent launches may start now: they only stream weights until this
  // grid has completed.
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) {
    for (int i = 0; i < nst; ++i) {
      mbar_init(b_full + 8 * i, 1);
      mbar_init(b_empty + 8 * i, NCW);
      cnt[i] = 0u;
    }
    *abort_flag = 0;
    *lo_flag = 0u;
    for (int m = 0; m < MAX_M; ++m) emax[m] = INT_MIN;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();

  if (warp == 0) {
    // -------------------------------------------------------------- producer
    if (lane == 0 && !p.stall) {
      const uint64_t pol = l2_evict_first_policy();
      const uint32_t unit_bytes = uint32_t(ipu) * (item_w_bytes(FMT) + item_s_bytes(FMT));
      // the first nst units fill the ring without the counter, which belongs
      // to the previous grid until it has completed
      const int nstatic = nst;
      int j = 0, next_dyn = -1;
      while (!*abort_flag) {
        int u;
        if (j < nstatic) {
          u = int(blockIdx.x) + j * int(gridDim.x);
        } else {
          if (next_dyn < 0) {
            asm volatile("griddepcontrol.wait;" ::: "memory");
            next_dyn = nstatic * int(gridDim.x) + int(atomicAdd(p.claim, 1u));
          }
          u = next_dyn;
          // claim the next unit now, so its atomic does not stall the stream
          if (u < p.units) next_dyn = nstatic * int(gridDim.x) + int(atomicAdd(p.claim, 1u));
        }
        if (u >= p.units) break;
        const int slot = j % nst;
        if (!wait_bar(b_empty + 8 * slot, (uint32_t(j / nst) & 1u) ^ 1u, abort_flag, p, ST_TIMEOUT_PRODUCER))
          break;
        const int rg = u / p.KS, sl = u - rg * p.KS;
        meta[slot] = make_int4(u, 0, 0, 0);
        mbar_expect_tx(b_full + 8 * slot, unit_bytes);
        // (x, y, z) = (byte in the 128-byte / 16-byte piece, row, piece along K)
        constexpr int PIECES = item_w_bytes(FMT) / BOX_W;   // 128-byte pieces of codes per item row
        tma_load_3d_hint(smem_u32(sW + size_t(slot) * ipu * item_w_bytes(FMT)), &tm_w, 0, rg * ROWS,
                         sl * PIECES * ipu, b_full + 8 * slot, pol);
        if (FMT == FMT_NVFP4)
          tma_load_3d_hint(smem_u32(sS + size_t(slot) * ipu * item_s_bytes(FMT)), &tm_s, 0, rg * ROWS,
                           sl * 2 * ipu, b_full + 8 * slot, pol);
        ++j;
      }
      // end marker: every consumer warp passes every unit, so one suffices
      if (!*abort_flag) {
        const int slot = j % nst;
        if (wait_bar(b_empty + 8 * slot, (uint32_t(j / nst) & 1u) ^ 1u, abort_flag, p, ST_TIMEOUT_PRODUCER)) {
          meta[slot] = make_int4(-1, 0, 0, 0);
          mbar_arrive(b_full + 8 * slot);
        }
      }
      if (*abort_flag) {
        // wait (bounded) for the copies still in flight before leaving
        const int first = j > nst ? j - nst : 0;
        for (int i = first; i < j; ++i) drain_bar(b_full + 8 * (i % nst), uint32_t(i / nst) & 1u, p);
      }
    }
    __syncwarp();
    asm volatile("griddepcontrol.wait;" ::: "memory");   // before the counters at the end
  } else {
    // ------------------------------------------------------------- consumers
    // X, the global scale, Y and the workspace may belong to the previous grid
    asm volatile("griddepcontrol.wait;" ::: "memory");
    stage_x(p, sX, emax, lo_flag, threadIdx.x - 32);
    const float gs = *p.gs;
    // per-token factors 2^-sh undoing the planes' scaling
    static_assert(MAX_M == 2, "per-token factors fh0, fh1");
    const float fh0 = emax[0] == INT_MIN ? 0.0f : ldexpf(1.0f, emax[0] - 14);
    const float fh1 = (p.M < 2 || emax[1] == INT_MIN) ? 0.0f : ldexpf(1.0f, emax[1] - 14);
    const int S = (*lo_flag ? 2 : 1) * p.M;
    {
      const int cw = warp - 1;
      if (FMT == FMT_FP8 || S <= 2)
        consume<1, FMT>(p, sW, sS, sX, sP, meta, cnt, b_full, b_empty, abort_flag, S, fh0, fh1, gs, cw, lane);
      else
        consume<2, FMT>(p, sW, sS, sX, sP, meta, cnt, b_full, b_empty, abort_flag, S, fh0, fh1, gs, cw, lane);
    }
  }
  __syncthreads();
  // the last CTA to finish resets the unit counter for the next call
  if (threadIdx.x == 0 && !*abort_flag) {
    __threadfence();
    if (atomicAdd(p.claim + 1, 1u) == gridDim.x - 1) {
      p.claim[0] = 0u;
      p.claim[1] = 0u;
      __threadfence();
    }
  }
}

}  // namespace rw

cudaError_t row_configure(RowConfig& c, int num_sms) {
  using namespace rw;
  if (c.M < 1 || c.M > MAX_M || c.K <= 0 || c.K % 256 != 0 || c.N <= 0) return cudaErrorInvalidConfiguration;
  if (c.fmt != FMT_NVFP4 && c.fmt != FMT_FP8) return cudaErrorInvalidConfiguration;
  int dev = 0, optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  c.units16 = (c.N + ROWS - 1) / ROWS;
  c.IT = (c.K + ITEM_K - 1) / ITEM_K;
  // K-slices of at most IPU_CAP items, split further while whole-slice units
  // would leave the SMs fewer than eight units each (keeping two items per slice)
  const int cap = c.fmt == FMT_FP8 ? IPU_CAP_FP8 : IPU_CAP;
  int KS = (c.IT + cap - 1) / cap;
  while ((long long)c.units16 * KS < 8LL * num_sms && (c.IT + 2 * KS - 1) / (2 * KS) >= 2) KS *= 2;
  c.ipu = (c.IT + KS - 1) / KS;
  c.KS = (c.IT + c.ipu - 1) / c.ipu;               // every slice holds at least one item
  c.units = c.units16 * c.KS;
  c.xstride = c.IT * XPIECE + XPAD;
  c.sp_row = 2 * c.M;
  const long long x_bytes = 2LL * c.M * c.xstride;
  const long long per_slot = (long long)c.ipu * (item_w_bytes(c.fmt) + item_s_bytes(c.fmt)) +
                             (long long)c.ipu * ROWS * c.sp_row * 4;
  const long long left = (long long)optin - 1024 - x_bytes - MISC_BYTES;
  long long nst = left / per_slot;
  if (nst > NST_MAX) nst = NST_MAX;
  if (nst < NST_MIN) return cudaErrorInvalidConfiguration;
  c.nst = int(nst);
  if ((long long)c.units + 2LL * c.nst * num_sms >= (1LL << 31)) return cudaErrorInvalidConfiguration;
  // X stays in registers while it is converted: at most XCH_MAX chunks per thread
  if ((long long)c.M * c.K / 8 > (long long)XCH_MAX * NCW * 32) return cudaErrorInvalidConfiguration;
  c.smem = size_t(1024 + nst * per_slot + x_bytes + MISC_BYTES);
  c.grid = num_sms;
  // workspace: status word, unit counters, K-split counters | K-split partials
  c.ws_counters_off = 256;
  c.ws_gcnt_off = 512;
  c.ws_partials_off = c.ws_gcnt_off + (c.KS > 1 ? ((size_t(c.units16) * 4 + 255) / 256) * 256 : 0);
  c.ws_bytes = c.ws_partials_off + (c.KS > 1 ? ((size_t(c.units16) * c.KS * c.M * ROWS * 4 + 255) / 256) * 256 : 0);
  e = cudaFuncSetAttribute(k_row<FMT_NVFP4>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_row<FMT_FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  return e;
}

bool encode_row_maps(int N, int K, int ipu, int fmt, const uint8_t* wp, const uint8_t* ws, void* map_w,
                     void* map_s) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint32_t one[3] = {1, 1, 1};
  if (fmt == rw::FMT_FP8) {
    // E4M3 codes [N][K] bytes as (128-byte piece, row, piece along K): boxes
    // of 128 bytes x 16 rows x 4 ipu pieces, 128-byte swizzle; no scale map
    const cuuint64_t dim8[3] = {128, cuuint64_t(N), cuuint64_t(K / 128)};
    const cuuint64_t str8[2] = {cuuint64_t(K), 128};
    const cuuint32_t box8[3] = {128, uint32_t(rw::ROWS), uint32_t(4 * ipu)};
    const CUresult r8 = fn(static_cast<CUtensorMap*>(map_w), CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
                           const_cast<uint8_t*>(wp), dim8, str8, box8, one, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    *static_cast<CUtensorMap*>(map_s) = *static_cast<CUtensorMap*>(map_w);
    return r8 == CUDA_SUCCESS;
  }
  // codes [N][K/2] bytes as (128-byte piece, row, piece along K): boxes of
  // 128 bytes x 16 rows x 2 ipu pieces, 128-byte swizzle
  const cuuint64_t dim_w[3] = {128, cuuint64_t(N), cuuint64_t(K / 256)};
  const cuuint64_t str_w[2] = {cuuint64_t(K / 2), 128};
  const cuuint32_t box_w[3] = {128, uint32_t(rw::ROWS), uint32_t(2 * ipu)};
  CUresult r = fn(static_cast<CUtensorMap*>(map_w), CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(wp),
                  dim_w, str_w, box_w, one, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  // scales [N][K/16] bytes as (16-byte piece, row, piece along K): boxes of
  // 16 bytes x 16 rows x 2 ipu pieces
  const cuuint64_t dim_s[3] = {16, cuuint64_t(N), cuuint64_t(K / 256)};
  const cuuint64_t str_s[2] = {cuuint64_t(K / 16), 16};
  const cuuint32_t box_s[3] = {16, uint32_t(rw::ROWS), uint32_t(2 * ipu)};
  r = fn(static_cast<CUtensorMap*>(map_s), CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(ws), dim_s,
         str_s, box_s, one, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

cudaError_t launch_row(const RowConfig& c, const void* map_w, const void* map_s, const float* row_scale,
                       const float* gs, const uint16_t* x, uint16_t* y, void* workspace,
                       long long timeout_cycles, bool stall, bool pdl, cudaStream_t st) {
  using namespace rw;
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  Params p;
  p.M = c.M; p.N = c.N; p.K = c.K;
  p.units16 = c.units16; p.KS = c.KS; p.units = c.units; p.IT = c.IT; p.ipu = c.ipu;
  p.nst = c.nst; p.xstride = c.xstride; p.sp_row = c.sp_row;
  p.gs = gs; p.x = x; p.y = y;
  p.row_scale = row_scale;
  p.status = reinterpret_cast<uint32_t*>(wsb);
  p.claim = reinterpret_cast<uint32_t*>(wsb + c.ws_counters_off);
  p.gcnt = reinterpret_cast<uint32_t*>(wsb + c.ws_gcnt_off);
  p.gpart = c.KS > 1 ? reinterpret_cast<float*>(wsb + c.ws_partials_off) : nullptr;
  p.timeout = timeout_cycles;
  p.stall = stall ? 1 : 0;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(c.grid);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = c.smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (c.fmt == FMT_FP8)
    return cudaLaunchKernelEx(&cfg, k_row<FMT_FP8>, *static_cast<const CUtensorMap*>(map_w),
                              *static_cast<const CUtensorMap*>(map_s), p);
  return cudaLaunchKernelEx(&cfg, k_row<FMT_NVFP4>, *static_cast<const CUtensorMap*>(map_w),
                            *static_cast<const CUtensorMap*>(map_s), p);
}

}  // namespace nvfp4
