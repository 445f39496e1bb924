// k_tc.cu -- tcgen05 tensor-core variant of the NVFP4 linear (sm_100a).
//
// Y[M][N] = X[M][K] W^T computed swap-AB: the 128-row MMA dimension is the
// weight rows, the N dimension of the MMA is the tokens (1 + drafted tokens
// checked in one pass; page "InventDB Sparkle", section "How it answers
// quickly"). The weight read dominates (page "Qwen3.8-27B-NVFP4-RTX5090 API &
// Inference Endpoint", section "Why lm_head is NVFP4, and why MTP is gone"),
// so the kernel is built around streaming W from HBM exactly once:
//
//   warp 0      TMA producer: 128-row x 256-element tiles of packed codes
//               (16 KB, 128-byte swizzle) and their E4M3 scales (2 KB) into a
//               6-stage shared-memory ring (mbarrier full/empty pairs).
//   warps 2-9   decoders: each thread owns one weight row and half of the
//               stage's K; it converts codes and scales with the hardware
//               e2m1x2/e4m3x2 -> f16x2 conversions, multiplies them (exact) and
//               stores the f16 A operand straight into tensor memory
//               (tcgen05.st), 3 TMEM stages deep.
//   warp 1      MMA issuer: tcgen05.mma kind::f16, A from TMEM, B = X from
//               shared memory, fp32 accumulators in TMEM (two buffers).
//   warps 10-13 epilogue: tcgen05.ld of the accumulators, global scale,
//               bf16 rounding, store (or deterministic split reduction).
//
// X operand. X is bf16 but kind::f16 needs A and B of the same type, and the
// exact W products are f16. Each CTA therefore keeps the K-slice of X it works
// on resident in shared memory as f16, scaled per token by a power of two so
// that the token's largest magnitude sits at 2^14, in two planes: "hi" holds
// every element within 2^28 of that maximum exactly (bf16 has 8 significant
// bits, f16 normals 11), "lo" holds the elements 2^28..2^57 below it, scaled up
// by 2^29. Elements further below keep only the lo plane's subnormal step
// (within 2^-68 of the maximum). Every product is then exact in fp32 and only
// the fp32 accumulation rounds.
//
// Work split. K is cut into S slices (so that a slice of X fits in shared
// memory); the CTAs of a slice share its (tile, k-step) space evenly (stream-K).
// A tile computed in several pieces writes fp32 partials to the workspace; the
// last piece to finish (atomic counter) adds them in k order, so results are
// identical from run to run. Counters are reset by that last piece.
//
// Every wait is bounded (clock64); on expiry the kernel records an error in
// the workspace status word, stops all roles, waits for its own in-flight TMA
// loads and MMAs, frees tensor memory and returns.
#include "kernels.h"
#include "nvfp4_device.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>
#include <climits>
#include <mutex>
#include <vector>

namespace nvfp4 {
namespace tc {

constexpr int KC = 256;                  // K elements per stage
constexpr int ROWS = 128;                // weight rows per tile (MMA M)
constexpr int NSTAGE = 6;                // shared-memory ring depth
constexpr int TSTAGE = 3;                // TMEM A ring depth
constexpr int W_BYTES = ROWS * KC / 2;   // 16384
constexpr int S_BYTES = ROWS * KC / 16;  // 2048
constexpr int A_COLS = KC / 2;           // TMEM columns per A stage (two f16 per column)
constexpr int D_COL0 = TSTAGE * A_COLS;  // 384: first accumulator column
constexpr int D_COLS = 64;               // columns per accumulator buffer (2 buffers)
// Consecutive MMAs of a stage rotate over D_COLS / n_mma independent
// accumulators (4 at N = 16, 2 at N = 32): MMAs into one accumulator
// serialise on it, independent ones overlap. The epilogue adds them.

constexpr int TMEM_COLS = 512;
// warp 0 producer, warps 1-2 MMA issuers (a tcgen05.mma holds its issuing
// thread for ~100+ cycles, so one thread cannot issue a stage's 16 MMAs at
// the stream rate; each warp owns half of the accumulators), 3-10 decoders,
// 11-14 epilogue
constexpr int NUM_WARPS = 15;
constexpr int NUM_THREADS = NUM_WARPS * 32;
constexpr int WARP_MMA0 = 1, NMW = 2;
constexpr int WARP_DEC0 = 3, NUM_DEC = 8, WARP_EPI0 = 11, NUM_EPI = 4;
constexpr int X_BUDGET = 96 * 1024;      // bytes of resident X slice
constexpr int LO_SHIFT = 29;             // lo plane scale relative to hi

// barrier ids (bar.sync)
constexpr int BAR_STAGED = 1;            // X staged + TMEM allocated: warps 1..13
constexpr int BAR_EPI = 2;               // epilogue warps
constexpr int BAR_STAGERS = 3;           // warps 2..13

// status word codes (OR-ed)
constexpr uint32_t ST_TIMEOUT_PRODUCER = 1u, ST_TIMEOUT_DECODE = 2u, ST_TIMEOUT_MMA = 4u,
                   ST_TIMEOUT_EPI = 8u, ST_TIMEOUT_DRAIN = 16u;

struct Params {
  int M, N, K, tiles, S, P, ks_base, ks_rem, nb, pmax, xk_max;
  const float* gs;
  const uint16_t* x;
  uint16_t* y;
  uint32_t* status;
  uint32_t* counters;
  float* partials;
  long long timeout;
  int stall;
};

struct Smem {
  uint32_t off_w, off_s, off_x, off_bar, off_misc, total;
};

__host__ __device__ inline Smem smem_layout(int nb, int xk_max) {
  Smem L;
  L.off_w = 0;
  L.off_s = L.off_w + NSTAGE * W_BYTES;
  L.off_x = L.off_s + NSTAGE * S_BYTES;
  L.off_bar = L.off_x + uint32_t(nb) * uint32_t(xk_max) * 2u;
  L.off_bar = (L.off_bar + 15u) & ~15u;
  L.off_misc = L.off_bar + 32 * 8;
  L.total = L.off_misc + 256 + 1024;     // + slack for 1024-byte alignment of the base
  return L;
}

// ---- PTX wrappers ---------------------------------------------------------

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  // K-major, no swizzle: 8-row x 16-byte core matrices; lbo = byte step
  // between the two 16-byte K halves of an MMA, sbo = byte step between
  // 8-row groups. Bits 46..47 = 1 (descriptor version for sm_100).
  return uint64_t((addr >> 4) & 0x3FFFu) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46);
}
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, "
      "%9, %10, %11, %12, %13, %14, %15, %16};"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]),
        "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]),
        "r"(v[13]), "r"(v[14]), "r"(v[15]) : "memory");
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

// Bounded wait on an mbarrier phase. Returns false if the CTA is aborting or
// the wait ran out (then the CTA starts aborting and the status word says who).
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
// Bounded wait that ignores the abort flag (used to drain in-flight work).
__device__ __forceinline__ void drain_bar(uint32_t b, uint32_t parity, const Params& p) {
  const long long t0 = clock64();
  while (!mbar_test(b, parity)) {
    if (clock64() - t0 > p.timeout) {
      atomicOr(p.status, ST_TIMEOUT_DRAIN);
      return;
    }
  }
}

// ---- work split -----------------------------------------------------------

struct Slice {
  int s, c, cnt, ks0;
  long long L, a, b;
};

__device__ __forceinline__ Slice my_slice(const Params& p) {
  Slice q;
  q.s = blockIdx.x / p.P;
  q.c = blockIdx.x % p.P;
  q.cnt = p.ks_base + (q.s < p.ks_rem ? 1 : 0);
  q.ks0 = q.s * p.ks_base + min(q.s, p.ks_rem);
  q.L = (long long)p.tiles * q.cnt;
  q.a = (long long)q.c * q.L / p.P;
  q.b = (long long)(q.c + 1) * q.L / p.P;
  return q;
}

__device__ __forceinline__ int slice_cnt(const Params& p, int s) {
  return p.ks_base + (s < p.ks_rem ? 1 : 0);
}

// Pieces of tile t within slice s.
__device__ __forceinline__ int pieces_in_slice(const Params& p, int t, int s) {
  const int cnt = slice_cnt(p, s);
  const long long L = (long long)p.tiles * cnt;
  return 1 + int(boundaries_in((long long)t * cnt, (long long)(t + 1) * cnt - 1, L, p.P));
}

// ---- X staging helpers ----------------------------------------------------

// ---- the kernel -------------------------------------------------------------

__global__ void __launch_bounds__(NUM_THREADS, 1)
k_tc(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_s,
     const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment by an offset: derived pointers stay in the shared window
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const Smem L = smem_layout(p.nb, p.xk_max);
  uint8_t* sW = smem + L.off_w;
  uint8_t* sS = smem + L.off_s;
  uint8_t* sX = smem + L.off_x;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.off_bar);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + L.off_misc);
  // misc: [0] tmem base, [1] abort, [2] need_lo, [3] last-piece flag,
  //       [16..31] emax per token (int)
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  int* emax = reinterpret_cast<int*>(misc + 16);

  const uint32_t b_full = smem_u32(bars), b_empty = b_full + 8 * NSTAGE,
                 b_afull = b_empty + 8 * NSTAGE, b_aempty = b_afull + 8 * TSTAGE,
                 b_dfull = b_aempty + 8 * TSTAGE, b_dempty = b_dfull + 16,
                 b_done = b_dempty + 16;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Slice sl = my_slice(p);
  const int klen = sl.cnt * KC;          // elements of X in this CTA's slice
  const int k0e = sl.ks0 * KC;
  const uint32_t sbo = uint32_t(p.xk_max) * 16u;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSTAGE; ++i) { mbar_init(b_full + 8 * i, 1); mbar_init(b_empty + 8 * i, NUM_DEC); }
    for (int i = 0; i < TSTAGE; ++i) { mbar_init(b_afull + 8 * i, NUM_DEC); mbar_init(b_aempty + 8 * i, NMW); }
    for (int i = 0; i < 2; ++i) { mbar_init(b_dfull + 8 * i, NMW); mbar_init(b_dempty + 8 * i, NUM_EPI); }
    for (int i = 0; i < NMW; ++i) mbar_init(b_done + 8 * i, 1);
    misc[1] = 0; misc[2] = 0; misc[3] = 0;
    for (int m = 0; m < 16; ++m) emax[m] = INT_MIN;
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
      long long n_issued = 0;
      if (!p.stall) {
        for (long long idx = sl.a; idx < sl.b; ++idx, ++n_issued) {
          const int t = int(idx / sl.cnt), j = int(idx % sl.cnt);
          const int st = int(n_issued % NSTAGE);
          const uint32_t ph = uint32_t(n_issued / NSTAGE) & 1u;
          if (!wait_bar(b_empty + 8 * st, ph ^ 1u, abort_flag, p, ST_TIMEOUT_PRODUCER)) break;
          mbar_expect_tx(b_full + 8 * st, W_BYTES + S_BYTES);
          tma_load_2d(smem_u32(sW + st * W_BYTES), &tm_w, (sl.ks0 + j) * (KC / 2), t * ROWS,
                      b_full + 8 * st);
          tma_load_2d(smem_u32(sS + st * S_BYTES), &tm_s, (sl.ks0 + j) * (KC / 16), t * ROWS,
                      b_full + 8 * st);
        }
      }
      if (*abort_flag) {
        // wait for the loads still in flight before the CTA may exit
        const long long first = n_issued > NSTAGE ? n_issued - NSTAGE : 0;
        for (long long i = first; i < n_issued; ++i)
          drain_bar(b_full + 8 * int(i % NSTAGE), uint32_t(i / NSTAGE) & 1u, p);
      }
    }
    __syncwarp();   // lanes 1..31 wait here for lane 0 before the block barrier
  } else {
    // -------------------------------------------- stage X (warps 2..13)
    if (warp >= WARP_DEC0) {
      // Every chunk (8 consecutive k of one token) is loaded once, all loads
      // of a thread in flight together; the slice holds at most
      // (nb/2) * xk_max / 8 <= 8 * 384 chunks, i.e. <= 8 per thread.
      constexpr int MAXC = 8;
      const int ts = threadIdx.x - WARP_DEC0 * 32, nts = (NUM_WARPS - WARP_DEC0) * 32;
      const int chunks = klen / 8;
      const int nreal = p.M * chunks;
      uint4 xv[MAXC];
#pragma unroll
      for (int c = 0; c < MAXC; ++c) {
        const int u = ts + c * nts;
        if (u < nreal) {
          const int m = u / chunks, kc = u - m * chunks;
          xv[c] = *reinterpret_cast<const uint4*>(p.x + size_t(m) * p.K + k0e + 8 * kc);
        }
      }
#pragma unroll
      for (int c = 0; c < MAXC; ++c) {
        const int u = ts + c * nts;
        if (u < nreal) {
          const int m = u / chunks;
          const uint32_t w[4] = {xv[c].x, xv[c].y, xv[c].z, xv[c].w};
          int mx = INT_MIN;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t b = (w[i >> 1] >> (16 * (i & 1))) & 0xFFFFu;
            if (b & 0x7FFFu) { uint32_t sg; mx = max(mx, bf16_exp(b, sg)); }
          }
          if (mx != INT_MIN) atomicMax(&emax[m], mx);
        }
      }
      named_bar(BAR_STAGERS, (NUM_WARPS - WARP_DEC0) * 32);
      const int mrows = p.M <= 8 ? 8 : 16;       // rows per plane
      bool lo_used = false;
#pragma unroll
      for (int c = 0; c < MAXC; ++c) {
        const int u = ts + c * nts;
        if (u < nreal) {
          const int m = u / chunks, kc = u - m * chunks;
          const int sh = (emax[m] == INT_MIN) ? 0 : 14 - emax[m];
          const uint32_t w[4] = {xv[c].x, xv[c].y, xv[c].z, xv[c].w};
          uint32_t hi[4] = {0u, 0u, 0u, 0u}, lo[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t b = (w[i >> 1] >> (16 * (i & 1))) & 0xFFFFu;
            if (b & 0x7FFFu) {
              uint32_t sg;
              const int th = bf16_exp(b, sg) + sh;
              if (th >= -14) hi[i >> 1] |= make_f16(b >> 15, th, sg) << (16 * (i & 1));
              else lo[i >> 1] |= make_f16_rn(b >> 15, th + LO_SHIFT, sg) << (16 * (i & 1));
            }
          }
          lo_used |= (lo[0] | lo[1] | lo[2] | lo[3]) != 0u;
          const int rl = mrows + m;
          *reinterpret_cast<uint4*>(sX + kc * 128 + (m >> 3) * sbo + (m & 7) * 16) =
              make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(sX + kc * 128 + (rl >> 3) * sbo + (rl & 7) * 16) =
              make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
      // rows of tokens >= M (both planes) are zero
      const int npad = mrows - p.M;
      for (int u = ts; u < 2 * npad * chunks; u += nts) {
        const int pr = u / chunks, kc = u - pr * chunks;
        const int r = (pr < npad) ? (p.M + pr) : (mrows + p.M + pr - npad);
        *reinterpret_cast<uint4*>(sX + kc * 128 + (r >> 3) * sbo + (r & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
      }
      if (lo_used) atomicOr(&misc[2], 1u);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    named_bar(BAR_STAGED, (NUM_WARPS - 1) * 32);
    fence_after();
    const bool need_lo = misc[2] != 0;
    const int n_mma = (p.M <= 8) ? 16 : (need_lo ? 32 : 16);
    const int nacc = D_COLS / n_mma;

    if (warp < WARP_DEC0) {
      // ---------------------------------------------------------- MMA issuers
      // warp w issues the MMAs of the accumulators a with a % NMW == w
      const int mw = warp - WARP_MMA0;
      if (lane == 0) {
        const uint32_t idesc = (1u << 4) | (uint32_t(n_mma >> 3) << 17) | (uint32_t(ROWS >> 4) << 24);
        const uint32_t x_base = smem_u32(sX);
        long long i = 0;
        int sidx = 0;
        bool ok = true;
        long long idx = sl.a;
        while (ok && idx < sl.b) {
          const int t = int(idx / sl.cnt);
          const long long seg_end = min(sl.b, (long long)(t + 1) * sl.cnt);
          const int db = sidx & 1;
          if (!wait_bar(b_dempty + 8 * db, (uint32_t(sidx >> 1) & 1u) ^ 1u, abort_flag, p,
                        ST_TIMEOUT_MMA)) { ok = false; break; }
          fence_after();
          const uint32_t d_tmem = tmem + D_COL0 + db * D_COLS;
          bool first = true;
          for (; idx < seg_end; ++idx, ++i) {
            const int j = int(idx % sl.cnt);
            const int ts = int(i % TSTAGE);
            if (!wait_bar(b_afull + 8 * ts, uint32_t(i / TSTAGE) & 1u, abort_flag, p,
                          ST_TIMEOUT_MMA)) { ok = false; break; }
            fence_after();
#pragma unroll
            for (int kk = 0; kk < KC / 16; ++kk) {
              if ((kk % nacc) % NMW != mw) continue;
              const uint32_t a_tmem = tmem + ts * A_COLS + kk * 8;
              const uint64_t bd = smem_desc(x_base + uint32_t(j * KC + kk * 16) * 16u, 128u, sbo);
              const int acc_i = kk % nacc;
              mma_f16_ts(d_tmem + acc_i * n_mma, a_tmem, bd, idesc, (first && kk < nacc) ? 0u : 1u);
            }
            first = false;
            mma_commit(b_aempty + 8 * ts);
          }
          if (!ok) break;
          mma_commit(b_dfull + 8 * db);
          ++sidx;
        }
        // all MMAs issued by this thread complete before tensor memory is freed
        mma_commit(b_done + 8 * mw);
        drain_bar(b_done + 8 * mw, 0u, p);
      }
      __syncwarp();   // reconverge warp 1 before the block barrier and dealloc
    } else if (warp < WARP_EPI0) {
      // ------------------------------------------------------------ decoders
      const int q = warp & 3, h = (warp - WARP_DEC0) >> 2;
      const int r = 32 * q + lane;
      const uint32_t t_row = tmem + (uint32_t(32 * q) << 16) + h * (A_COLS / 2);
      long long i = 0;
      for (long long idx = sl.a; idx < sl.b; ++idx, ++i) {
        const int st = int(i % NSTAGE);
        bool ok = wait_bar(b_full + 8 * st, uint32_t(i / NSTAGE) & 1u, abort_flag, p, ST_TIMEOUT_DECODE);
        if (!__all_sync(0xffffffffu, ok)) break;
        const uint8_t* rowp = sW + st * W_BYTES + r * 128;
        uint4 c[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          c[u] = *reinterpret_cast<const uint4*>(rowp + (((4 * h + u) ^ (r & 7)) << 4));
        const uint4 sc = *reinterpret_cast<const uint4*>(sS + st * S_BYTES + r * 16);
        __syncwarp();
        if (lane == 0) mbar_arrive(b_empty + 8 * st);
        const int ts = int(i % TSTAGE);
        ok = wait_bar(b_aempty + 8 * ts, (uint32_t(i / TSTAGE) & 1u) ^ 1u, abort_flag, p,
                      ST_TIMEOUT_DECODE);
        if (!__all_sync(0xffffffffu, ok)) break;
        fence_after();
        const uint32_t s4[2] = {h ? sc.z : sc.x, h ? sc.w : sc.y};   // 8 scale bytes
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          // chunk u: 32 elements = scale blocks 2u, 2u+1
          const uint32_t sp = e4m3x2_to_f16x2(s4[u >> 1] >> (16 * (u & 1)));
          const uint32_t sa = bcast_lo(sp), sb = bcast_hi(sp);
          const uint32_t wv[4] = {c[u].x, c[u].y, c[u].z, c[u].w};
          uint32_t out[16];
#pragma unroll
          for (int wi = 0; wi < 4; ++wi) {
            uint32_t hh[4];
            e2m1x8_to_f16x2x4(wv[wi], hh);
            const uint32_t s = wi < 2 ? sa : sb;
#pragma unroll
            for (int e = 0; e < 4; ++e) out[4 * wi + e] = hmul2(hh[e], s);
          }
          tmem_st16(t_row + ts * A_COLS + 16 * u, out);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(b_afull + 8 * ts);
      }
    } else {
      // ------------------------------------------------------------ epilogue
      const int q = warp & 3;
      const int r = 32 * q + lane;
      const float gs = *p.gs;
      const int et = threadIdx.x - WARP_EPI0 * 32;          // 0..127
      const int mrows = p.M <= 8 ? 8 : 16;
      // unscale factors of the hi and lo planes per token (exact powers of two)
      float f_hi[16], f_lo[16];
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        const bool live = m < p.M && emax[m] != INT_MIN;
        const int sh = live ? 14 - emax[m] : 0;
        f_hi[m] = live ? ldexpf(1.0f, -sh) : 0.0f;
        f_lo[m] = (live && mrows + m < n_mma) ? ldexpf(1.0f, -(sh + LO_SHIFT)) : 0.0f;
      }
      int sidx = 0;
      long long idx = sl.a;
      while (idx < sl.b) {
        const int t = int(idx / sl.cnt);
        const long long seg_start = idx;
        const long long seg_end = min(sl.b, (long long)(t + 1) * sl.cnt);
        idx = seg_end;
        const int db = sidx & 1;
        const bool ok = wait_bar(b_dfull + 8 * db, uint32_t(sidx >> 1) & 1u, abort_flag, p,
                                 ST_TIMEOUT_EPI);
        if (!named_bar_and(BAR_EPI, NUM_EPI * 32, ok)) break;
        fence_after();
        uint32_t raw[64];
        const uint32_t taddr = tmem + (uint32_t(32 * q) << 16) + D_COL0 + db * D_COLS;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (16 * u < nacc * n_mma) tmem_ld16(taddr + 16 * u, raw + 16 * u);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        float acc[32];
        if (n_mma == 16) {
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            acc[c] = ((__uint_as_float(raw[c]) + __uint_as_float(raw[16 + c])) +
                      __uint_as_float(raw[32 + c])) + __uint_as_float(raw[48 + c]);
            acc[16 + c] = 0.0f;
          }
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) acc[c] = __uint_as_float(raw[c]) + __uint_as_float(raw[32 + c]);
        }
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(b_dempty + 8 * db);
        ++sidx;
        float v[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const float lo = (mrows == 8) ? acc[(8 + m) & 31] : acc[(16 + m) & 31];
          v[m] = acc[m] * f_hi[m] + lo * f_lo[m];
        }
        // pieces of this tile: over all slices, and this piece's ordinal
        int npieces = 0;
        for (int s2 = 0; s2 < p.S; ++s2) npieces += pieces_in_slice(p, t, s2);
        const int row = t * ROWS + r;
        if (npieces == 1) {
          if (row < p.N) {
#pragma unroll
            for (int m = 0; m < 16; ++m)
              if (m < p.M) p.y[size_t(m) * p.N + row] = float_to_bf16_bits(gs * v[m]);
          }
          continue;
        }
        const int ord = int(boundaries_in((long long)t * sl.cnt, seg_start, sl.L, p.P));
        const long long slot = ((long long)t * p.S + sl.s) * p.pmax + ord;
        float* part = p.partials + slot * p.M * ROWS;
#pragma unroll
        for (int m = 0; m < 16; ++m)
          if (m < p.M) part[m * ROWS + r] = v[m];
        // publish: CTA barrier, then one gpu-scope fence + counter increment
        // (the fence is cumulative over the writes ordered before it by the barrier)
        named_bar(BAR_EPI, NUM_EPI * 32);
        if (et == 0) {
          __threadfence();
          const unsigned old = atomicAdd(&p.counters[t], 1u);
          __threadfence();
          misc[3] = (old == unsigned(npieces - 1)) ? 1u : 0u;
        }
        named_bar(BAR_EPI, NUM_EPI * 32);
        const bool last = misc[3] != 0;
        if (last) {
          float sum[16];
#pragma unroll
          for (int m = 0; m < 16; ++m) sum[m] = 0.0f;
          for (int s2 = 0; s2 < p.S; ++s2) {
            const int np = pieces_in_slice(p, t, s2);
            for (int o = 0; o < np; ++o) {
              const float* pp = p.partials + (((long long)t * p.S + s2) * p.pmax + o) * p.M * ROWS;
#pragma unroll
              for (int m = 0; m < 16; ++m)
                if (m < p.M) sum[m] += __ldcg(pp + m * ROWS + r);
            }
          }
          if (row < p.N) {
#pragma unroll
            for (int m = 0; m < 16; ++m)
              if (m < p.M) p.y[size_t(m) * p.N + row] = float_to_bf16_bits(gs * sum[m]);
          }
          if (et == 0) atomicExch(&p.counters[t], 0u);
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

// ---- host side --------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

}  // namespace tc

cudaError_t tc_configure(TcConfig& c, int num_sms) {
  using namespace tc;
  if (c.M < 1 || c.M > 16 || c.K % KC != 0 || c.K <= 0 || c.N <= 0) return cudaErrorInvalidValue;
  c.nb = c.M <= 8 ? 16 : 32;
  c.tiles = (c.N + ROWS - 1) / ROWS;
  const int ksteps = c.K / KC;
  const int max_ks = X_BUDGET / (c.nb * KC * 2);
  int S = (ksteps + max_ks - 1) / max_ks;
  if (S < 1) S = 1;
  int P = num_sms / S;
  if (P < 1) return cudaErrorInvalidConfiguration;
  const int ks_base = ksteps / S, ks_rem = ksteps % S;
  const long long min_units = (long long)c.tiles * ks_base;
  if (P > min_units) P = int(min_units);
  c.S = S; c.P = P; c.ks_base = ks_base; c.ks_rem = ks_rem;
  c.grid = S * P;
  c.xk_max = (ks_base + (ks_rem ? 1 : 0)) * KC;
  // X staging holds at most 8 chunks of 8 elements per staging thread
  if ((long long)c.M * c.xk_max / 8 > 8LL * (NUM_WARPS - WARP_DEC0) * 32) return cudaErrorInvalidConfiguration;
  // pieces per (tile, slice): simulate the boundaries
  int pmax = 1;
  bool split = S > 1;
  for (int s = 0; s < S; ++s) {
    const int cnt = ks_base + (s < ks_rem ? 1 : 0);
    const long long L = (long long)c.tiles * cnt;
    std::vector<int> pieces(c.tiles, 1);
    for (int cc = 1; cc < P; ++cc) {
      const long long bnd = (long long)cc * L / P;
      if (bnd % cnt != 0) {                 // boundary strictly inside a tile
        pieces[bnd / cnt] += 1;
        split = true;
      }
    }
    for (int t = 0; t < c.tiles; ++t) pmax = pieces[t] > pmax ? pieces[t] : pmax;
  }
  c.pmax = pmax;
  c.split = split;
  const Smem L = smem_layout(c.nb, c.xk_max);
  c.smem = L.total;
  c.ws_counters_off = 256;
  c.ws_partials_off = c.ws_counters_off + ((size_t(c.tiles) * 4 + 255) / 256) * 256;
  c.ws_bytes = split ? c.ws_partials_off + size_t(c.tiles) * S * pmax * c.M * ROWS * 4 : 256;
  // The attribute is per function, shared by every plan: set it to the
  // device's opt-in maximum once rather than to this plan's size.
  int dev = 0, optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  if (c.smem > size_t(optin)) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(k_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e != cudaSuccess) return e;
  if (!encode_fn()) return cudaErrorNotSupported;
  return cudaSuccess;
}

bool encode_weight_maps(int N, int K, int box_rows, const uint8_t* wp, const uint8_t* ws,
                        void* map_w, void* map_s) {
  auto fn = tc::encode_fn();
  if (!fn) return false;
  // codes: [N][K/2] bytes, box 128 bytes x box_rows rows, 128-byte swizzle
  const cuuint64_t dim_w[2] = {cuuint64_t(K / 2), cuuint64_t(N)};
  const cuuint64_t str_w[1] = {cuuint64_t(K / 2)};
  const cuuint32_t box_w[2] = {128, cuuint32_t(box_rows)};
  const cuuint32_t one[2] = {1, 1};
  CUresult r = fn(static_cast<CUtensorMap*>(map_w), CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                  const_cast<uint8_t*>(wp), dim_w, str_w, box_w, one,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  // scales: [N][K/16] bytes, box 16 bytes x box_rows rows
  const cuuint64_t dim_s[2] = {cuuint64_t(K / 16), cuuint64_t(N)};
  const cuuint64_t str_s[1] = {cuuint64_t(K / 16)};
  const cuuint32_t box_s[2] = {16, cuuint32_t(box_rows)};
  r = fn(static_cast<CUtensorMap*>(map_s), CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
         const_cast<uint8_t*>(ws), dim_s, str_s, box_s, one, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_x_planes_map(const void* planes, int pitch_bytes, int cols, int box_bytes, void* map) {
  auto fn = tc::encode_fn();
  if (!fn) return false;
  // f16 X planes in the workspace: `cols` columns of `pitch_bytes`, read as
  // 32-bit words, one box = one K-step of every column
  const cuuint64_t dim[2] = {cuuint64_t(pitch_bytes / 4), cuuint64_t(cols)};
  const cuuint64_t str[1] = {cuuint64_t(pitch_bytes)};
  const cuuint32_t box[2] = {cuuint32_t(box_bytes / 4), cuuint32_t(cols)};
  const cuuint32_t one[2] = {1, 1};
  const CUresult r = fn(static_cast<CUtensorMap*>(map), CU_TENSOR_MAP_DATA_TYPE_UINT32, 2,
                        const_cast<void*>(planes), dim, str, box, one, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool tensor_maps_supported() { return tc::encode_fn() != nullptr; }

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() { return tc::encode_fn(); }

cudaError_t launch_tc(const TcConfig& c, const void* map_w, const void* map_s, const float* gs,
                      const uint16_t* x, uint16_t* y, void* workspace, long long timeout_cycles,
                      bool stall, cudaStream_t st) {
  using namespace tc;
  Params p;
  p.M = c.M; p.N = c.N; p.K = c.K; p.tiles = c.tiles; p.S = c.S; p.P = c.P;
  p.ks_base = c.ks_base; p.ks_rem = c.ks_rem; p.nb = c.nb; p.pmax = c.pmax; p.xk_max = c.xk_max;
  p.gs = gs; p.x = x; p.y = y;
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  p.status = reinterpret_cast<uint32_t*>(wsb);
  p.counters = reinterpret_cast<uint32_t*>(wsb + c.ws_counters_off);
  p.partials = c.split ? reinterpret_cast<float*>(wsb + c.ws_partials_off) : nullptr;
  p.timeout = timeout_cycles;
  p.stall = stall ? 1 : 0;
  k_tc<<<c.grid, NUM_THREADS, c.smem, st>>>(*static_cast<const CUtensorMap*>(map_w),
                                             *static_cast<const CUtensorMap*>(map_s), p);
  return cudaGetLastError();
}

}  // namespace nvfp4
