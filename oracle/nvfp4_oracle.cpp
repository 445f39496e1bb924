// nvfp4_oracle.cpp -- plain, slow, host-only reference for the NVFP4 linear.
//
// TEST INFRASTRUCTURE ONLY (see nvfp4_oracle.h). No code here is shared with
// the CUDA library; nothing on the product path may load this file's library.
//
// Build: g++ -O2 -std=c++17 -ffp-contract=off -fno-fast-math -shared -fPIC -pthread
// (-ffp-contract=off keeps every fp32 quantiser step a separately rounded op.)

#include "nvfp4_oracle.h"

#include <cmath>
#include <cstring>
#include <thread>
#include <vector>
#include <algorithm>

namespace {

// Ranges shorter than this run on the calling thread alone.
constexpr int64_t kParallelMin = 4096;

// Run body(lo, hi) over [0, n) split into nthreads contiguous pieces
// (ora_threads_for(n, nthreads) of them are non-empty).
template <class F>
void split_range(int64_t n, int nthreads, F body) {
  if (nthreads < 1) nthreads = 1;
  if (n < kParallelMin || nthreads == 1) { body(int64_t(0), n); return; }
  int64_t per = (n + nthreads - 1) / nthreads;
  std::vector<std::thread> ts;
  for (int t = 0; t < nthreads; ++t) {
    int64_t lo = t * per, hi = std::min(n, lo + per);
    if (lo >= hi) break;
    ts.emplace_back([=] { body(lo, hi); });
  }
  for (auto& th : ts) th.join();
}

// All 127 non-negative finite E4M3 magnitudes, indexed by code 0x00..0x7E.
// They increase with the code, which the nearest-value search relies on.
struct E4M3Table {
  double v[127];
  E4M3Table() { for (int c = 0; c < 127; ++c) v[c] = ora_e4m3_decode(uint32_t(c)); }
};
const E4M3Table& e4m3_table() { static E4M3Table t; return t; }

// E2M1 magnitudes by code 0..7.
const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

// Nearest entry of an increasing table to a (0 <= a < table[n-1]), ties to the
// even index (for both formats the code's last bit is the mantissa's last bit).
int nearest_even(const double* table, int n, double a) {
  int lo = 0, hi = n - 1;            // invariant: table[lo] <= a < table[hi]
  while (hi - lo > 1) {
    int mid = (lo + hi) / 2;
    if (table[mid] <= a) lo = mid; else hi = mid;
  }
  double dlo = a - table[lo], dhi = table[hi] - a;   // exact in fp64
  if (dlo < dhi) return lo;
  if (dhi < dlo) return hi;
  return (lo % 2 == 0) ? lo : hi;
}

}  // namespace

extern "C" {

int ora_threads_for(int64_t n, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (n < kParallelMin || nthreads == 1) return 1;
  const int64_t per = (n + nthreads - 1) / nthreads;
  return int((n + per - 1) / per);
}

// OCP Microscaling spec, E2M1: sign bit 3, exponent bits 2..1 (bias 1),
// mantissa bit 0; exponent 0 is subnormal with value m * 0.5.
double ora_e2m1_decode(uint32_t code) {
  uint32_t s = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
  double mag = (e == 0) ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, int(e) - 1);
  return s ? -mag : mag;
}

// OCP 8-bit FP spec, E4M3 ("fn"): sign bit 7, exponent bits 6..3 (bias 7),
// mantissa bits 2..0; exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN;
// no infinities, so the largest finite value is 1.75 * 2^8 = 448.
double ora_e4m3_decode(uint32_t code) {
  code &= 0xFFu;
  uint32_t s = code >> 7, e = (code >> 3) & 15u, m = code & 7u;
  if (e == 15 && m == 7) return std::nan("");
  double mag = (e == 0) ? std::ldexp(double(m) / 8.0, -6)
                        : std::ldexp(1.0 + double(m) / 8.0, int(e) - 7);
  return s ? -mag : mag;
}

int ora_e4m3_is_nan(uint32_t code) { return ((code & 0x7Fu) == 0x7Fu) ? 1 : 0; }

uint32_t ora_e2m1_encode(float r) {
  if (std::isnan(r)) return 0;
  double a = std::fabs(double(r));
  uint32_t mag = (a >= 6.0) ? 7u : uint32_t(nearest_even(kE2M1, 8, a));
  if (mag == 0) return 0;                       // reading R6: no negative zero
  return (std::signbit(r) ? 8u : 0u) | mag;
}

uint32_t ora_e4m3_encode(float u) {
  if (std::isnan(u)) return 0x7Fu;
  double a = std::fabs(double(u));
  uint32_t mag = (a >= 448.0) ? 0x7Eu
                              : uint32_t(nearest_even(e4m3_table().v, 127, a));
  return (std::signbit(u) ? 0x80u : 0u) | mag;
}

int ora_global_scale(const float* w, int64_t n, float* gs, int nthreads) {
  if (!gs || (n > 0 && !w) || n < 0) return -1;
  std::vector<float> part(std::max(1, nthreads), 0.0f);
  std::vector<int> bad(std::max(1, nthreads), 0);
  int nt = std::max(1, nthreads);
  int64_t per = (n + nt - 1) / nt;
  std::vector<std::thread> ts;
  for (int t = 0; t < nt; ++t) {
    ts.emplace_back([&, t] {
      int64_t lo = t * per, hi = std::min(n, lo + per);
      float m = 0.0f; int b = 0;
      for (int64_t i = lo; i < hi; ++i) {
        float a = std::fabs(w[i]);
        if (!std::isfinite(a)) b = 1;
        else if (a > m) m = a;
      }
      part[t] = m; bad[t] = b;
    });
  }
  for (auto& th : ts) th.join();
  float amax = 0.0f;
  for (int t = 0; t < nt; ++t) {
    if (bad[t]) return -2;
    amax = std::max(amax, part[t]);
  }
  // Reading R3: gs = amax / (6 * 448); 6*448 = 2688 is exact in fp32.
  *gs = amax / 2688.0f;
  return 0;
}

int ora_quantize_rows(const float* w, int64_t nrows, int64_t K, float gs,
                      uint8_t* packed, uint8_t* scales, int nthreads) {
  if (nrows < 0 || K < 0 || K % 16 != 0) return -1;
  if (nrows == 0 || K == 0) return 0;
  if (!w || !packed || !scales) return -1;
  const int64_t nblk = K / 16;
  split_range(nrows, nthreads, [&](int64_t lo, int64_t hi) {
    for (int64_t n = lo; n < hi; ++n) {
      const float* row = w + n * K;
      for (int64_t b = 0; b < nblk; ++b) {
        const float* blk = row + b * 16;
        // Block amax, exact.
        float amax_b = 0.0f;
        for (int j = 0; j < 16; ++j) amax_b = std::max(amax_b, std::fabs(blk[j]));
        // Reading R7: each step below is one fp32 operation, rounded to nearest.
        float t = amax_b / 6.0f;                 // block amax / 6
        float u = (gs > 0.0f) ? t / gs : 0.0f;   // ... under the global scale
        uint32_t s_code = ora_e4m3_encode(u);    // RNE, saturating (reading R4)
        float ds = float(ora_e4m3_decode(s_code));  // exact
        float denom = ds * gs;                   // quantise against the DECODED scale
        scales[n * nblk + b] = uint8_t(s_code);
        uint8_t* out = packed + n * (K / 2) + b * 8;
        for (int j = 0; j < 16; j += 2) {
          uint32_t q0 = 0, q1 = 0;
          if (denom > 0.0f) {                    // reading R5
            q0 = ora_e2m1_encode(blk[j] / denom);
            q1 = ora_e2m1_encode(blk[j + 1] / denom);
          }
          out[j / 2] = uint8_t(q0 | (q1 << 4));  // reading R1: even element low
        }
      }
    }
  });
  return 0;
}

int ora_quantize(const float* w, int64_t N, int64_t K, uint8_t* packed,
                 uint8_t* scales, float* gs, int nthreads) {
  if (N < 0 || K < 0 || K % 16 != 0 || !gs) return -1;
  int rc = ora_global_scale(w, N * K, gs, nthreads);
  if (rc) return rc;
  return ora_quantize_rows(w, N, K, *gs, packed, scales, nthreads);
}

int ora_dequant_f64(const uint8_t* packed, const uint8_t* scales, float gs,
                    int64_t N, int64_t K, double* out) {
  if (N < 0 || K < 0 || K % 16 != 0) return -1;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      uint32_t byte = packed[n * (K / 2) + k / 2];
      uint32_t code = (k % 2 == 0) ? (byte & 0xFu) : (byte >> 4);
      double s = ora_e4m3_decode(scales[n * (K / 16) + k / 16]);
      out[n * K + k] = ora_e2m1_decode(code) * s * double(gs);
    }
  return 0;
}

int ora_dequant_bf16_nogs(const uint8_t* packed, const uint8_t* scales,
                          int64_t N, int64_t K, uint16_t* out) {
  if (N < 0 || K < 0 || K % 16 != 0) return -1;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      uint32_t byte = packed[n * (K / 2) + k / 2];
      uint32_t code = (k % 2 == 0) ? (byte & 0xFu) : (byte >> 4);
      double p = ora_e2m1_decode(code) * ora_e4m3_decode(scales[n * (K / 16) + k / 16]);
      out[n * K + k] = ora_bf16_rne(p);
    }
  return 0;
}

int64_t ora_count_bad(const uint8_t* scales, int64_t n_scales, float gs) {
  int64_t bad = 0;
  for (int64_t i = 0; i < n_scales; ++i) bad += ora_e4m3_is_nan(scales[i]);
  if (std::isnan(gs) || std::isinf(gs) || gs < 0.0f) bad += 1;
  return bad;
}

double ora_bf16_value(uint16_t bits) {
  uint32_t u = uint32_t(bits) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return double(f);
}

uint16_t ora_bf16_rne(double v) {
  if (std::isnan(v)) return 0x7FC0;
  uint16_t sign = std::signbit(v) ? 0x8000 : 0;
  double a = std::fabs(v);
  if (a == 0.0) return sign;
  // Midpoint between the largest finite bf16 ((2 - 2^-7) * 2^127) and 2^128;
  // it rounds to the even neighbour, 2^128, i.e. to infinity.
  if (a >= std::ldexp(2.0 - std::ldexp(1.0, -8), 127)) return uint16_t(sign | 0x7F80);
  int ex;
  std::frexp(a, &ex);                   // a = f * 2^ex, f in [0.5, 1)
  int E = ex - 1;                       // a in [2^E, 2^(E+1))
  double quantum = (E < -126) ? std::ldexp(1.0, -133) : std::ldexp(1.0, E - 7);
  double r = std::nearbyint(a / quantum) * quantum;   // ties to even
  float f = float(r);                   // exact: r is a bf16 value
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return uint16_t(sign | (u >> 16));
}

int ora_linear(const uint8_t* packed, const uint8_t* scales, float gs,
               const uint16_t* x_bf16, int64_t M, int64_t N, int64_t K,
               const int64_t* rows, int64_t nrows, double* y, double* absdot,
               int nthreads) {
  if (M < 0 || N < 0 || K < 0 || K % 16 != 0 || nrows < 0) return -1;
  if (!rows && nrows != N) return -1;
  if (nrows == 0 || M == 0) return 0;
  if (!y || (K > 0 && (!packed || !scales || !x_bf16))) return -1;
  if (rows)
    for (int64_t i = 0; i < nrows; ++i)
      if (rows[i] < 0 || rows[i] >= N) return -1;
  std::vector<double> x(size_t(M * K));
  for (int64_t i = 0; i < M * K; ++i) x[size_t(i)] = ora_bf16_value(x_bf16[i]);
  split_range(nrows, nthreads, [&](int64_t lo, int64_t hi) {
    std::vector<double> wrow(static_cast<size_t>(K));
    for (int64_t i = lo; i < hi; ++i) {
      int64_t n = rows ? rows[i] : i;
      // Dequantise row n exactly: w_hat = e2m1(q) * e4m3(s) * gs.
      for (int64_t k = 0; k < K; ++k) {
        uint32_t byte = packed[n * (K / 2) + k / 2];
        uint32_t code = (k % 2 == 0) ? (byte & 0xFu) : (byte >> 4);
        wrow[size_t(k)] = ora_e2m1_decode(code) *
                          ora_e4m3_decode(scales[n * (K / 16) + k / 16]) * double(gs);
      }
      for (int64_t m = 0; m < M; ++m) {
        const double* xm = x.data() + m * K;
        double acc = 0.0, aacc = 0.0;
        for (int64_t k = 0; k < K; ++k) {
          double p = wrow[size_t(k)] * xm[k];
          acc += p;
          aacc += std::fabs(p);
        }
        y[m * nrows + i] = acc;
        if (absdot) absdot[m * nrows + i] = aacc;
      }
    }
  });
  return 0;
}

// SiLU(v) = v * sigmoid(v) = v / (1 + e^-v). For v below about -709, e^-v
// overflows to +inf and the quotient is -0.0, the limit of SiLU there.
double ora_silu(double v) { return v / (1.0 + std::exp(-v)); }

// Gated output of a fused gate+up projection (reading R11): weight rows 2c
// and 2c+1 are the gate and up rows of output column c. Both dot products are
// taken by ora_linear (same exact dequantisation, fp64 sums); the gate passes
// through SiLU and multiplies the up value, all in fp64.
int ora_swiglu_linear(const uint8_t* packed, const uint8_t* scales, float gs,
                      const uint16_t* x_bf16, int64_t M, int64_t N2, int64_t K,
                      const int64_t* cols, int64_t ncols, double* h, double* gate,
                      double* up, double* absdot_gate, double* absdot_up, int nthreads) {
  if (M < 0 || N2 < 0 || N2 % 2 != 0 || ncols < 0) return -1;
  if (!cols && ncols != N2 / 2) return -1;
  if (ncols == 0 || M == 0) return 0;
  if (!h) return -1;
  std::vector<int64_t> rows(size_t(2 * ncols));
  for (int64_t c = 0; c < ncols; ++c) {
    int64_t col = cols ? cols[c] : c;
    if (col < 0 || col >= N2 / 2) return -1;
    rows[size_t(c)] = 2 * col;                 // gate rows first ...
    rows[size_t(ncols + c)] = 2 * col + 1;     // ... then the matching up rows
  }
  std::vector<double> y(size_t(M * 2 * ncols)), ad(size_t(M * 2 * ncols));
  int st = ora_linear(packed, scales, gs, x_bf16, M, N2, K, rows.data(), 2 * ncols,
                      y.data(), ad.data(), nthreads);
  if (st != 0) return st;
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t c = 0; c < ncols; ++c) {
      double g = y[size_t(m * 2 * ncols + c)];
      double u = y[size_t(m * 2 * ncols + ncols + c)];
      h[m * ncols + c] = ora_silu(g) * u;
      if (gate) gate[m * ncols + c] = g;
      if (up) up[m * ncols + c] = u;
      if (absdot_gate) absdot_gate[m * ncols + c] = ad[size_t(m * 2 * ncols + c)];
      if (absdot_up) absdot_up[m * ncols + c] = ad[size_t(m * 2 * ncols + ncols + c)];
    }
  }
  return 0;
}

// The k largest entries of each row of y [M][N], largest first; equal values
// are ordered by ascending index (reading R10: the lowest index wins a tie).
// k = 1 is the greedy argmax.
int ora_topk(const double* y, int64_t M, int64_t N, int64_t k, int64_t* idx) {
  if (M < 0 || N < 0 || k < 0 || k > N) return -1;
  if (M == 0 || k == 0) return 0;
  if (!y || !idx) return -1;
  for (int64_t i = 0; i < M * N; ++i)
    if (std::isnan(y[i])) return -3;
  std::vector<int64_t> order(static_cast<size_t>(N));
  for (int64_t m = 0; m < M; ++m) {
    const double* row = y + m * N;
    for (int64_t j = 0; j < N; ++j) order[size_t(j)] = j;
    auto before = [row](int64_t a, int64_t b) {
      return row[a] > row[b] || (row[a] == row[b] && a < b);
    };
    std::partial_sort(order.begin(), order.begin() + k, order.end(), before);
    for (int64_t j = 0; j < k; ++j) idx[m * k + j] = order[size_t(j)];
  }
  return 0;
}

// W4A4 reference (reading R14): both operands NVFP4. X [M][K] is given as
// codes, block scales and its own per-tensor scale, like W; each is
// dequantised exactly by ora_dequant_f64 and the products are summed in fp64.
int ora_linear_w4a4(const uint8_t* w_packed, const uint8_t* w_scales, float gs_w,
                    const uint8_t* x_packed, const uint8_t* x_scales, float gs_x,
                    int64_t M, int64_t N, int64_t K, const int64_t* rows, int64_t nrows,
                    double* y, double* absdot, int nthreads) {
  if (M < 0 || N < 0 || K < 0 || K % 16 != 0 || nrows < 0) return -1;
  if (!rows && nrows != N) return -1;
  if (nrows == 0 || M == 0) return 0;
  if (!y || (K > 0 && (!w_packed || !w_scales || !x_packed || !x_scales))) return -1;
  if (rows)
    for (int64_t i = 0; i < nrows; ++i)
      if (rows[i] < 0 || rows[i] >= N) return -1;
  std::vector<double> xhat(size_t(M * K));
  if (K > 0) ora_dequant_f64(x_packed, x_scales, gs_x, M, K, xhat.data());
  split_range(nrows, nthreads, [&](int64_t lo, int64_t hi) {
    std::vector<double> what(static_cast<size_t>(K));
    for (int64_t i = lo; i < hi; ++i) {
      const int64_t n = rows ? rows[i] : i;
      if (K > 0) ora_dequant_f64(w_packed + n * (K / 2), w_scales + n * (K / 16), gs_w, 1, K,
                                 what.data());
      for (int64_t m = 0; m < M; ++m) {
        double sum = 0.0, asum = 0.0;
        for (int64_t k = 0; k < K; ++k) {
          const double prod = what[size_t(k)] * xhat[size_t(m * K + k)];
          sum += prod;
          asum += std::fabs(prod);
        }
        y[m * nrows + i] = sum;
        if (absdot) absdot[m * nrows + i] = asum;
      }
    }
  });
  return 0;
}

// FP8 weight tier (reading R15): one fp32 scale per output row,
// s_n = amax(|W[n]|) / 448, and codes E4M3(w / s_n) (RNE, saturating, each
// step one fp32 operation); a row with s_n = 0 gets all-zero codes.
int ora_quantize_fp8_rows(const float* w, int64_t N, int64_t K, uint8_t* codes,
                          float* row_scales, int nthreads) {
  if (N < 0 || K < 0) return -1;
  if (N == 0) return 0;
  if (!w || !row_scales || (K > 0 && !codes)) return -1;
  for (int64_t i = 0; i < N * K; ++i)
    if (!std::isfinite(w[i])) return -2;
  split_range(N, nthreads, [&](int64_t lo, int64_t hi) {
    for (int64_t n = lo; n < hi; ++n) {
      const float* row = w + n * K;
      float amax = 0.0f;
      for (int64_t k = 0; k < K; ++k) amax = std::max(amax, std::fabs(row[k]));
      const float sn = amax / 448.0f;
      row_scales[n] = sn;
      for (int64_t k = 0; k < K; ++k)
        codes[n * K + k] = (sn > 0.0f) ? uint8_t(ora_e4m3_encode(row[k] / sn)) : uint8_t(0);
    }
  });
  return 0;
}

// FP8 weight tier reference linear: w_hat[n][k] = e4m3(code) * s_n, summed
// against the bf16 X in fp64.
int ora_linear_fp8(const uint8_t* codes, const float* row_scales, const uint16_t* x_bf16,
                   int64_t M, int64_t N, int64_t K, const int64_t* rows, int64_t nrows,
                   double* y, double* absdot, int nthreads) {
  if (M < 0 || N < 0 || K < 0 || nrows < 0) return -1;
  if (!rows && nrows != N) return -1;
  if (nrows == 0 || M == 0) return 0;
  if (!y || !row_scales || (K > 0 && (!codes || !x_bf16))) return -1;
  if (rows)
    for (int64_t i = 0; i < nrows; ++i)
      if (rows[i] < 0 || rows[i] >= N) return -1;
  std::vector<double> xv(size_t(M * K));
  for (int64_t i = 0; i < M * K; ++i) xv[size_t(i)] = ora_bf16_value(x_bf16[i]);
  split_range(nrows, nthreads, [&](int64_t lo, int64_t hi) {
    for (int64_t i = lo; i < hi; ++i) {
      const int64_t n = rows ? rows[i] : i;
      const double sn = double(row_scales[n]);
      for (int64_t m = 0; m < M; ++m) {
        double sum = 0.0, asum = 0.0;
        for (int64_t k = 0; k < K; ++k) {
          const double prod = ora_e4m3_decode(codes[n * K + k]) * sn * xv[size_t(m * K + k)];
          sum += prod;
          asum += std::fabs(prod);
        }
        y[m * nrows + i] = sum;
        if (absdot) absdot[m * nrows + i] = asum;
      }
    }
  });
  return 0;
}

double ora_bytes_model(int64_t M, int64_t N, int64_t K) {
  return double(N) * double(K) / 2.0 + double(N) * double(K) / 16.0 +
         2.0 * double(M) * double(K) + 2.0 * double(M) * double(N);
}

}  // extern "C"
