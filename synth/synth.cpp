// synth.cpp -- seeded synthetic inputs for the NVFP4 linear (host only).
//
// This module is shared by the tests, the oracle's callers and the benchmark.
// It holds none of the linear's arithmetic: no quantisation, no decode, no
// dot products. It only draws numbers.
//
// Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
// number generators", OOPSLA 2014; constants as published by Vigna) used as a
// counter-based generator: draw i of stream (seed, id) is mix(key + (i+1)*gamma)
// with key = mix(mix(seed) ^ (id * 0xD1B54A32D192ED03)). Uniforms in (0, 1) use
// the top 53 bits; normals use the Box-Muller transform on draws (2p, 2p+1):
// element 2p is r*cos(2*pi*u2), element 2p+1 is r*sin(2*pi*u2).
//
// Build: g++ -O2 -std=c++17 -shared -fPIC -pthread

#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>
#include <algorithm>

namespace {

const uint64_t kGamma = 0x9E3779B97F4A7C15ull;

inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

inline uint64_t stream_key(uint64_t seed, uint64_t id) {
  return mix64(mix64(seed) ^ (id * 0xD1B54A32D192ED03ull));
}

inline uint64_t draw(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * kGamma); }

inline double uniform(uint64_t key, uint64_t i) {
  return (double(draw(key, i) >> 11) + 0.5) * 0x1.0p-53;
}

inline double normal(uint64_t key, uint64_t i) {
  uint64_t p = i >> 1;
  double u1 = uniform(key, 2 * p), u2 = uniform(key, 2 * p + 1);
  double r = std::sqrt(-2.0 * std::log(u1));
  const double two_pi = 6.283185307179586476925286766559;
  return (i & 1) ? r * std::sin(two_pi * u2) : r * std::cos(two_pi * u2);
}

// bf16 bit pattern of a float, round to nearest even (inputs are finite here).
inline uint16_t to_bf16(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return uint16_t(u >> 16);
}

template <class F>
void par_for(int64_t n, int nthreads, F body) {
  if (nthreads < 1) nthreads = 1;
  if (n < 65536 || nthreads == 1) { body(int64_t(0), n); return; }
  int64_t per = (n + nthreads - 1) / nthreads;
  std::vector<std::thread> ts;
  for (int t = 0; t < nthreads; ++t) {
    int64_t lo = t * per, hi = std::min(n, lo + per);
    if (lo >= hi) break;
    ts.emplace_back([=] { body(lo, hi); });
  }
  for (auto& th : ts) th.join();
}

}  // namespace

extern "C" {

uint64_t synth_draw(uint64_t seed, uint64_t id, uint64_t i) { return draw(stream_key(seed, id), i); }
double synth_uniform(uint64_t seed, uint64_t id, uint64_t i) { return uniform(stream_key(seed, id), i); }
double synth_normal(uint64_t seed, uint64_t id, uint64_t i) { return normal(stream_key(seed, id), i); }

// out[i] = float(sigma * z(start + i)), z the normal stream (seed, id).
void synth_normal_f32(uint64_t seed, uint64_t id, uint64_t start, int64_t n,
                      double sigma, float* out, int nthreads) {
  uint64_t key = stream_key(seed, id);
  par_for(n, nthreads, [&](int64_t lo, int64_t hi) {
    for (int64_t i = lo; i < hi; ++i) out[i] = float(sigma * normal(key, start + uint64_t(i)));
  });
}

// `count` distinct indices in [0, K) drawn by a partial Fisher-Yates shuffle on
// the uniform stream (seed, id); written to idx[0..count).
int synth_distinct_indices(uint64_t seed, uint64_t id, int64_t K, int64_t count, int64_t* idx) {
  if (count > K || count < 0) return -1;
  uint64_t key = stream_key(seed, id);
  std::vector<int64_t> perm(static_cast<size_t>(K));
  for (int64_t i = 0; i < K; ++i) perm[size_t(i)] = i;
  for (int64_t i = 0; i < count; ++i) {
    int64_t j = i + int64_t(uniform(key, uint64_t(i)) * double(K - i));
    if (j >= K) j = K - 1;
    std::swap(perm[size_t(i)], perm[size_t(j)]);
    idx[i] = perm[size_t(i)];
  }
  return 0;
}

// Activation rows X[M][K] as bf16 bit patterns.
//   kind 0: N(0,1)                                  (stream 1)
//   kind 1: N(0,1), with `n_outliers` distinct channels (same for every row,
//           stream 2) multiplied by `outlier_gain` before rounding
//   kind 2: SiLU(a) * b, a, b ~ N(0,1)              (streams 3, 4)
//   kind 3: z / sqrt(mean(z^2) + 1e-6) per row, z ~ N(0,1)   (stream 1)
int synth_x_bf16(int kind, uint64_t seed, int64_t M, int64_t K, int64_t n_outliers,
                 double outlier_gain, uint16_t* out) {
  if (M < 0 || K < 0) return -1;
  uint64_t k1 = stream_key(seed, 1), k3 = stream_key(seed, 3), k4 = stream_key(seed, 4);
  std::vector<double> row(static_cast<size_t>(K));
  std::vector<int64_t> outl;
  if (kind == 1) {
    if (n_outliers > K) return -1;
    outl.resize(size_t(n_outliers));
    if (n_outliers > 0) synth_distinct_indices(seed, 2, K, n_outliers, outl.data());
  }
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t k = 0; k < K; ++k) {
      uint64_t i = uint64_t(m * K + k);
      double v;
      if (kind == 2) {
        double a = normal(k3, i), b = normal(k4, i);
        v = a / (1.0 + std::exp(-a)) * b;
      } else {
        v = normal(k1, i);
      }
      row[size_t(k)] = v;
    }
    if (kind == 1)
      for (int64_t c : outl) row[size_t(c)] *= outlier_gain;
    if (kind == 3) {
      double ss = 0.0;
      for (int64_t k = 0; k < K; ++k) ss += row[size_t(k)] * row[size_t(k)];
      double inv = 1.0 / std::sqrt(ss / double(K > 0 ? K : 1) + 1e-6);
      for (int64_t k = 0; k < K; ++k) row[size_t(k)] *= inv;
    }
    if (kind < 0 || kind > 3) return -1;
    for (int64_t k = 0; k < K; ++k) out[m * K + k] = to_bf16(float(row[size_t(k)]));
  }
  return 0;
}

}  // extern "C"
