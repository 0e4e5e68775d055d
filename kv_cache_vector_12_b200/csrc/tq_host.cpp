// Host-side construction of the method's fixed parameters: the rotation Pi,
// the QJL projection S and the Lloyd-Max codebooks.
//
// Rotation: the first step of the method multiplies every vector by a random
// orthogonal matrix (ai-accelerate.xyz TurboQuant explainer, section
// "ステップ1: PolarQuant").  Pi is the Q factor of a seeded Gaussian matrix,
// made unique by a positive diagonal of R, then rounded to bf16: the bf16
// matrix is the one both quantize and decode use.
//
// Codebook: the same section quantizes each coordinate on its own with the
// optimal (Lloyd-Max) scalar quantizer.  Lloyd's iteration on N(0,1), scaled
// by 1/sqrt(d) for the N(0,1/d) law of a rotated unit vector's coordinates
// (or, as a variant, on the exact law of one coordinate of a unit vector),
// held in fp16 (the pages fix no precision; fp16 costs < 1e-5 of the
// distortion and makes every centroid an exact tensor-core operand).
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "tq_internal.h"

namespace tq {

// SplitMix64 (Steele, Lea & Flood 2014) read as a counter-based generator:
// output n (n >= 1) of the generator seeded with `seed` is the variant-13
// finaliser applied to seed + n * 0x9E3779B97F4A7C15.
static inline uint64_t splitmix64_at(uint64_t seed, uint64_t n) {
  uint64_t z = seed + n * 0x9E3779B97F4A7C15ULL;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

// `count` standard normals of stream `stream` (Pi: 0, S: 1).  Box-Muller on
// 53-bit uniforms: pair p uses counters base+2p+1 (u1 in (0,1]) and
// base+2p+2 (u2 in [0,1)); element e is component e%2 of pair e/2.
void gaussian_stream(uint64_t seed, uint32_t stream, size_t count, double *out) {
  const uint64_t base = (uint64_t)stream << 32;
  const double inv53 = 1.0 / 9007199254740992.0;
  const double two_pi = 2.0 * M_PI;
  for (size_t p = 0; 2 * p < count; ++p) {
    const uint64_t a = splitmix64_at(seed, base + 2 * p + 1);
    const uint64_t b = splitmix64_at(seed, base + 2 * p + 2);
    const double u1 = (double)((a >> 11) + 1) * inv53;
    const double u2 = (double)(b >> 11) * inv53;
    const double r = std::sqrt(-2.0 * std::log(u1));
    const double theta = two_pi * u2;
    out[2 * p] = r * std::cos(theta);
    if (2 * p + 1 < count) out[2 * p + 1] = r * std::sin(theta);
  }
}

// Round a double to the nearest bfloat16 (ties to even) by clearing the 45
// low mantissa bits of the double with carry; returns the bf16 bit pattern.
// IEEE half bits of a double, rounded to nearest even, subnormals included;
// magnitudes from 65520 up become infinity.
uint16_t double_to_half_bits(double x) {
  const uint16_t sign = std::signbit(x) ? 0x8000u : 0u;
  const double a = std::fabs(x);
  if (!(a < 65520.0)) return (uint16_t)(sign | 0x7C00u);
  if (a < 0x1p-14) return (uint16_t)(sign | (uint16_t)std::nearbyint(a * 0x1p24));  // 1024 is the smallest normal
  int e;
  const double f = std::frexp(a, &e);         // a = f 2^e, f in [0.5, 1)
  double m = std::nearbyint(f * 2048.0);      // 11 significant bits, 1024 .. 2048
  if (m == 2048.0) {
    m = 1024.0;
    ++e;
  }
  const int biased = e - 1 + 15;
  if (biased >= 31) return (uint16_t)(sign | 0x7C00u);
  return (uint16_t)(sign | (biased << 10) | ((int)m - 1024));
}

double half_bits_to_double(uint16_t h) {
  const int e = (h >> 10) & 0x1F, m = h & 0x3FF;
  const double v = e == 0 ? std::ldexp((double)m, -24) : std::ldexp((double)(m + 1024), e - 25);
  return (h & 0x8000u) ? -v : v;
}

uint16_t double_to_bf16_bits(double x) {
  uint64_t u;
  std::memcpy(&u, &x, 8);
  const uint64_t drop = 45;
  const uint64_t lsb = (u >> drop) & 1u;
  u += ((uint64_t)1 << (drop - 1)) - 1 + lsb;
  u &= ~(((uint64_t)1 << drop) - 1);
  double r;
  std::memcpy(&r, &u, 8);
  const float f = (float)r;  // exact: 8 significant bits in fp32's range
  uint32_t fb;
  std::memcpy(&fb, &f, 4);
  return (uint16_t)(fb >> 16);
}

float bf16_bits_to_float(uint16_t h) {
  const uint32_t fb = (uint32_t)h << 16;
  float f;
  std::memcpy(&f, &fb, 4);
  return f;
}

// Householder QR of the n x n row-major matrix a (overwritten).  Returns Q
// (row-major) with every column multiplied by the sign of R's diagonal entry,
// i.e. the unique Q whose R has a positive diagonal.
static std::vector<double> signed_householder_q(std::vector<double> a, int n) {
  std::vector<std::vector<double>> vs(n);
  std::vector<double> rdiag(n);
  for (int k = 0; k < n; ++k) {
    double norm2 = 0.0;
    for (int i = k; i < n; ++i) norm2 += a[(size_t)i * n + k] * a[(size_t)i * n + k];
    const double norm = std::sqrt(norm2);
    const double x0 = a[(size_t)k * n + k];
    const double alpha = x0 >= 0.0 ? -norm : norm;  // R_kk
    std::vector<double> v(n - k);
    for (int i = k; i < n; ++i) v[i - k] = a[(size_t)i * n + k];
    v[0] -= alpha;
    double vn2 = 0.0;
    for (double e : v) vn2 += e * e;
    if (vn2 > 0.0) {
      const double inv = 1.0 / std::sqrt(vn2);
      for (double &e : v) e *= inv;
      for (int j = k; j < n; ++j) {  // A[k:, k:] -= 2 v (v^T A[k:, k:])
        double dot = 0.0;
        for (int i = k; i < n; ++i) dot += v[i - k] * a[(size_t)i * n + j];
        for (int i = k; i < n; ++i) a[(size_t)i * n + j] -= 2.0 * v[i - k] * dot;
      }
    }
    rdiag[k] = vn2 > 0.0 ? alpha : x0;
    vs[k] = std::move(v);
  }
  // Q = H_0 H_1 ... H_{n-1}: apply the reflections to I from the last one.
  std::vector<double> q((size_t)n * n, 0.0);
  for (int i = 0; i < n; ++i) q[(size_t)i * n + i] = 1.0;
  for (int k = n - 1; k >= 0; --k) {
    const std::vector<double> &v = vs[k];
    double vn2 = 0.0;
    for (double e : v) vn2 += e * e;
    if (vn2 == 0.0) continue;
    for (int j = 0; j < n; ++j) {
      double dot = 0.0;
      for (int i = k; i < n; ++i) dot += v[i - k] * q[(size_t)i * n + j];
      for (int i = k; i < n; ++i) q[(size_t)i * n + j] -= 2.0 * v[i - k] * dot;
    }
  }
  for (int j = 0; j < n; ++j)
    if (rdiag[j] < 0.0)
      for (int i = 0; i < n; ++i) q[(size_t)i * n + j] = -q[(size_t)i * n + j];
  return q;
}

void rotation_bf16(int d, uint64_t seed, uint16_t *pi_bits) {
  std::vector<double> g((size_t)d * d);
  gaussian_stream(seed, 0, g.size(), g.data());
  const std::vector<double> q = signed_householder_q(std::move(g), d);
  for (size_t i = 0; i < q.size(); ++i) pi_bits[i] = double_to_bf16_bits(q[i]);
}

void qjl_matrix(int d, uint64_t seed, float *s) {
  std::vector<double> g((size_t)d * d);
  gaussian_stream(seed, 1, g.size(), g.data());
  for (size_t i = 0; i < g.size(); ++i) s[i] = (float)g[i];
}

// Standard normal density and the probability of (a, b], computed on the
// side of zero that avoids cancellation.
static double npdf(double x) {
  return std::isinf(x) ? 0.0 : std::exp(-0.5 * x * x) * 0.3989422804014327;
}
static double nmass(double a, double b) {
  if (a >= 0.0) return 0.5 * std::erfc(a * M_SQRT1_2) - 0.5 * std::erfc(b * M_SQRT1_2);
  return 0.5 * std::erfc(-b * M_SQRT1_2) - 0.5 * std::erfc(-a * M_SQRT1_2);
}

// Lloyd-Max centroids of N(0,1) with 2^bits levels, ascending.  Starts from
// evenly spaced centroids on [-2, 2] and alternates the two optimality
// conditions (thresholds at midpoints, centroids at conditional means) until
// no centroid moves by more than 1e-15; then symmetrises exactly.
void lloyd_max_gaussian(int bits, double *c) {
  const int L = 1 << bits;
  for (int j = 0; j < L; ++j) c[j] = -2.0 + 4.0 * (j + 0.5) / L;
  std::vector<double> t(L + 1), nc(L);
  for (int it = 0; it < 2000000; ++it) {
    t[0] = -INFINITY;
    t[L] = INFINITY;
    for (int j = 1; j < L; ++j) t[j] = 0.5 * (c[j - 1] + c[j]);
    double move = 0.0;
    for (int j = 0; j < L; ++j) {
      nc[j] = (npdf(t[j]) - npdf(t[j + 1])) / nmass(t[j], t[j + 1]);
      move = std::fmax(move, std::fabs(nc[j] - c[j]));
    }
    for (int j = 0; j < L; ++j) c[j] = nc[j];
    if (move <= 1e-15) break;
  }
  for (int j = 0; j < L / 2; ++j) {
    const double m = 0.5 * (c[L - 1 - j] - c[j]);
    c[j] = -m;
    c[L - 1 - j] = m;
  }
}

// Round a double in half's normal range to the nearest IEEE half (ties to
// even): keep 10 of the double's 52 mantissa bits, carrying into the exponent.
double round_to_half(double x) {
  uint64_t u;
  std::memcpy(&u, &x, 8);
  const uint64_t drop = 42;
  const uint64_t lsb = (u >> drop) & 1u;
  u += ((uint64_t)1 << (drop - 1)) - 1 + lsb;
  u &= ~(((uint64_t)1 << drop) - 1);
  double r;
  std::memcpy(&r, &u, 8);
  return r;
}

// Regularised incomplete beta function I_x(a, b), from its continued
// fraction (DLMF 8.17.22) evaluated by the modified Lentz method, on the side
// of (a + 1) / (a + b + 2) where the fraction converges fast
// (I_x(a, b) = 1 - I_{1-x}(b, a) on the other side).
static double incomplete_beta(double a, double b, double x) {
  if (x <= 0.0) return 0.0;
  if (x >= 1.0) return 1.0;
  if (x > (a + 1.0) / (a + b + 2.0)) return 1.0 - incomplete_beta(b, a, 1.0 - x);
  const double tiny = 1e-300;
  const double log_front = a * std::log(x) + b * std::log1p(-x) -
                           (std::lgamma(a) + std::lgamma(b) - std::lgamma(a + b));
  // 1 / (1 + e1 / (1 + e2 / (1 + ...))) with
  //   e_{2m+1} = -(a + m)(a + b + m) x / ((a + 2m)(a + 2m + 1)),
  //   e_{2m}   =  m (b - m) x / ((a + 2m - 1)(a + 2m)).
  double num = -(a + b) * x / (a + 1.0);  // e_1
  double dd = 1.0 + num;
  if (std::fabs(dd) < tiny) dd = tiny;
  dd = 1.0 / dd;
  double cc = 1.0, f = dd;
  for (int m = 1; m < 10000; ++m) {
    for (int odd = 0; odd < 2; ++odd) {
      num = odd ? -(a + m) * (a + b + m) * x / ((a + 2.0 * m) * (a + 2.0 * m + 1.0))
                : m * (b - m) * x / ((a + 2.0 * m - 1.0) * (a + 2.0 * m));
      dd = 1.0 + num * dd;
      if (std::fabs(dd) < tiny) dd = tiny;
      cc = 1.0 + num / cc;
      if (std::fabs(cc) < tiny) cc = tiny;
      dd = 1.0 / dd;
      f *= dd * cc;
      if (odd && std::fabs(dd * cc - 1.0) < 1e-16) return std::exp(log_front) * f / a;
    }
  }
  return std::exp(log_front) * f / a;
}

// The coordinate X of a uniform unit vector in R^d has the density
// (1 - x^2)^((d-3)/2) / B(1/2, (d-1)/2) on (-1, 1): (X + 1) / 2 is
// Beta(h, h) with h = (d - 1) / 2.  Mass of (lo, hi], on the side of zero
// that avoids cancellation.
static double sphere_mass(double lo, double hi, int d) {
  const double h = 0.5 * (d - 1);
  if (lo >= 0.0) return incomplete_beta(h, h, 0.5 * (1.0 - lo)) - incomplete_beta(h, h, 0.5 * (1.0 - hi));
  return incomplete_beta(h, h, 0.5 * (1.0 + hi)) - incomplete_beta(h, h, 0.5 * (1.0 + lo));
}

// int_lo^hi x f(x) dx = ((1 - lo^2)^h - (1 - hi^2)^h) / (2 h B(1/2, h)).
static double sphere_first_moment(double lo, double hi, int d) {
  const double h = 0.5 * (d - 1);
  const double beta_half_h = std::exp(std::lgamma(0.5) + std::lgamma(h) - std::lgamma(h + 0.5));
  return (std::pow(1.0 - lo * lo, h) - std::pow(1.0 - hi * hi, h)) / (2.0 * h * beta_half_h);
}

// Lloyd-Max centroids of that law with 2^bits levels, ascending.  Starts from
// the N(0, 1/d) centroids (its large-d limit) and alternates the two
// optimality conditions until no centroid moves by more than 1e-15; then
// symmetrises exactly.
void lloyd_max_sphere(int bits, int d, double *c) {
  const int L = 1 << bits;
  lloyd_max_gaussian(bits, c);
  const double inv_sqrt_d = 1.0 / std::sqrt((double)d);
  for (int j = 0; j < L; ++j) c[j] = std::fmax(-0.999, std::fmin(0.999, c[j] * inv_sqrt_d));
  std::vector<double> t(L + 1), nc(L);
  for (int it = 0; it < 2000000; ++it) {
    t[0] = -1.0;
    t[L] = 1.0;
    for (int j = 1; j < L; ++j) t[j] = 0.5 * (c[j - 1] + c[j]);
    double move = 0.0;
    for (int j = 0; j < L; ++j) {
      nc[j] = sphere_first_moment(t[j], t[j + 1], d) / sphere_mass(t[j], t[j + 1], d);
      move = std::fmax(move, std::fabs(nc[j] - c[j]));
    }
    for (int j = 0; j < L; ++j) c[j] = nc[j];
    if (move <= 1e-15) break;
  }
  for (int j = 0; j < L / 2; ++j) {
    const double m = 0.5 * (c[L - 1 - j] - c[j]);
    c[j] = -m;
    c[L - 1 - j] = m;
  }
}

// Codebook of `bits` bits, rounded to fp16 (exact as fp32), thresholds at the
// exact midpoints.  TQ_LAW_GAUSSIAN: Lloyd-Max centroids of N(0,1) / sqrt(d),
// for the N(0, 1/d) law; TQ_LAW_SPHERE: Lloyd-Max centroids of the exact
// coordinate law of a unit vector in R^d.
void codebook(int bits, int d, int law, float *centroids, float *thresholds) {
  const int L = 1 << bits;
  std::vector<double> c(L);
  if (law == TQ_LAW_SPHERE) {
    lloyd_max_sphere(bits, d, c.data());
  } else {
    lloyd_max_gaussian(bits, c.data());
    const double inv_sqrt_d = 1.0 / std::sqrt((double)d);
    for (int j = 0; j < L; ++j) c[j] *= inv_sqrt_d;
  }
  for (int j = 0; j < L; ++j) centroids[j] = (float)round_to_half(c[j]);
  for (int j = 0; j + 1 < L; ++j)
    thresholds[j] = (float)(0.5 * ((double)centroids[j] + (double)centroids[j + 1]));
}

// The quantize kernel finds m = #{j : t_j < |y|} over the positive thresholds
// by binary search, selecting each level's threshold (scaled by -2^64) with
// fp32 fused multiply-adds from differences of the scaled thresholds.  That
// is exact only if every difference and every selection is exact in fp32;
// this replays the kernel's arithmetic for every path of the search.
bool threshold_search_exact(int bits, const float *thresholds) {
  const int half = 1 << (bits - 1);
  float nt[kMaxLevels / 2];
  for (int j = 0; j < half - 1; ++j) nt[j] = -thresholds[half + j] * 0x1p64f;
  if (bits == 2) return true;
  if (bits == 3) {
    const float d20 = nt[2] - nt[0];
    return std::fma(0.f, d20, nt[0]) == nt[0] && std::fma(1.f, d20, nt[0]) == nt[2];
  }
  if (bits != 4) return false;
  const float d51 = nt[5] - nt[1], d40 = nt[4] - nt[0], d20 = nt[2] - nt[0];
  const float ddd = (nt[6] - nt[4]) - d20;
  for (int b2 = 0; b2 < 2; ++b2) {
    if (std::fma((float)b2, d51, nt[1]) != nt[b2 ? 5 : 1]) return false;
    const float base = std::fma((float)b2, d40, nt[0]);
    const float step = std::fma((float)b2, ddd, d20);
    for (int b1 = 0; b1 < 2; ++b1)
      if (std::fma((float)b1, step, base) != nt[4 * b2 + 2 * b1]) return false;
  }
  return true;
}

}  // namespace tq
