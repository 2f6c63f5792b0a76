// nf4_tables.cpp -- the CUDA library's own NF4 codebook and encode tables.
//
// Codebook (QLoRA, arXiv:2305.14314, as summarised by automatone "QLoRA paper
// explained", paragraph "4-bit NormalFloat (NF4)": levels at the quantiles of
// a standard normal; creativeworksofknowledge "QLoRA: Fine-Tune 70B on One
// GPU", section "1. NF4": Gaussian-proportional levels, denser near zero).
// The comparison types of automatone, "4-bit NormalFloat (NF4)" (evenly spaced
// 4-bit integers, exponent-spaced 4-bit floats) get tables of their own: INT4
// levels (2i - 15) / 15, and FP4 the E2M1 values divided by 6 (15 distinct
// values; the last code repeats +1).
//
// NF4 construction: 8 positive levels at Phi^-1(1/2 + (delta - 1/2) j / 8),
// j = 1..8, 7 negative levels at -Phi^-1(1/2 + (delta - 1/2) j / 7), j = 1..7,
// and an exact zero, all divided by Phi^-1(delta), with
// delta = 1 - (1/30 + 1/32) / 2; evaluated in double and rounded once to float.
//
// The inverse normal CDF here is Newton's method on Phi(x) = erfc(-x/sqrt 2)/2
// with the normal density as derivative -- computed independently of any other
// implementation, so that comparing tables across implementations is a check.
#include "nf4_tables.h"

#include <cmath>
#include <cstring>
#include <limits>
#include <mutex>

namespace qlora {
namespace {

double inv_normal_cdf(double p) {
  // Newton from 0; Phi is convex for x > 0 and concave for x < 0, so iterates
  // approach the root monotonically after the first step.
  double x = 0.0;
  const double inv_sqrt2pi = 0.39894228040143267794;
  for (int it = 0; it < 100; ++it) {
    const double f = 0.5 * std::erfc(-x / std::sqrt(2.0)) - p;
    const double d = inv_sqrt2pi * std::exp(-0.5 * x * x);
    const double step = f / d;
    x -= step;
    if (std::fabs(step) <= 1e-17 * std::fmax(1.0, std::fabs(x))) break;
  }
  return x;
}

// Smallest float strictly greater than the exact midpoint of a and b.
float above_midpoint(float a, float b) {
  const double mid = 0.5 * (static_cast<double>(a) + static_cast<double>(b));  // exact
  float f = static_cast<float>(mid);
  if (static_cast<double>(f) <= mid) f = std::nextafter(f, std::numeric_limits<float>::infinity());
  return f;
}

// The bucket the encode kernel assigns to n: RN(16 n + 16), computed with one
// fused multiply-add against 2^23 so that the integer lands in the low bits.
int bucket_of(float n) {
  const float v = std::fmaf(n, 16.0f, 16.0f + 8388608.0f);
  uint32_t u;
  std::memcpy(&u, &v, 4);
  return static_cast<int>(u & 63u);
}

uint32_t ordered_key(float f) {  // monotone map of floats in [-1, 1] to integers
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
float from_key(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// The 16 levels of each 4-bit type, ascending, in [-1, 1].
void make_levels(int type, float (&level)[16]) {
  if (type == kTypeNf4) {
    const double delta = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0);
    const double top = inv_normal_cdf(delta);
    for (int j = 1; j <= 7; ++j)
      level[7 - j] = static_cast<float>(-inv_normal_cdf(0.5 + (delta - 0.5) * j / 7.0) / top);
    level[7] = 0.0f;
    for (int j = 1; j <= 8; ++j)
      level[7 + j] = static_cast<float>(inv_normal_cdf(0.5 + (delta - 0.5) * j / 8.0) / top);
  } else if (type == kTypeInt4) {
    // 16 evenly spaced integers -15, -13, ..., 15 over the half-range 15
    for (int i = 0; i < 16; ++i) level[i] = static_cast<float>(static_cast<double>(2 * i - 15) / 15.0);
  } else {
    // E2M1: magnitudes m * 2^-1 (exponent field 0) and (1 + m/2) * 2^(e - 1);
    // the 8 non-negative ones ascending are the table's upper half from index 7
    double mag[8];
    int k = 0;
    for (int e = 0; e < 4; ++e)
      for (int m = 0; m < 2; ++m) mag[k++] = e == 0 ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, e - 1);
    const double top = mag[7];
    for (int i = 0; i < 8; ++i) level[7 + i] = static_cast<float>(mag[i] / top);
    for (int i = 1; i < 8; ++i) level[7 - i] = static_cast<float>(-mag[i] / top);   // -0 is the same level as +0
    level[15] = level[14];    // 15 distinct values: the last code repeats +1 and is never chosen
  }
}

Nf4Tables build(int type) {
  Nf4Tables t{};
  make_levels(type, t.level);

  // Nearest level with ties to the lower index <=> count of thresholds <= n,
  // where threshold i is the first float past the midpoint of levels i, i+1.
  for (int i = 0; i < 15; ++i) t.threshold[i] = above_midpoint(t.level[i], t.level[i + 1]);

  // For each bucket find the float interval [lo, hi] of n in [-1, 1] that the
  // kernel's bucket formula maps to it (monotone, so bisect on float order).
  t.ok = true;
  t.fast_ok = true;
  const uint32_t kmin = ordered_key(-1.0f), kmax = ordered_key(1.0f);
  for (int u = 0; u < kNumBuckets; ++u) {
    uint32_t lo = kmin, hi = kmax;  // first key with bucket >= u
    while (lo < hi) {
      uint32_t mid = lo + (hi - lo) / 2;
      if (bucket_of(from_key(mid)) >= u) hi = mid; else lo = mid + 1;
    }
    const uint32_t first = lo;
    lo = kmin; hi = kmax;           // first key with bucket >= u + 1
    if (bucket_of(from_key(kmax)) <= u) {
      lo = kmax + 1;
    } else {
      while (lo < hi) {
        uint32_t mid = lo + (hi - lo) / 2;
        if (bucket_of(from_key(mid)) >= u + 1) hi = mid; else lo = mid + 1;
      }
    }
    const uint32_t last = lo - 1;
    if (first > last) { t.bucket_base[u] = 15; t.bucket_thr[u] = INFINITY; continue; }
    const float nlo = from_key(first), nhi = from_key(last);
    int base = 0, inside = 0;
    float thr = INFINITY;
    for (int i = 0; i < 15; ++i) {
      if (t.threshold[i] <= nlo) ++base;
      else if (t.threshold[i] <= nhi) { ++inside; thr = t.threshold[i]; }
    }
    if (inside > 1) t.ok = false;
    // The encoder's reciprocal path only re-checks the threshold of the bucket
    // its estimate falls in; that is exact when no threshold is within 2^-18
    // of a bucket edge (the estimate is within 2^-22 of the IEEE quotient, and
    // the fast-path threshold within 2^-19 of the true one).
    if (inside == 1 && (static_cast<double>(thr) - nlo <= 0x1.0p-18 || nhi - static_cast<double>(thr) <= 0x1.0p-18))
      t.fast_ok = false;
    t.bucket_base[u] = static_cast<uint8_t>(base);
    t.bucket_thr[u] = thr;
    uint32_t tb = 0x7F7FFFE0u;                 // about 3.4e38: no threshold in this bucket
    if (inside == 1) std::memcpy(&tb, &thr, 4);
    t.bucket_fast[u] = (tb & ~31u) | static_cast<uint32_t>(base + 1);
  }
  return t;
}

}  // namespace

const Nf4Tables& level_tables(int type) {
  static Nf4Tables tables[kNumTypes];
  static std::once_flag once;
  std::call_once(once, [] {
    for (int i = 0; i < kNumTypes; ++i) tables[i] = build(i);
  });
  return tables[(type >= 0 && type < kNumTypes) ? type : kTypeNf4];
}

const Nf4Tables& nf4_tables() { return level_tables(kTypeNf4); }

}  // namespace qlora
