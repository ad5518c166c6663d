// codebook.cpp -- builds the NF4 table on the host, once.
//
// (The uniform INT4 table of the format variants is built here as well.)
//
// NF4 ("从LoRA到QLoRA" §2.3; "QLoRA 原理精讲" §2.1): 16 quantiles of N(0,1)
// taken at probabilities spaced uniformly, normalized to [-1, 1].  The table
// has an exact zero so that zero weights and padding survive a round trip:
// 8 quantiles at p = d + (1/2 - d) i/8 (i = 0..7) for the positive half, 7 at
// p = d + (1/2 - d) i/7 for the negative half (negated), plus 0, where d is
// the mean of the end probabilities 1 - 1/30 and 1 - 1/32 of equal-mass
// splits into 15 and 16 bins; every value is divided by the largest
// magnitude.
//
// The quantile function is inverted with Newton's method on the normal CDF
// (std::erfc), in long double, from a logistic starting guess; the result is
// rounded once to fp32.
#include <cmath>
#include <mutex>
#include "format.h"

namespace nf4 {
namespace {

long double phi_cdf(long double z) { return 0.5L * std::erfc(-z / std::sqrt(2.0L)); }
long double phi_pdf(long double z) {
  const long double inv_sqrt_2pi = 0.398942280401432677939946059934381868L;
  return inv_sqrt_2pi * std::exp(-0.5L * z * z);
}

// z with Phi(z) = p, for p in (0, 1).
long double normal_quantile(long double p) {
  // logistic approximation to start: z0 = log(p/(1-p)) * sqrt(3)/pi
  long double z = std::log(p / (1.0L - p)) * 0.5513288954217920495L;
  for (int it = 0; it < 100; ++it) {
    long double step = (phi_cdf(z) - p) / phi_pdf(z);
    z -= step;
    if (std::fabs(step) < 1e-30L) break;
  }
  return z;
}

void set_thresholds(Codebook& cb) {
  for (int i = 0; i < 15; ++i) {
    // midpoint of two fp32 values is exact in double; round it down to fp32
    double mid = (static_cast<double>(cb.code[i]) + static_cast<double>(cb.code[i + 1])) * 0.5;
    float t = static_cast<float>(mid);
    if (static_cast<double>(t) > mid) t = std::nextafter(t, -INFINITY);
    cb.thr[i] = t;
  }
}

// Uniform INT4 ("QLoRA 原理精讲" §2.1: the 16 integers -8..7, evenly spaced),
// divided by 8 so that the table lies in [-1, 1]: code i = (i - 8) / 8.
Codebook build_int4() {
  Codebook cb{};
  for (int i = 0; i < 16; ++i) cb.code[i] = static_cast<float>(i - 8) / 8.0f;
  set_thresholds(cb);
  return cb;
}

Codebook build() {
  Codebook cb{};
  const long double d = 0.5L * ((1.0L - 1.0L / 30.0L) + (1.0L - 1.0L / 32.0L));
  long double pos[8], neg[7];
  for (int i = 0; i < 8; ++i) pos[i] = normal_quantile(d + (0.5L - d) * i / 8.0L);   // descending
  for (int i = 0; i < 7; ++i) neg[i] = -normal_quantile(d + (0.5L - d) * i / 7.0L);  // ascending
  const long double scale = pos[0] > -neg[0] ? pos[0] : -neg[0];
  // ascending order: neg[0] (= -1) ... neg[6], 0, pos[7] ... pos[0] (= 1)
  for (int i = 0; i < 7; ++i) cb.code[i] = static_cast<float>(neg[i] / scale);
  cb.code[7] = 0.0f;
  for (int i = 0; i < 8; ++i) cb.code[8 + i] = static_cast<float>(pos[7 - i] / scale);
  set_thresholds(cb);
  return cb;
}

}  // namespace

const Codebook& host_codebook() {
  static Codebook cb;
  static std::once_flag once;
  std::call_once(once, [] { cb = build(); });
  return cb;
}

const Codebook& host_codebook(int quant_type) {
  if (quant_type != kQuantInt4) return host_codebook();
  static Codebook cb;
  static std::once_flag once;
  std::call_once(once, [] { cb = build_int4(); });
  return cb;
}

}  // namespace nf4
