// codebook.cpp -- host construction of the NF4 levels and thresholds.
//
// NF4 ("QLoRA", llm-compass, 方法与公式 item 1; learn-interview-questions QLoRA
// page, section 2): 16 levels at standard-normal quantiles with equal
// expected mass per bin, normalised to [-1, 1].  An exact zero is kept by
// splitting the code 8 positive / 7 negative: with
// delta = 1 - (1/32 + 1/30)/2, the positive levels are Phi^-1 at
// delta - i (delta - 1/2)/8 (i = 0..7), the negative ones minus Phi^-1 at
// delta - i (delta - 1/2)/7 (i = 0..6), all divided by Phi^-1(delta).
//
// Phi^-1 is computed in long double: bisection on Phi(x) = erfc(-x/sqrt 2)/2
// to bracket the root, then Newton steps with the normal density.  The fp32
// rounding of every level is insensitive to errors far below 1e-12.
#include <cmath>
#include <cstdint>
#include <cstring>

namespace qnf4_host {

static long double phi_cdf(long double x) {
  return 0.5L * std::erfc(-x / std::sqrt(2.0L));
}

static long double phi_pdf(long double x) {
  return std::exp(-0.5L * x * x) / std::sqrt(2.0L * 3.14159265358979323846264338327950288L);
}

long double inverse_normal_cdf(long double p) {
  long double lo = -12.0L, hi = 12.0L;
  for (int i = 0; i < 80; ++i) {          // bracket to ~1e-23 relative width
    const long double mid = 0.5L * (lo + hi);
    if (phi_cdf(mid) < p) lo = mid; else hi = mid;
  }
  long double x = 0.5L * (lo + hi);
  for (int i = 0; i < 3; ++i) x -= (phi_cdf(x) - p) / phi_pdf(x);
  return x;
}

// levels[16] ascending, thresholds[15]: exact midpoints of consecutive fp32
// levels rounded toward -infinity to fp32.
void build_codebook(float levels[16], float thresholds[15]) {
  const long double delta = 1.0L - 0.5L * (1.0L / 32.0L + 1.0L / 30.0L);
  const long double norm = inverse_normal_cdf(delta);
  long double v[16];
  int n = 0;
  for (int i = 0; i <= 6; ++i)            // negative side, ascending
    v[n++] = -inverse_normal_cdf(delta - i * (delta - 0.5L) / 7.0L) / norm;
  v[n++] = 0.0L;
  for (int i = 7; i >= 0; --i)            // positive side, ascending
    v[n++] = inverse_normal_cdf(delta - i * (delta - 0.5L) / 8.0L) / norm;
  for (int j = 0; j < 16; ++j) levels[j] = static_cast<float>(v[j]);
  levels[0] = -1.0f;                       // -Phi^-1(delta)/Phi^-1(delta)
  levels[7] = 0.0f;
  levels[15] = 1.0f;
  if (thresholds != nullptr) {
    for (int j = 0; j < 15; ++j) {
      const double mid = 0.5 * (static_cast<double>(levels[j]) + static_cast<double>(levels[j + 1]));
      float t = static_cast<float>(mid);
      if (static_cast<double>(t) > mid) t = std::nextafter(t, -INFINITY);
      thresholds[j] = t;
    }
  }
}

// Uniform INT4 comparison code: levels fp32(k/7) for k = -7..7 at codes
// 0..14 (zero at code 7), code 15 a second +1; thresholds as above.
void build_int4_codebook(float levels[16], float thresholds[15]) {
  for (int k = 0; k < 15; ++k) levels[k] = static_cast<float>((k - 7) / 7.0);
  levels[15] = 1.0f;
  if (thresholds != nullptr) {
    for (int j = 0; j < 15; ++j) {
      const double mid = 0.5 * (static_cast<double>(levels[j]) + static_cast<double>(levels[j + 1]));
      float t = static_cast<float>(mid);
      if (static_cast<double>(t) > mid) t = std::nextafter(t, -INFINITY);
      thresholds[j] = t;
    }
  }
}

}  // namespace qnf4_host
