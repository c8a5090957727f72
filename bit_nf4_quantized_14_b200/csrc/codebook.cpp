// Host construction of the NF4 codebook (PEFT page, zerotofrontier.app/sft/peft,
// "NF4, derived from normal quantiles"): normal quantiles of evenly spaced probabilities from 0.9677
// down to 0.5 -- 8 on the positive side, 7 on the negative side, the 0.5 end dropped on both -- plus an
// exact 0, divided by z* = Phi^-1(0.9677) so the ends are exactly -1 and +1.
//
// Phi^-1 here: the Abramowitz & Stegun 26.2.23 rational approximation (|error| < 4.5e-4) as a start,
// refined by Newton steps on Phi(x) - p in long double with the C library's erfcl, until the step no
// longer changes x. Levels are rounded once to fp32; thresholds are the exact midpoints of adjacent fp32
// levels rounded once to fp32.
#include <cmath>
#include <mutex>

namespace qnf4 {

static long double normal_cdf_l(long double x) { return 0.5L * std::erfc(-x / std::sqrt(2.0L)); }

static long double normal_ppf_l(long double p) {   // 0.5 < p < 1
  const long double q = 1.0L - p;
  const long double t = std::sqrt(-2.0L * std::log(q));
  long double x = t - (2.515517L + 0.802853L * t + 0.010328L * t * t) /
                          (1.0L + 1.432788L * t + 0.189269L * t * t + 0.001308L * t * t * t);
  const long double inv_sqrt_2pi = 0.398942280401432677939946059934381868L;
  for (int i = 0; i < 60; ++i) {
    const long double f = normal_cdf_l(x) - p;
    const long double step = f / (inv_sqrt_2pi * std::exp(-0.5L * x * x));
    const long double nx = x - step;
    if (nx == x) break;
    x = nx;
  }
  return x;
}

void build_nf4_codebook(float levels[16], float thresholds[15]) {
  static std::once_flag once;
  static float L[16], T[15];
  std::call_once(once, [] {
    const long double p0 = 0.9677L, p_end = 0.5L;
    const long double z = normal_ppf_l(p0);
    float neg[7], pos[8];
    for (int i = 0; i < 8; ++i) {                    // 9 evenly spaced points, last (0.5) dropped
      const long double p = p0 - static_cast<long double>(i) * (p0 - p_end) / 8.0L;
      pos[i] = static_cast<float>(normal_ppf_l(p) / z);
    }
    for (int i = 0; i < 7; ++i) {                    // 8 evenly spaced points, last (0.5) dropped
      const long double p = p0 - static_cast<long double>(i) * (p0 - p_end) / 7.0L;
      neg[i] = static_cast<float>(-normal_ppf_l(p) / z);
    }
    for (int i = 0; i < 7; ++i) L[i] = neg[i];       // neg[0] = -1 ... neg[6] nearest zero
    L[7] = 0.0f;
    for (int i = 0; i < 8; ++i) L[8 + i] = pos[7 - i];
    for (int j = 0; j < 15; ++j)
      T[j] = static_cast<float>((static_cast<double>(L[j]) + static_cast<double>(L[j + 1])) / 2.0);
  });
  for (int i = 0; i < 16; ++i) levels[i] = L[i];
  for (int j = 0; j < 15; ++j) thresholds[j] = T[j];
}

}  // namespace qnf4
