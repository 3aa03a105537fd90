// NF4 codebook of the CUDA library, derived on the host at load time.
//
// 16 levels at quantiles of a standard normal with equal probability mass per
// bin ("QLoRA and Quantized Training", The idea; "A 65B fine-tune on the GPU
// you already have", figure 3), built so that 0 and the endpoints +-1 are
// exact: with the tail probability o = 1 - (1/32 + 1/30)/2, the positive
// levels are Phi^-1 at 8 probabilities evenly spaced from o down to (but not
// including) 1/2, the negative levels are -Phi^-1 at 7 such probabilities,
// plus 0, all divided by Phi^-1(o) and rounded once to fp32.
//
// Phi^-1 is computed here independently: bisection on the complementary error
// function in long double, polished by Newton steps.
#include <algorithm>
#include <cmath>
#include <mutex>

#include "internal.h"

namespace qlora {
namespace {

long double normal_cdf(long double z) { return 0.5L * std::erfc(-z / std::sqrt(2.0L)); }

long double normal_quantile(long double p) {
  long double lo = -12.0L, hi = 12.0L;
  for (int i = 0; i < 200; ++i) {
    const long double mid = 0.5L * (lo + hi);
    if (normal_cdf(mid) < p) lo = mid; else hi = mid;
  }
  long double z = 0.5L * (lo + hi);
  const long double inv_sqrt_2pi = 0.398942280401432677939946059934381868L;
  for (int i = 0; i < 3; ++i) {
    const long double pdf = inv_sqrt_2pi * std::exp(-0.5L * z * z);
    z -= (normal_cdf(z) - p) / pdf;
  }
  return z;
}

Nf4Tables build_tables() {
  const long double o = 1.0L - 0.5L * (1.0L / 32.0L + 1.0L / 30.0L);
  long double v[16];
  int c = 0;
  for (int i = 0; i < 8; ++i) v[c++] = normal_quantile(o - i * (o - 0.5L) / 8.0L);
  for (int i = 0; i < 7; ++i) v[c++] = -normal_quantile(o - i * (o - 0.5L) / 7.0L);
  v[c++] = 0.0L;
  std::sort(v, v + 16);
  const long double top = normal_quantile(o);
  Nf4Tables t{};
  for (int i = 0; i < 16; ++i) t.level[i] = static_cast<float>(static_cast<double>(v[i] / top));
  for (int i = 0; i < 15; ++i) {
    volatile float s = t.level[i] + t.level[i + 1];  // fp32 add, then exact halving
    t.mid[i] = s * 0.5f;
  }
  t.pad_ = 0.0f;
  return t;
}

}  // namespace

const Nf4Tables &nf4_tables() {
  static const Nf4Tables tables = build_tables();
  return tables;
}

}  // namespace qlora
