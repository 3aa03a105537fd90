// Codebooks of the CUDA library, derived on the host at load time: NF4 and
// the two uniform-bin 4-bit baselines it is compared with.
//
// NF4 ("QLoRA and Quantized Training", The idea; "A 65B fine-tune on the GPU
// you already have", figure 3):
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
//
// Baselines ("QLoRA Explained", The three ideas behind QLoRA: NF4 beats the
// standard 4-bit integer and float formats on normal data; "A 65B fine-tune",
// figure 3: their bins are uniform).  The pages do not define them; taken:
//   FP4  the e2m1 float (sign, 2 exponent bits with bias 1, 1 mantissa bit,
//        subnormals at exponent 0), its 16 bit patterns decoded and divided by
//        the largest magnitude, 6; ascending, so code 7 is -0 and code 8 +0.
//   INT4 symmetric absmax integers: i/7 for i = -7..7 at codes 0..14, code 15
//        repeating +1 (never chosen: its midpoint with code 14 is 1).
// Midpoints as for NF4: fp32(L_i + L_i+1) halved.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <limits>
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
  return t;
}

// Value of the e2m1 bit pattern `b` (bit 3 sign, bits 2..1 exponent, bit 0
// mantissa).
double e2m1_value(int b) {
  const int e = (b >> 1) & 3, m = b & 1;
  const double mag = e == 0 ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, e - 1);
  return (b & 8) ? -mag : mag;
}

Nf4Tables build_fp4() {
  // Negative patterns from the largest magnitude down to -0, then +0 up.
  int order[16];
  for (int i = 0; i < 8; ++i) order[i] = 15 - i;   // 1111 (-6) .. 1000 (-0)
  for (int i = 0; i < 8; ++i) order[8 + i] = i;    // 0000 (+0) .. 0111 (+6)
  const double top = e2m1_value(7);
  Nf4Tables t{};
  for (int i = 0; i < 16; ++i) t.level[i] = static_cast<float>(e2m1_value(order[i]) / top);
  t.level[7] = -0.0f;
  return t;
}

Nf4Tables build_int4() {
  Nf4Tables t{};
  for (int i = 0; i < 15; ++i) t.level[i] = static_cast<float>(static_cast<double>(i - 7) / 7.0);
  t.level[15] = 1.0f;
  return t;
}

Nf4Tables with_midpoints(Nf4Tables t) {
  for (int i = 0; i < 15; ++i) {
    volatile float s = t.level[i] + t.level[i + 1];  // fp32 add, then exact halving
    t.mid[i] = s * 0.5f;
  }
  t.pad_ = 0.0f;
  return t;
}

// Bucket tables of a codebook for the quantizer (see QuantBuckets).
QuantBuckets build_buckets(const Nf4Tables &t) {
  QuantBuckets q{};
  int bucket_of[15];
  for (int i = 0; i < 15; ++i) {
    // The device's rn(15.4 x + 16): one fp32 FMA with 1.5 * 2^23 + 16.
    const float u = std::fmaf(t.mid[i], 15.4f, 12582928.0f);
    uint32_t bits;
    std::memcpy(&bits, &u, 4);
    const int b = static_cast<int>(bits - 0x4B400000u);
    bucket_of[i] = b < 0 ? 0 : (b > 31 ? 31 : b);
    if (t.mid[i] == 0.0f) q.zero_mid = 1;
  }
  q.ok = 1;
  for (int b = 0; b < 32; ++b) {
    int c = 0;
    while (c < 15 && bucket_of[c] < b) ++c;
    q.code[b] = static_cast<uint32_t>(c);
    q.thr[b] = c < 15 ? t.mid[c] : std::numeric_limits<float>::infinity();
    // A second midpoint in this bucket must be out of reach of |x| <= 1.
    for (int i = c + 1; i < 15 && bucket_of[i] == b; ++i)
      if (t.mid[i] < 1.0f) q.ok = 0;
  }
  return q;
}

}  // namespace

const Nf4Tables &codebook_tables(int codebook) {
  static const Nf4Tables tables[kCodebookCount] = {with_midpoints(build_tables()), with_midpoints(build_fp4()),
                                                   with_midpoints(build_int4())};
  return tables[(codebook >= 0 && codebook < kCodebookCount) ? codebook : kCodebookNF4];
}

const QuantBuckets &codebook_buckets(int codebook) {
  static const QuantBuckets b[kCodebookCount] = {build_buckets(codebook_tables(kCodebookNF4)),
                                                 build_buckets(codebook_tables(kCodebookFP4)),
                                                 build_buckets(codebook_tables(kCodebookINT4))};
  return b[(codebook >= 0 && codebook < kCodebookCount) ? codebook : kCodebookNF4];
}

const Nf4Tables &nf4_tables() { return codebook_tables(kCodebookNF4); }

}  // namespace qlora
