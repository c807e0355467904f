// codebook.cpp — host construction of the NormalFloat-4 code book.
//
// "QLoRA: Efficient Finetuning of Quantized LLMs" (intuitivepapers.ai),
// §NormalFloat: the literal Q^-1(i/2^k) of the paper is infinite at the ends,
// so the released construction pulls the tail probability in to 0.9677083,
// takes 8 positive normal quantiles at probabilities evenly spaced from that
// offset towards 1/2 (9 points, 1/2 itself dropped), 7 negative ones the same
// way with 8 points, adds an exact 0, sorts, and divides by the largest
// magnitude so the ends are exactly -1 and +1.
//
// Precision: several levels sit within a few hundredths of a float32 ulp of a
// rounding boundary (level 1 at 0.003 ulp), so the quantile function must be
// good to ~1e-13 relative.  We use Wichura's algorithm AS 241 (PPND16, Applied
// Statistics 37, 1988; ~1e-16 relative) and polish it with one Newton step on
// Phi(x) = erfc(-x/sqrt 2)/2.  A plain rational approximation good to 1e-9
// (e.g. Acklam's, unrefined) would round level 1 the wrong way.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include "internal.h"

namespace qlora {
namespace {

double poly(const double *c, int n, double x) {  // c[0] + c[1] x + ... + c[n-1] x^(n-1)
  double acc = c[n - 1];
  for (int i = n - 2; i >= 0; --i) acc = acc * x + c[i];
  return acc;
}

// Wichura AS 241, PPND16: inverse of the standard normal CDF.
double ppnd16(double p) {
  static const double a[8] = {3.3871328727963666080e0, 1.3314166789178437745e+2, 1.9715909503065514427e+3,
                              1.3731693765509461125e+4, 4.5921953931549871457e+4, 6.7265770927008700853e+4,
                              3.3430575583588128105e+4, 2.5090809287301226727e+3};
  static const double b[8] = {1.0,
                              4.2313330701600911252e+1,
                              6.8718700749205790830e+2,
                              5.3941960214247511077e+3,
                              2.1213794301586595867e+4,
                              3.9307895800092710610e+4,
                              2.8729085735721942674e+4,
                              5.2264952788528545610e+3};
  static const double c[8] = {1.42343711074968357734e0, 4.63033784615654529590e0, 5.76949722146069140550e0,
                              3.64784832476320460504e0, 1.27045825245236838258e0, 2.41780725177450611770e-1,
                              2.27238449892691845833e-2, 7.74545014278341407640e-4};
  static const double d[8] = {1.0,
                              2.05319162663775882187e0,
                              1.67638483018380384940e0,
                              6.89767334985100004550e-1,
                              1.48103976427480074590e-1,
                              1.51986665636164571966e-2,
                              5.47593808499534494600e-4,
                              1.05075007164441684324e-9};
  static const double e[8] = {6.65790464350110377720e0, 5.46378491116411436990e0, 1.78482653991729133580e0,
                              2.96560571828504891230e-1, 2.65321895265761230930e-2, 1.24266094738807843860e-3,
                              2.71155556874348757815e-5, 2.01033439929228813265e-7};
  static const double f[8] = {1.0,
                              5.99832206555887937690e-1,
                              1.36929880922735805310e-1,
                              1.48753612908506148525e-2,
                              7.86869131145613259100e-4,
                              1.84631831751005468180e-5,
                              1.42151175831644588870e-7,
                              2.04426310338993978564e-15};
  const double q = p - 0.5;
  if (std::fabs(q) <= 0.425) {
    const double r = 0.180625 - q * q;
    return q * poly(a, 8, r) / poly(b, 8, r);
  }
  double r = q < 0 ? p : 1.0 - p;
  r = std::sqrt(-std::log(r));
  double x;
  if (r <= 5.0) {
    r -= 1.6;
    x = poly(c, 8, r) / poly(d, 8, r);
  } else {
    r -= 5.0;
    x = poly(e, 8, r) / poly(f, 8, r);
  }
  return q < 0 ? -x : x;
}

double inv_normal_cdf(double p) {
  double x = ppnd16(p);
  // one Newton step on Phi(x) - p
  const double phi = 0.5 * std::erfc(-x / std::sqrt(2.0));
  const double pdf = std::exp(-0.5 * x * x) / std::sqrt(2.0 * M_PI);
  x -= (phi - p) / pdf;
  return x;
}

}  // namespace

void build_codebook_f64(double levels[16]) {
  const double offset = 0.9677083;
  double v[16];
  int n = 0;
  const double step_pos = (0.5 - offset) / 8.0;  // 9 points from offset to 1/2
  for (int i = 0; i < 8; ++i) v[n++] = inv_normal_cdf(offset + i * step_pos);
  const double step_neg = (0.5 - offset) / 7.0;  // 8 points from offset to 1/2
  for (int i = 0; i < 7; ++i) v[n++] = -inv_normal_cdf(offset + i * step_neg);
  v[n++] = 0.0;
  std::sort(v, v + 16);
  double mx = 0.0;
  for (double t : v) mx = std::max(mx, std::fabs(t));
  for (int i = 0; i < 16; ++i) levels[i] = v[i] / mx;
}

void thresholds_f32(const float levels[16], float thresholds[15]) {
  for (int i = 0; i < 15; ++i) {
    // exact midpoint of two float32 values in float64, then the smallest float32 above it
    const double m = (static_cast<double>(levels[i]) + static_cast<double>(levels[i + 1])) * 0.5;
    float t = static_cast<float>(m);
    if (static_cast<double>(t) <= m) t = std::nextafter(t, INFINITY);
    thresholds[i] = t;
  }
  // Of two equal levels the upper one is never the nearest (ties go to the lower
  // index): its threshold moves up to the next one, so the count skips it.
  for (int i = 13; i >= 0; --i)
    if (levels[i] == levels[i + 1]) thresholds[i] = thresholds[i + 1];
}

void build_codebook_f32(float levels[16], float thresholds[15]) {
  double l64[16];
  build_codebook_f64(l64);
  float l32[16];
  for (int i = 0; i < 16; ++i) l32[i] = static_cast<float>(l64[i]);
  if (levels) std::memcpy(levels, l32, sizeof(l32));
  if (thresholds) thresholds_f32(l32, thresholds);
}

bool build_format_codebook_f32(int codebook, float levels[16], float thresholds[15]) {
  float l32[16];
  if (codebook == QLORA_CB_NF4) {
    build_codebook_f32(l32, nullptr);
  } else if (codebook == QLORA_CB_INT4) {
    // the symmetric absmax integer grid k/7, k = -7..7, plus -8/7 (never the nearest in [-1, 1])
    for (int i = 0; i < 16; ++i) l32[i] = static_cast<float>((i - 8) / 7.0);
  } else if (codebook == QLORA_CB_FP4_E2M1 || codebook == QLORA_CB_FP4_E3M0) {
    // non-negative values of the sign + 3-bit float layout, divided by the largest;
    // both zeros of the layout are the level +0
    static const double e2m1[8] = {0, 0.5, 1, 1.5, 2, 3, 4, 6};
    static const double e3m0[8] = {0, 0.25, 0.5, 1, 2, 4, 8, 16};
    const double *pos = codebook == QLORA_CB_FP4_E2M1 ? e2m1 : e3m0;
    for (int i = 1; i < 8; ++i) {
      l32[8 + i] = static_cast<float>(pos[i] / pos[7]);
      l32[7 - i] = -l32[8 + i];
    }
    l32[7] = 0.0f;
    l32[8] = 0.0f;
  } else {
    return false;
  }
  if (levels) std::memcpy(levels, l32, sizeof(l32));
  if (thresholds) thresholds_f32(l32, thresholds);
  return true;
}

}  // namespace qlora
