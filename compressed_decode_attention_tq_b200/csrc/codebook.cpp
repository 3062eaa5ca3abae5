// Host Lloyd-Max codebook for the C ABI (tq_codebook).
//
// "TurboQuant explained" (Mobilint blog), section "Coordinates Become Predictable
// After Rotation": a coordinate of a randomly rotated unit vector in R^d has density
// f_X(t) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) (1 - t^2)^((d-3)/2) on [-1, 1], i.e.
// (t + 1)/2 ~ Beta(a, a) with a = (d - 1)/2; it tends to N(0, 1/d).
// Section "Designing the Optimal Codebook Without Data": Lloyd-Max alternates
// (1) boundaries = midpoints of adjacent centroids and (2) centroids = conditional
// means of their cells until convergence.
//
// The cell mass uses the regularized incomplete Beta function, evaluated with the
// continued fraction of Abramowitz & Stegun 26.5.8 (modified Lentz evaluation); the
// first moment uses the antiderivative of t f_X(t), -K (1 - t^2)^a / (2a).  The
// Gaussian option uses erfc and the Gaussian first moment sigma (phi(lo/s) - phi(hi/s)).
#include <cmath>
#include <cstdint>
#include <vector>

#include "tq.h"
#include "tq_internal.h"

namespace {

// log B(a, b)
double log_beta_fn(double a, double b) { return std::lgamma(a) + std::lgamma(b) - std::lgamma(a + b); }

// Continued fraction part of I_x(a, b) (A&S 26.5.8), valid for x < (a + 1)/(a + b + 2).
double inc_beta_cf(double a, double b, double x) {
  const double tiny = 1e-300;
  double c = 1.0;
  double dd = 1.0 - (a + b) * x / (a + 1.0);
  if (std::fabs(dd) < tiny) dd = tiny;
  dd = 1.0 / dd;
  double h = dd;
  for (int m = 1; m <= 10000; ++m) {
    const double m2 = 2.0 * m;
    // even step d_{2m}
    double num = m * (b - m) * x / ((a + m2 - 1.0) * (a + m2));
    dd = 1.0 + num * dd;
    if (std::fabs(dd) < tiny) dd = tiny;
    c = 1.0 + num / c;
    if (std::fabs(c) < tiny) c = tiny;
    dd = 1.0 / dd;
    h *= dd * c;
    // odd step d_{2m+1}
    num = -(a + m) * (a + b + m) * x / ((a + m2) * (a + m2 + 1.0));
    dd = 1.0 + num * dd;
    if (std::fabs(dd) < tiny) dd = tiny;
    c = 1.0 + num / c;
    if (std::fabs(c) < tiny) c = tiny;
    dd = 1.0 / dd;
    const double del = dd * c;
    h *= del;
    if (std::fabs(del - 1.0) < 1e-16) break;
  }
  return h;
}

// Regularized incomplete Beta I_x(a, b).
double inc_beta(double a, double b, double x) {
  if (x <= 0.0) return 0.0;
  if (x >= 1.0) return 1.0;
  const double lfront = a * std::log(x) + b * std::log1p(-x) - log_beta_fn(a, b);
  if (x < (a + 1.0) / (a + b + 2.0)) return std::exp(lfront) * inc_beta_cf(a, b, x) / a;
  return 1.0 - std::exp(lfront) * inc_beta_cf(b, a, 1.0 - x) / b;
}

struct Density {
  int d;
  bool gauss;
  double cdf(double t) const {
    if (gauss) return 0.5 * std::erfc(-t * std::sqrt(d / 2.0));
    if (t <= -1.0) return 0.0;
    if (t >= 1.0) return 1.0;
    const double a = (d - 1) / 2.0;
    return inc_beta(a, a, (t + 1.0) / 2.0);
  }
  // int_lo^hi t f(t) dt
  double first_moment(double lo, double hi) const {
    if (gauss) {
      const double s = 1.0 / std::sqrt((double)d);
      auto phi = [](double z) { return std::exp(-0.5 * z * z) / std::sqrt(2.0 * M_PI); };
      const double plo = std::isinf(lo) ? 0.0 : phi(lo / s);
      const double phi_hi = std::isinf(hi) ? 0.0 : phi(hi / s);
      return s * (plo - phi_hi);
    }
    const double a = (d - 1) / 2.0;
    const double k = std::exp(std::lgamma(d / 2.0) - std::lgamma((d - 1) / 2.0)) / std::sqrt(M_PI);
    auto tail = [&](double t) {
      t = std::fmin(1.0, std::fmax(-1.0, t));
      return std::pow(1.0 - t * t, a);
    };
    return k / (d - 1.0) * (tail(lo) - tail(hi));
  }
};

}  // namespace

extern "C" tq_status tq_codebook(int32_t bits, int32_t head_dim, int32_t density, float* centroids,
                                 float* boundaries) {
  if (bits < 1 || bits > 8) return tqi::fail(TQ_ERR_INVALID_ARG, "tq_codebook: bits must be in 1..8");
  if (head_dim < 3) return tqi::fail(TQ_ERR_INVALID_ARG, "tq_codebook: head_dim must be >= 3");
  if (density != TQ_DENSITY_BETA && density != TQ_DENSITY_GAUSS)
    return tqi::fail(TQ_ERR_INVALID_ARG, "tq_codebook: unknown density");
  if (!centroids || !boundaries)
    return tqi::fail(TQ_ERR_INVALID_ARG, "tq_codebook: null output pointer");
  const int n = 1 << bits;
  const Density f{head_dim, density == TQ_DENSITY_GAUSS};
  const double sigma = 1.0 / std::sqrt((double)head_dim);
  const double lo_end = f.gauss ? -INFINITY : -1.0, hi_end = f.gauss ? INFINITY : 1.0;
  std::vector<double> c(n), cn(n), edge(n + 1);
  for (int i = 0; i < n; ++i)
    c[i] = (n == 1) ? 0.0 : -2.0 * sigma + 4.0 * sigma * i / (n - 1);
  for (int it = 0; it < 100000; ++it) {
    edge[0] = lo_end;
    edge[n] = hi_end;
    for (int i = 1; i < n; ++i) edge[i] = 0.5 * (c[i - 1] + c[i]);
    double delta = 0.0;
    for (int i = 0; i < n; ++i) {
      const double mass = f.cdf(edge[i + 1]) - f.cdf(edge[i]);
      cn[i] = f.first_moment(edge[i], edge[i + 1]) / mass;
      delta = std::fmax(delta, std::fabs(cn[i] - c[i]));
    }
    c.swap(cn);
    if (delta < 1e-13) break;
  }
  // symmetrise: the density is even, so the exact fixed point is
  for (int i = 0; i < n / 2; ++i) {
    const double v = 0.5 * (c[n - 1 - i] - c[i]);
    c[i] = -v;
    c[n - 1 - i] = v;
  }
  for (int i = 0; i < n; ++i) centroids[i] = (float)c[i];
  for (int i = 0; i + 1 < n; ++i) boundaries[i] = (i == n / 2 - 1) ? 0.0f : (float)(0.5 * (c[i] + c[i + 1]));
  return TQ_OK;
}

// Uniform grid of the dithered quantizer ("Minimum Distortion Quantization with Specified
// Output Distribution" page, third abstract).  With subtractive dither the expected squared
// error of a coordinate y is delta^2/12 inside the outer levels and delta^2/12 + (|y| - A)^2
// beyond them (A = (n-1) delta / 2), so D(delta) = delta^2/12 + 2 int_A^inf (t - A)^2 f(t) dt
// and dD/d delta = delta/6 - 2 (n-1) [P1(A) - A P0(A)], P_k(A) = int_A^inf t^k f(t) dt.  The
// derivative grows with delta (its own derivative is 1/6 + (n-1)^2 P0 > 0); its root is
// found by bisection.
extern "C" tq_status tq_dither_codebook(int32_t bits, int32_t head_dim, int32_t density, float* centroids,
                                        float* boundaries) {
  if (bits < 1 || bits > 8) return tqi::fail(TQ_ERR_INVALID_ARG, "tq_dither_codebook: bits must be in 1..8");
  if (head_dim < 3) return tqi::fail(TQ_ERR_INVALID_ARG, "tq_dither_codebook: head_dim must be >= 3");
  if (density != TQ_DENSITY_BETA && density != TQ_DENSITY_GAUSS)
    return tqi::fail(TQ_ERR_INVALID_ARG, "tq_dither_codebook: unknown density");
  if (!centroids || !boundaries)
    return tqi::fail(TQ_ERR_INVALID_ARG, "tq_dither_codebook: null output pointer");
  const int n = 1 << bits;
  const Density f{head_dim, density == TQ_DENSITY_GAUSS};
  const double hi_end = f.gauss ? INFINITY : 1.0;
  auto slope = [&](double step) {
    const double A = (n - 1) * step / 2.0;
    if (!f.gauss && A >= 1.0) return step / 6.0;
    double p0;
    if (f.gauss) {
      p0 = 0.5 * std::erfc(A * std::sqrt(f.d / 2.0));
    } else {
      const double a = (f.d - 1) / 2.0;
      p0 = inc_beta(a, a, (1.0 - A) / 2.0);  // 1 - F(A), by the density's symmetry
    }
    const double p1 = f.first_moment(A, hi_end);
    return step / 6.0 - 2.0 * (n - 1) * (p1 - A * p0);
  };
  double lo = 0.0;
  double hi = f.gauss ? 80.0 / std::sqrt((double)head_dim) / (n - 1) : 2.0 / (n - 1);
  while (slope(hi) <= 0.0) hi *= 2.0;
  for (int it = 0; it < 200; ++it) {
    const double mid = 0.5 * (lo + hi);
    if (mid == lo || mid == hi) break;
    if (slope(mid) > 0.0)
      hi = mid;
    else
      lo = mid;
  }
  const double step = 0.5 * (lo + hi);
  for (int j = 0; j < n; ++j) centroids[j] = (float)((j - (n - 1) / 2.0) * step);
  for (int j = 0; j + 1 < n; ++j) boundaries[j] = (float)((j + 1.0 - n / 2.0) * step);
  return TQ_OK;
}
