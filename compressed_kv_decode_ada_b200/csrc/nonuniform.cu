// nonuniform.cu -- host tables of the non-uniform angle quantiser (an f_b
// variant): equal-mass cells for each polar angle under the angle law of a
// uniform direction on the sphere, reconstruction at the cell median; the
// azimuth keeps the uniform cells.
//
// Method: "SPHERICAL KV: Angle-Domain Attention and Rate-Distortion Retention
// for Efficient Long-Context Inference", technical summary section 2.1
// leaves the angle quantiser open.  For a uniform direction in R^d the polar
// angle phi_i (i = 1 .. d-2) has the density sin^k(phi) / Z_k, k = d - 1 - i,
// on [0, pi]; the cells are bounded by its j / 2^b quantiles and the
// reconstruction angle of cell j is its (j + 1/2) / 2^b quantile.
//
// Computation (host, fp64): the CDF F_k(theta) = int_0^theta sin^k / Z_k is
// tabulated per k on 4096 equal panels of [0, pi] by 8-point Gauss-Legendre
// quadrature (the nodes are the roots of the Legendre polynomial P_8, found
// by Newton's method on its three-term recurrence); a quantile is found by
// locating its panel in the table, then Newton steps on
// F_k(theta) - p = 0 with F_k' = sin^k / Z_k, kept inside the panel.
#include <cfloat>
#include <cmath>
#include <vector>

#include "spkv_common.cuh"

namespace spkv {
namespace {

constexpr int kGL = 8;          // Gauss-Legendre points per panel
constexpr int kPanels = 4096;   // panels over [0, pi]

struct GaussLegendre {
  double x[kGL], w[kGL];  // nodes and weights on [-1, 1]
  GaussLegendre() {
    const double pi = 3.14159265358979323846;
    for (int m = 0; m < kGL; ++m) {
      double t = std::cos(pi * (m + 0.75) / (kGL + 0.5));  // initial guess of root m
      double dp = 0.0;
      for (int it = 0; it < 100; ++it) {
        // P_n(t) by (n+1) P_{n+1} = (2n+1) t P_n - n P_{n-1}; P_n' from P_n, P_{n-1}
        double p0 = 1.0, p1 = t;
        for (int n = 1; n < kGL; ++n) {
          const double p2 = ((2.0 * n + 1.0) * t * p1 - n * p0) / (n + 1.0);
          p0 = p1;
          p1 = p2;
        }
        dp = kGL * (t * p1 - p0) / (t * t - 1.0);
        const double dt = p1 / dp;
        t -= dt;
        if (std::fabs(dt) < 1e-16) break;
      }
      x[m] = t;
      w[m] = 2.0 / ((1.0 - t * t) * dp * dp);
    }
  }
};

double sin_pow(double t, int k) {
  const double s = std::sin(t);
  double r = 1.0, base = s;
  for (int e = k; e > 0; e >>= 1) {  // s^k by squaring
    if (e & 1) r *= base;
    base *= base;
  }
  return r;
}

// int_a^b sin^k by one Gauss-Legendre panel.
double panel(const GaussLegendre &gl, double a, double b, int k) {
  const double h = 0.5 * (b - a), c = 0.5 * (a + b);
  double s = 0.0;
  for (int m = 0; m < kGL; ++m) s += gl.w[m] * sin_pow(c + h * gl.x[m], k);
  return s * h;
}

// The CDF of sin^k on [0, pi] on the panel grid, and its quantiles.
struct SinePowerLaw {
  const GaussLegendre &gl;
  int k;
  double Z;                  // int_0^pi sin^k
  std::vector<double> cum;   // cum[p] = int_0^(p * pi / kPanels) sin^k / Z
  SinePowerLaw(const GaussLegendre &g, int k_) : gl(g), k(k_), cum(kPanels + 1) {
    const double pi = 3.14159265358979323846, hp = pi / kPanels;
    cum[0] = 0.0;
    for (int p = 0; p < kPanels; ++p) cum[p + 1] = cum[p] + panel(gl, p * hp, (p + 1) * hp, k);
    Z = cum[kPanels];
    for (int p = 0; p <= kPanels; ++p) cum[p] /= Z;
  }
  double cdf(double theta) const {
    const double pi = 3.14159265358979323846, hp = pi / kPanels;
    int p = (int)(theta / hp);
    p = p < 0 ? 0 : (p >= kPanels ? kPanels - 1 : p);
    return cum[p] + panel(gl, p * hp, theta, k) / Z;
  }
  double quantile(double prob) const {
    const double pi = 3.14159265358979323846, hp = pi / kPanels;
    // the panel holding prob (cum is nondecreasing)
    int lo = 0, hi = kPanels;
    while (hi - lo > 1) {
      const int mid = (lo + hi) / 2;
      if (cum[mid] <= prob) lo = mid;
      else hi = mid;
    }
    double a = lo * hp, b = (lo + 1) * hp;
    double t = 0.5 * (a + b);
    for (int it = 0; it < 60; ++it) {
      const double f = cdf(t) - prob;
      if (f > 0) b = t;
      else a = t;
      const double dens = sin_pow(t, k) / Z;
      double tn = dens > 0 ? t - f / dens : 0.5 * (a + b);
      if (!(tn > a && tn < b)) tn = 0.5 * (a + b);  // stay in the bracket
      // done when the Newton step or the bracket is down to two ulps of t
      // (the iteration cap is only a backstop)
      const double two_ulps = 2.0 * DBL_EPSILON * std::fabs(t) + 1e-300;
      const bool done = std::fabs(tn - t) <= two_ulps || b - a <= two_ulps;
      t = tn;
      if (done) break;
    }
    return t;
  }
};

}  // namespace
}  // namespace spkv

extern "C" spkv_status spkv_nonuniform_tables(int32_t d, int32_t b, double *edge_cos, double *mid_cos,
                                              double *mid_sin) {
  using namespace spkv;
  if (d < 3 || d > 4096 || b < 1 || b > 12 || !edge_cos || !mid_cos || !mid_sin) return SPKV_ERR_INVALID_ARG;
  static const GaussLegendre gl;
  const int n = 1 << b;
  for (int i = 1; i <= d - 2; ++i) {
    const SinePowerLaw law(gl, d - 1 - i);
    double *ec = edge_cos + (size_t)(i - 1) * (n - 1);
    double *mc = mid_cos + (size_t)(i - 1) * n;
    double *ms = mid_sin + (size_t)(i - 1) * n;
    for (int j = 1; j < n; ++j) ec[j - 1] = std::cos(law.quantile((double)j / n));
    for (int j = 0; j < n; ++j) {
      const double t = law.quantile((j + 0.5) / n);
      mc[j] = std::cos(t);
      ms[j] = std::sin(t);
    }
  }
  return SPKV_OK;
}
