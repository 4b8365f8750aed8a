// Gaussian Lloyd-Max quantizers computed on the host by the library itself.
//
// SpectralQuant README, "Repository Structure": nonuniform_quantization.py --
// Lloyd-Max with per-regime codebooks. Each coordinate is divided by its own
// scale before quantization, so one unit-Gaussian quantizer per width b = 1..8
// serves every coordinate.
//
// Method: the optimal quantizer satisfies the centroid condition (each level is
// E[Z | Z in its cell]) and the nearest-neighbour condition (thresholds halfway
// between adjacent levels). On the positive half (the Gaussian is symmetric,
// so the middle threshold is 0), a few hundred Lloyd steps start the levels,
// then Newton's method on F_k(p) = centroid_k(p) - p_k with its analytic
// tridiagonal Jacobian converges quadratically:
//   for a cell (a, c) with probability P and centroid mu,
//   d mu / d a = phi(a) (mu - a) / P,   d mu / d c = phi(c) (c - mu) / P,
//   and each inner threshold is the mean of its two neighbouring levels.
#include <cmath>
#include <mutex>
#include <vector>

#include "../../include/sq.h"

namespace sq {

namespace {

const double kInvSqrt2Pi = 0.39894228040143267794;
const double kInvSqrt2 = 0.70710678118654752440;

double phi(double x) { return std::isinf(x) ? 0.0 : kInvSqrt2Pi * std::exp(-0.5 * x * x); }
double upper(double x) { return 0.5 * std::erfc(x * kInvSqrt2); }   // 1 - Phi(x)

struct Cell { double p, mu, m2; };

// Moments of N(0,1) on (a, c), 0 <= a < c <= inf.
Cell moments(double a, double c) {
  double p = upper(a) - upper(c);
  double pa = phi(a), pc = phi(c);
  double apa = std::isinf(a) ? 0.0 : a * pa;
  double cpc = std::isinf(c) ? 0.0 : c * pc;
  return {p, (pa - pc) / p, 1.0 + (apa - cpc) / p};
}

// Edges of the positive cells for positive levels p[0..n-1].
void edges(const std::vector<double>& p, std::vector<double>& lo, std::vector<double>& hi) {
  size_t n = p.size();
  lo.assign(n, 0.0);
  hi.assign(n, INFINITY);
  for (size_t k = 1; k < n; ++k) lo[k] = hi[k - 1] = 0.5 * (p[k - 1] + p[k]);
}

// x with upper(x) = q, q in (0, 0.5], by bisection.
double upper_inv(double q) {
  double lo = 0.0, hi = 40.0;
  for (int i = 0; i < 200; ++i) {
    double mid = 0.5 * (lo + hi);
    if (upper(mid) > q) lo = mid; else hi = mid;
  }
  return 0.5 * (lo + hi);
}

void solve_positive(int b, std::vector<double>& p) {
  size_t n = (size_t)1 << (b - 1);
  p.assign(n, 0.0);
  std::vector<double> lo, hi;
  // Start: centroids of equal-probability cells of (0, inf).
  lo.assign(n, 0.0);
  hi.assign(n, INFINITY);
  for (size_t k = 1; k < n; ++k) lo[k] = hi[k - 1] = upper_inv(0.5 * (1.0 - (double)k / (double)n));
  for (size_t k = 0; k < n; ++k) p[k] = moments(lo[k], hi[k]).mu;
  if (n == 1) return;
  for (int it = 0; it < 300; ++it) {
    edges(p, lo, hi);
    for (size_t k = 0; k < n; ++k) p[k] = moments(lo[k], hi[k]).mu;
  }
  std::vector<double> f(n), dl(n), dd(n), du(n), cp(n), dp(n);
  for (int it = 0; it < 60; ++it) {
    edges(p, lo, hi);
    double fmax = 0.0;
    for (size_t k = 0; k < n; ++k) {
      Cell c = moments(lo[k], hi[k]);
      f[k] = c.mu - p[k];
      fmax = std::fmax(fmax, std::fabs(f[k]));
      double dmu_lo = (k > 0) ? phi(lo[k]) * (c.mu - lo[k]) / c.p : 0.0;
      double dmu_hi = (k + 1 < n) ? phi(hi[k]) * (hi[k] - c.mu) / c.p : 0.0;
      dl[k] = 0.5 * dmu_lo;
      du[k] = 0.5 * dmu_hi;
      dd[k] = 0.5 * dmu_lo + 0.5 * dmu_hi - 1.0;
    }
    if (fmax < 1e-15) break;
    // Thomas algorithm for J * delta = -f.
    cp[0] = du[0] / dd[0];
    dp[0] = -f[0] / dd[0];
    for (size_t k = 1; k < n; ++k) {
      double den = dd[k] - dl[k] * cp[k - 1];
      cp[k] = du[k] / den;
      dp[k] = (-f[k] - dl[k] * dp[k - 1]) / den;
    }
    for (size_t k = n; k-- > 0;) {
      double delta = dp[k] - ((k + 1 < n) ? cp[k] * dp[k + 1] : 0.0);
      dp[k] = delta;
      p[k] += delta;
    }
  }
  for (int it = 0; it < 50; ++it) {
    edges(p, lo, hi);
    for (size_t k = 0; k < n; ++k) p[k] = moments(lo[k], hi[k]).mu;
  }
}

struct Table {
  double levels[256];
  double thresholds[255];
  double D;
};

Table g_tables[SQ_MAX_BITS + 1];
std::once_flag g_once;

void build_all() {
  for (int b = 1; b <= SQ_MAX_BITS; ++b) {
    std::vector<double> p;
    solve_positive(b, p);
    size_t n = p.size();
    Table& t = g_tables[b];
    for (size_t k = 0; k < n; ++k) {
      t.levels[n + k] = p[k];
      t.levels[n - 1 - k] = -p[k];
    }
    for (size_t k = 0; k + 1 < 2 * n; ++k) t.thresholds[k] = 0.5 * (t.levels[k] + t.levels[k + 1]);
    t.thresholds[n - 1] = 0.0;
    std::vector<double> lo, hi;
    edges(p, lo, hi);
    double dist = 0.0;
    for (size_t k = 0; k < n; ++k) {
      Cell c = moments(lo[k], hi[k]);
      dist += c.p * (c.m2 - 2.0 * p[k] * c.mu + p[k] * p[k]);
    }
    t.D = 2.0 * dist;
  }
}

}  // namespace

// Table of width b (1..8); nullptr otherwise.
const double* codebook_levels(int b) {
  std::call_once(g_once, build_all);
  return (b >= 1 && b <= SQ_MAX_BITS) ? g_tables[b].levels : nullptr;
}
const double* codebook_thresholds(int b) {
  std::call_once(g_once, build_all);
  return (b >= 1 && b <= SQ_MAX_BITS) ? g_tables[b].thresholds : nullptr;
}
double codebook_distortion(int b) {
  std::call_once(g_once, build_all);
  if (b == 0) return 1.0;
  return (b >= 1 && b <= SQ_MAX_BITS) ? g_tables[b].D : NAN;
}

}  // namespace sq

extern "C" sq_status sq_codebook(int b, double* levels, double* thresholds, double* D) {
  if (b < 1 || b > SQ_MAX_BITS) return SQ_ERR_ARG;
  const double* lv = sq::codebook_levels(b);
  const double* th = sq::codebook_thresholds(b);
  int n = 1 << b;
  if (levels)
    for (int i = 0; i < n; ++i) levels[i] = lv[i];
  if (thresholds)
    for (int i = 0; i < n - 1; ++i) thresholds[i] = th[i];
  if (D) *D = sq::codebook_distortion(b);
  return SQ_OK;
}
