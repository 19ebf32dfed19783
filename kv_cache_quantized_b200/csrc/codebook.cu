// Design-time codebook of the axr library (host, fp64).
//
// AXELRAM Abstract: after the orthogonal transform each coordinate of the unit key is close to N(0, 1/d), so the
// optimal scalar quantizer depends only on (d, b).  Here: the Lloyd-Max quantizer of N(0,1) with L = 2^b levels,
// found by Lloyd's fixed-point iteration on the positive half (the optimum is symmetric about zero), then scaled by
// 1/sqrt(d).  Computed once per (d, b) and cached.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "axr_common.cuh"

namespace {

constexpr double kInvSqrt2Pi = 0.39894228040143267794;

double npdf(double x) { return std::isinf(x) ? 0.0 : kInvSqrt2Pi * std::exp(-0.5 * x * x); }

// P(X >= x), X ~ N(0,1)
double upper(double x) { return 0.5 * std::erfc(x / std::sqrt(2.0)); }

// Positive-half Lloyd iteration.  m = L/2 positive levels g[0] < ... < g[m-1]; cell boundaries on the positive
// axis are a_0 = 0 (for even L the middle threshold is exactly zero by symmetry), a_i = (g[i-1] + g[i]) / 2, and
// a_m = +inf.  Centroid of [a, b): (pdf(a) - pdf(b)) / (upper(a) - upper(b)).
bool lloyd_positive_half(int L, double* g) {
  const int m = L / 2;
  for (int i = 0; i < m; ++i) g[i] = 3.0 * (i + 0.5) / m;  // spread over [0, 3]
  double a[9];
  for (int it = 0; it < 200000; ++it) {
    a[0] = 0.0;
    for (int i = 1; i < m; ++i) a[i] = 0.5 * (g[i - 1] + g[i]);
    a[m] = INFINITY;
    double moved = 0.0;
    for (int i = 0; i < m; ++i) {
      const double num = npdf(a[i]) - npdf(a[i + 1]);
      const double den = upper(a[i]) - upper(a[i + 1]);
      const double next = num / den;
      moved = std::fmax(moved, std::fabs(next - g[i]));
      g[i] = next;
    }
    if (moved < 1e-15) return true;
  }
  return false;
}

struct Entry {
  bool ready = false;
  bool ok = false;
  double c[axr::kMaxLevels];
  double t[axr::kMaxLevels];
  axr::Codebook dev;
};

std::mutex g_mu;
Entry g_cache[13][5];  // log2(d) in 0..12, bits in 1..4

bool is_pow2(int d) { return d >= 1 && (d & (d - 1)) == 0; }

int ilog2(int d) {
  int r = 0;
  while ((1 << r) < d) ++r;
  return r;
}

const Entry* entry_for(int d, int bits) {
  if (!is_pow2(d) || d > 4096 || bits < 1 || bits > 4) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  Entry& e = g_cache[ilog2(d)][bits];
  if (!e.ready) {
    const int L = 1 << bits, m = L / 2;
    double g[8];
    e.ok = lloyd_positive_half(L, g);
    const double s = 1.0 / std::sqrt(static_cast<double>(d));
    for (int i = 0; i < m; ++i) {
      e.c[m + i] = g[i] * s;
      e.c[m - 1 - i] = -g[i] * s;
    }
    for (int k = 1; k < L; ++k) e.t[k - 1] = 0.5 * (e.c[k - 1] + e.c[k]);
    e.t[m - 1] = 0.0;  // exact by symmetry
    for (int k = 0; k < axr::kMaxLevels; ++k) {
      e.dev.c[k] = k < L ? static_cast<float>(e.c[k]) : 0.0f;
      e.dev.gamma[k] = k < L ? static_cast<float>(e.c[k] * std::sqrt(static_cast<double>(d))) : 0.0f;
      // thresholds in N(0,1) units for the writer (see axr::Codebook)
      e.dev.tau[k] = k < L - 1 ? static_cast<float>(e.t[k] * std::sqrt(static_cast<double>(d))) : INFINITY;
    }
    e.ready = true;
  }
  return e.ok ? &e : nullptr;
}

}  // namespace

namespace axr {
const Codebook* codebook_for(int d, int bits) {
  const Entry* e = entry_for(d, bits);
  return e ? &e->dev : nullptr;
}
}  // namespace axr

extern "C" axr_status axr_codebook(int d, int bits, double* centroids, double* thresholds) {
  if (!centroids || !thresholds) return axr::set_error(AXR_EINVAL, "axr_codebook: null output pointer");
  if (!is_pow2(d) || d > 4096) return axr::set_error(AXR_EUNSUPPORTED, "axr_codebook: d=%d is not a power of two <= 4096", d);
  if (bits < 1 || bits > 4) return axr::set_error(AXR_EUNSUPPORTED, "axr_codebook: bits=%d outside 1..4", bits);
  const Entry* e = entry_for(d, bits);
  if (!e) return axr::set_error(AXR_EINVAL, "axr_codebook: Lloyd iteration did not converge");
  const int L = 1 << bits;
  for (int k = 0; k < L; ++k) centroids[k] = e->c[k];
  for (int k = 0; k + 1 < L; ++k) thresholds[k] = e->t[k];
  return AXR_OK;
}
