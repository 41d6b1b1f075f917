// Host-side parts of libtq: error reporting, layout sizes and the Lloyd-Max
// codebook builder (tq_make_codebook).
//
// Codebook source: 7minutos.es "KV cache ... TurboQuant", Etapa 1 — after a
// random rotation a coordinate of a unit vector in R^d has density
// proportional to (1 - x^2)^((d-3)/2); Lloyd-Max alternates midpoint
// boundaries and cell-mean levels; the table depends only on (d, b) and is
// computed once. gist.science TurboESM section 2C — separate K / V tables
// fitted to their own rotated coordinates (empirical mode).
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include "tq_internal.h"

namespace tq {

namespace {
thread_local std::string g_last_error;
}

tq_status fail(tq_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

void clear_error() { g_last_error.clear(); }

tq_status check_bits(int bits, const char* what) {
  if (bits < 2 || bits > 4) return fail(TQ_ERR_INVALID_ARG, "%s must be 2, 3 or 4 (got %d)", what, bits);
  return TQ_OK;
}

tq_status check_layout(const tq_layout* layout) {
  if (!layout) return fail(TQ_ERR_INVALID_ARG, "layout is NULL");
  if (layout->d < 8 || layout->d > kMaxD || layout->d % 8 != 0)
    return fail(TQ_ERR_INVALID_ARG, "d must be a multiple of 8 in [8, %d] (got %d)", kMaxD, layout->d);
  tq_status st = check_bits(layout->key_bits, "key_bits");
  if (st != TQ_OK) return st;
  return check_bits(layout->value_bits, "value_bits");
}

// ---------------------------------------------------------------------------
// Lloyd-Max on the coordinate law f_d(x) ~ (1 - x^2)^((d-3)/2).
//
// Integrals use composite 16-point Gauss-Legendre on panels no wider than a
// sixteenth of the coordinate scale 1/sqrt(d), restricted to |x| <= 40/sqrt(d)
// (the density is below e^-800 beyond). Nodes come from Newton iteration on
// the Legendre recurrence.
// ---------------------------------------------------------------------------
namespace {

struct GaussLegendre16 {
  double x[16], w[16];
  GaussLegendre16() {
    const int n = 16;
    for (int i = 0; i < n; ++i) {
      double z = std::cos(M_PI * (i + 0.75) / (n + 0.5));
      for (int it = 0; it < 100; ++it) {
        double p0 = 1.0, p1 = z;
        for (int k = 2; k <= n; ++k) {
          double pk = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
          p0 = p1;
          p1 = pk;
        }
        double dp = n * (z * p1 - p0) / (z * z - 1.0);
        double dz = p1 / dp;
        z -= dz;
        if (std::fabs(dz) < 1e-16) break;
      }
      double p0 = 1.0, p1 = z;
      for (int k = 2; k <= n; ++k) {
        double pk = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
        p0 = p1;
        p1 = pk;
      }
      double dp = n * (z * p1 - p0) / (z * z - 1.0);
      x[i] = z;
      w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
    }
  }
};

const GaussLegendre16& gl16() {
  static GaussLegendre16 g;
  return g;
}

struct Moments {
  double m0 = 0, m1 = 0, m2 = 0;
};

double log_density(double x, int d) { return 0.5 * (d - 3) * std::log1p(-x * x); }

Moments integrate(double a, double b, int d) {
  Moments m;
  if (!(b > a)) return m;
  const double sigma = 1.0 / std::sqrt(static_cast<double>(d));
  const double max_w = sigma / 16.0;
  const long panels = std::max(4L, static_cast<long>(std::ceil((b - a) / max_w)));
  const double h = (b - a) / panels;
  const GaussLegendre16& g = gl16();
  for (long p = 0; p < panels; ++p) {
    const double lo = a + p * h, c = lo + 0.5 * h;
    for (int i = 0; i < 16; ++i) {
      const double x = c + 0.5 * h * g.x[i];
      const double f = std::exp(log_density(x, d)) * 0.5 * h * g.w[i];
      m.m0 += f;
      m.m1 += x * f;
      m.m2 += x * x * f;
    }
  }
  return m;
}

double support(int d) { return std::min(1.0, 40.0 / std::sqrt(static_cast<double>(d))); }

// Cell j spans (t_{j-1}, t_j] with t_{-1} = -L and t_{n-1} = +L.
void cell_edges(const std::vector<double>& t, int d, std::vector<double>& e) {
  const double L = support(d);
  e.assign(t.size() + 2, 0.0);
  e[0] = -L;
  for (size_t j = 0; j < t.size(); ++j) e[j + 1] = std::min(L, std::max(-L, t[j]));
  e.back() = L;
}

void quantile_start(int d, int n, std::vector<double>& c) {
  // CDF on a fine grid by the same quadrature, then linear inversion.
  const double L = support(d);
  const int grid = 40000;
  std::vector<double> xs(grid + 1), cdf(grid + 1, 0.0);
  for (int i = 0; i <= grid; ++i) xs[i] = -L + 2.0 * L * i / grid;
  for (int i = 1; i <= grid; ++i) cdf[i] = cdf[i - 1] + integrate(xs[i - 1], xs[i], d).m0;
  for (int i = 0; i <= grid; ++i) cdf[i] /= cdf[grid];
  c.resize(n);
  for (int j = 0; j < n; ++j) {
    const double p = (j + 0.5) / n;
    const int k = static_cast<int>(std::lower_bound(cdf.begin(), cdf.end(), p) - cdf.begin());
    const int k0 = std::max(1, std::min(grid, k));
    const double f = (p - cdf[k0 - 1]) / std::max(1e-300, cdf[k0] - cdf[k0 - 1]);
    c[j] = xs[k0 - 1] + f * (xs[k0] - xs[k0 - 1]);
  }
}

tq_status lloyd_analytic(int d, int bits, std::vector<double>& c, double* mse) {
  const int n = 1 << bits;
  quantile_start(d, n, c);
  std::vector<double> t(n - 1), e;
  for (int it = 0; it < 10000; ++it) {
    for (int j = 0; j + 1 < n; ++j) t[j] = 0.5 * (c[j] + c[j + 1]);
    cell_edges(t, d, e);
    double moved = 0.0;
    for (int j = 0; j < n; ++j) {
      Moments m = integrate(e[j], e[j + 1], d);
      if (m.m0 > 0.0) {
        const double nc = m.m1 / m.m0;
        moved = std::max(moved, std::fabs(nc - c[j]));
        c[j] = nc;
      }
    }
    if (moved < 1e-13) break;
  }
  std::vector<double> sym(n);
  for (int j = 0; j < n; ++j) sym[j] = 0.5 * (c[j] - c[n - 1 - j]);
  c = sym;
  if (mse) {
    for (int j = 0; j + 1 < n; ++j) t[j] = 0.5 * (c[j] + c[j + 1]);
    cell_edges(t, d, e);
    double num = 0.0, den = 0.0;
    for (int j = 0; j < n; ++j) {
      Moments m = integrate(e[j], e[j + 1], d);
      num += m.m2 - 2.0 * c[j] * m.m1 + c[j] * c[j] * m.m0;
      den += m.m0;
    }
    *mse = num / den;
  }
  return TQ_OK;
}

// Empirical Lloyd on sorted samples: cell sums from prefix sums, so each
// iteration is O(levels * log n). Start at the type-7 (linear interpolation)
// sample quantiles (j + 1/2) / 2^bits.
tq_status lloyd_empirical(const float* samples, int64_t ns, int bits, std::vector<double>& c, double* mse) {
  const int n = 1 << bits;
  std::vector<double> x(samples, samples + ns);
  for (double v : x)
    if (!std::isfinite(v)) return fail(TQ_ERR_INVALID_ARG, "samples contain a non-finite value");
  std::sort(x.begin(), x.end());
  std::vector<double> prefix(ns + 1, 0.0);
  for (int64_t i = 0; i < ns; ++i) prefix[i + 1] = prefix[i] + x[i];
  c.resize(n);
  for (int j = 0; j < n; ++j) {
    const double h = (ns - 1) * ((j + 0.5) / n);
    const int64_t lo = static_cast<int64_t>(std::floor(h));
    const int64_t hi = std::min<int64_t>(lo + 1, ns - 1);
    c[j] = x[lo] + (h - lo) * (x[hi] - x[lo]);
  }
  std::vector<int64_t> edges(n + 1), prev;
  for (int it = 0; it < 10000; ++it) {
    edges[0] = 0;
    edges[n] = ns;
    for (int j = 0; j + 1 < n; ++j) {
      const double t = 0.5 * (c[j] + c[j + 1]);
      // Samples <= t stay below the boundary (a tie goes to the lower cell).
      edges[j + 1] = std::upper_bound(x.begin(), x.end(), t) - x.begin();
    }
    for (int j = 0; j < n; ++j) {
      const int64_t cnt = edges[j + 1] - edges[j];
      if (cnt > 0) c[j] = (prefix[edges[j + 1]] - prefix[edges[j]]) / static_cast<double>(cnt);
    }
    if (edges == prev) break;
    prev = edges;
  }
  if (mse) {
    // Cells as defined by the final boundaries.
    double s = 0.0;
    std::vector<double> t(n - 1);
    for (int j = 0; j + 1 < n; ++j) t[j] = 0.5 * (c[j] + c[j + 1]);
    for (int64_t i = 0; i < ns; ++i) {
      const int cell = static_cast<int>(std::lower_bound(t.begin(), t.end(), x[i]) - t.begin());
      s += (x[i] - c[cell]) * (x[i] - c[cell]);
    }
    *mse = s / static_cast<double>(ns);
  }
  return TQ_OK;
}

}  // namespace

namespace {
std::atomic<uint64_t> g_launches{0};
}  // namespace

void count_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

uint64_t pipeline_wait_ns() {
  const char* e = std::getenv("TQ_TEST_WAIT_NS");
  if (e == nullptr || *e == 0) return 2000000000ull;
  char* end = nullptr;
  const unsigned long long v = std::strtoull(e, &end, 10);
  return (end != e && v <= 2000000000ull) ? static_cast<uint64_t>(v) : 2000000000ull;
}

}  // namespace tq

extern "C" {

uint64_t tq_kernel_launches(void) { return tq::g_launches.load(std::memory_order_relaxed); }

const char* tq_last_error_string(void) { return tq::g_last_error.c_str(); }

const char* tq_version(void) { return "tq-b200 0.1 (sm_100a)"; }

int64_t tq_idx_row_bytes(int32_t d, int32_t bits) {
  if (d <= 0 || d % 8 != 0 || bits < 1 || bits > 8) return -1;
  return tq::idx_row_bytes(d, bits);
}

int64_t tq_sign_words(int32_t d) { return d <= 0 ? -1 : tq::sign_words(d); }

int64_t tq_packed_bytes(const tq_layout* layout, int64_t n_vectors, int32_t is_key) {
  if (tq::check_layout(layout) != TQ_OK || n_vectors < 0) return -1;
  const int bits = is_key ? layout->key_bits : layout->value_bits;
  int64_t per = tq::idx_row_bytes(layout->d, bits) + 4;
  if (is_key) per += 4 * tq::sign_words(layout->d) + 4;
  return per * n_vectors;
}

tq_status tq_make_codebook(int32_t d, int32_t bits, int32_t mode, const float* samples, int64_t n_samples,
                           float* centroids, float* boundaries, double* mse_out) {
  tq::clear_error();
  if (bits < 1 || bits > 4) return tq::fail(TQ_ERR_INVALID_ARG, "bits must be in 1..4 (got %d)", bits);
  if (!centroids || !boundaries) return tq::fail(TQ_ERR_INVALID_ARG, "centroids/boundaries are NULL");
  std::vector<double> c;
  tq_status st;
  if (mode == 0) {
    if (d < 3 || d > 1 << 24) return tq::fail(TQ_ERR_INVALID_ARG, "d must be in [3, 2^24] for mode 0 (got %d)", d);
    st = tq::lloyd_analytic(d, bits, c, mse_out);
  } else if (mode == 1) {
    if (!samples || n_samples < (1 << bits))
      return tq::fail(TQ_ERR_INVALID_ARG, "mode 1 needs at least 2^bits samples");
    st = tq::lloyd_empirical(samples, n_samples, bits, c, mse_out);
  } else {
    return tq::fail(TQ_ERR_INVALID_ARG, "mode must be 0 (analytic) or 1 (empirical), got %d", mode);
  }
  if (st != TQ_OK) return st;
  const int n = 1 << bits;
  for (int j = 0; j < n; ++j) centroids[j] = static_cast<float>(c[j]);
  for (int j = 0; j + 1 < n; ++j) boundaries[j] = static_cast<float>(0.5 * (c[j] + c[j + 1]));
  for (int j = 0; j + 1 < n; ++j)
    if (!(boundaries[j] > (j ? boundaries[j - 1] : -INFINITY)))
      return tq::fail(TQ_ERR_INVALID_ARG, "codebook collapsed: boundaries not strictly increasing");
  return TQ_OK;
}

tq_status tq_residual_mean(const float* samples, int64_t n_samples, const float* centroids, const float* boundaries,
                           int32_t bits, double* e_bar) {
  tq::clear_error();
  if (bits < 1 || bits > 8) return tq::fail(TQ_ERR_INVALID_ARG, "bits must be in 1..8 (got %d)", bits);
  if (!samples || n_samples < 1 || !centroids || !boundaries || !e_bar)
    return tq::fail(TQ_ERR_INVALID_ARG, "NULL pointer or no samples");
  const int nb = (1 << bits) - 1;
  for (int j = 1; j < nb; ++j)
    if (!(boundaries[j] > boundaries[j - 1])) return tq::fail(TQ_ERR_INVALID_ARG, "boundaries not strictly increasing");
  double s = 0.0;
  for (int64_t i = 0; i < n_samples; ++i) {
    const double u = samples[i];
    // code = #{j : u > t_j} (ties go to the lower code, as in the quantiser)
    const int code = static_cast<int>(std::lower_bound(boundaries, boundaries + nb, static_cast<float>(u),
                                                       [](float t, float x) { return t < x; }) -
                                      boundaries);
    s += std::fabs(u - static_cast<double>(centroids[code]));
  }
  *e_bar = s / static_cast<double>(n_samples);
  return TQ_OK;
}

}  // extern "C"
