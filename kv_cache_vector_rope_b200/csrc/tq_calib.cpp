// Host-side calibration utilities of libtq (offline, like the codebook):
//   tq_fit_rotation      per-head rotation Pi_h = Pi_rand V^T from calibration
//                        vectors (V: right singular vectors, by a cyclic Jacobi
//                        eigen-solve of X^T X in fp64)
//   tq_rotate_normalize  coordinates of Pi x / ||x||, the samples the dual
//                        (K / V) Lloyd codebooks are fitted to
//
// Source: gist.science "TurboESM ..." section 2B (a Pi per layer and head,
// computed by SVD of real activations) and section 2C (separate K and V
// tables fitted to their own post-rotation distributions).
//
// Readings: the calibration matrix is used uncentred; singular vectors are
// ordered by decreasing singular value and each is signed so that its
// largest-magnitude entry (first one on a tie) is positive; Pi_h = Pi_rand V^T
// (turn into the singular basis first, then apply the seeded rotation).
#include <algorithm>
#include <cmath>
#include <numeric>
#include <vector>

#include "tq_internal.h"

namespace tq {
namespace {

// Eigen-decomposition of the symmetric d x d matrix A (row-major, destroyed)
// by cyclic Jacobi rotations. On return w holds the eigenvalues and the
// columns of V the eigenvectors.
void jacobi_eigen(std::vector<double>& A, int d, std::vector<double>& w, std::vector<double>& V) {
  V.assign(static_cast<size_t>(d) * d, 0.0);
  for (int i = 0; i < d; ++i) V[i * d + i] = 1.0;
  double total = 0.0;
  for (double x : A) total += x * x;
  for (int sweep = 0; sweep < 100; ++sweep) {
    double off = 0.0;
    for (int p = 0; p < d; ++p)
      for (int q = p + 1; q < d; ++q) off += A[p * d + q] * A[p * d + q];
    if (off <= 1e-30 * total) break;
    for (int p = 0; p < d; ++p) {
      for (int q = p + 1; q < d; ++q) {
        const double apq = A[p * d + q];
        if (apq == 0.0) continue;
        const double app = A[p * d + p], aqq = A[q * d + q];
        const double theta = (aqq - app) / (2.0 * apq);
        const double t = (theta >= 0 ? 1.0 : -1.0) / (std::fabs(theta) + std::sqrt(theta * theta + 1.0));
        const double c = 1.0 / std::sqrt(t * t + 1.0), s = t * c;
        for (int k = 0; k < d; ++k) {   // A <- A J (columns p, q)
          const double akp = A[k * d + p], akq = A[k * d + q];
          A[k * d + p] = c * akp - s * akq;
          A[k * d + q] = s * akp + c * akq;
        }
        for (int k = 0; k < d; ++k) {   // A <- J^T A (rows p, q)
          const double apk = A[p * d + k], aqk = A[q * d + k];
          A[p * d + k] = c * apk - s * aqk;
          A[q * d + k] = s * apk + c * aqk;
        }
        for (int k = 0; k < d; ++k) {   // V <- V J
          const double vkp = V[k * d + p], vkq = V[k * d + q];
          V[k * d + p] = c * vkp - s * vkq;
          V[k * d + q] = s * vkp + c * vkq;
        }
      }
    }
  }
  w.resize(d);
  for (int i = 0; i < d; ++i) w[i] = A[i * d + i];
}

}  // namespace
}  // namespace tq

extern "C" tq_status tq_fit_rotation(int32_t d, const float* X, int64_t n, const float* Pi_rand, float* Pi_out) {
  using namespace tq;
  clear_error();
  if (d < 2 || d > kMaxD) return fail(TQ_ERR_INVALID_ARG, "d must be in [2, %d] (got %d)", kMaxD, d);
  if (n < 1 || !X || !Pi_rand || !Pi_out) return fail(TQ_ERR_INVALID_ARG, "need n >= 1 and non-NULL X, Pi_rand, Pi_out");
  // Gram matrix G = X^T X in fp64.
  std::vector<double> G(static_cast<size_t>(d) * d, 0.0);
  for (int64_t r = 0; r < n; ++r) {
    const float* x = X + r * d;
    for (int i = 0; i < d; ++i) {
      const double xi = x[i];
      if (!std::isfinite(xi)) return fail(TQ_ERR_INVALID_ARG, "X contains a non-finite value");
      for (int j = i; j < d; ++j) G[i * d + j] += xi * static_cast<double>(x[j]);
    }
  }
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < i; ++j) G[i * d + j] = G[j * d + i];
  std::vector<double> w, V;
  jacobi_eigen(G, d, w, V);
  // Order by decreasing eigenvalue (= squared singular value).
  std::vector<int> order(d);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return w[a] > w[b]; });
  std::vector<double> Vs(static_cast<size_t>(d) * d);
  for (int c = 0; c < d; ++c) {
    const int src = order[c];
    int kmax = 0;
    for (int k = 1; k < d; ++k)
      if (std::fabs(V[k * d + src]) > std::fabs(V[kmax * d + src])) kmax = k;
    const double sgn = V[kmax * d + src] < 0.0 ? -1.0 : 1.0;
    for (int k = 0; k < d; ++k) Vs[k * d + c] = sgn * V[k * d + src];
  }
  // Pi_out = Pi_rand V^T: (Pi_rand V^T)[i][j] = sum_k Pi_rand[i][k] V[j][k].
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) {
      double acc = 0.0;
      for (int k = 0; k < d; ++k) acc += static_cast<double>(Pi_rand[i * d + k]) * Vs[j * d + k];
      Pi_out[i * d + j] = static_cast<float>(acc);
    }
  return TQ_OK;
}

extern "C" tq_status tq_rotate_normalize(int32_t d, const float* X, int64_t n, const float* Pi, float* u_out,
                                         int64_t* n_out) {
  using namespace tq;
  clear_error();
  if (d < 2 || d > kMaxD) return fail(TQ_ERR_INVALID_ARG, "d must be in [2, %d] (got %d)", kMaxD, d);
  if (n < 0 || !X || !Pi || !u_out || !n_out) return fail(TQ_ERR_INVALID_ARG, "NULL pointer or negative n");
  int64_t m = 0;
  for (int64_t r = 0; r < n; ++r) {
    const float* x = X + r * d;
    double ss = 0.0;
    for (int j = 0; j < d; ++j) ss += static_cast<double>(x[j]) * x[j];
    if (!(ss > 0.0)) continue;   // a zero vector has no direction
    const double inv = 1.0 / std::sqrt(ss);
    float* u = u_out + m * d;
    for (int i = 0; i < d; ++i) {
      double acc = 0.0;
      for (int j = 0; j < d; ++j) acc += static_cast<double>(Pi[i * d + j]) * x[j];
      u[i] = static_cast<float>(acc * inv);
    }
    ++m;
  }
  *n_out = m;
  return TQ_OK;
}
