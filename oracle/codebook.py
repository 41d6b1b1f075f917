"""Lloyd-Max codebooks (oracle; test infrastructure only).

Follows 7minutos.es "KV cache ... TurboQuant", Etapa 1 (PolarQuant):
  * after a random orthogonal rotation, x_i^2 / sum_j x_j^2 ~ Beta(1/2, (d-1)/2),
    i.e. a coordinate of a uniformly random unit vector has density
    f_d(x) proportional to (1 - x^2)^((d-3)/2) on [-1, 1];
  * Lloyd-Max places 2^b levels to minimise the mean squared error: the
    boundary between two levels is their midpoint, each level is the mean of
    the values in its cell, repeated until the error stops improving
    (worked example with samples [1.42, -0.85, 2.31, 0.97] and levels [0.5, 1.5]);
  * the codebook depends only on (d, b) and is computed once, offline.
The TurboESM pages (gist.science, section 2C "Dual LUT") fit separate K and V
tables to their own post-rotation distributions; that is the empirical mode.

Readings where the pages are silent: start from the 2^b equiprobable quantiles,
stop when no level moves by 1e-13 (analytic) or no sample changes cell
(empirical), and make the analytic codebook exactly symmetric.
"""
from __future__ import annotations

import dataclasses

import numpy as np

_GL_X, _GL_W = np.polynomial.legendre.leggauss(8)


@dataclasses.dataclass
class Codebook:
    centroids: np.ndarray    # [2^b] float64, increasing
    boundaries: np.ndarray   # [2^b - 1] float64, midpoints of adjacent centroids
    mse: float               # per-coordinate distortion E[(x - c(x))^2]
    iterations: int


def coordinate_log_density(x: np.ndarray, d: int) -> np.ndarray:
    """log f_d(x) up to an additive constant: ((d-3)/2) * log(1 - x^2)."""
    return 0.5 * (d - 3) * np.log1p(-x * x)


def _support(d: int) -> float:
    # Beyond 40 standard deviations (sigma = 1/sqrt(d)) the density is below e^-800.
    return min(1.0, 40.0 / np.sqrt(d))


def _cell_moments(a: float, b: float, d: int, panels: int) -> tuple[float, float, float]:
    """(int f, int x f, int x^2 f) over [a, b] by composite 8-point Gauss-Legendre,
    with f = exp(log f_d) unnormalised."""
    if b <= a:
        return 0.0, 0.0, 0.0
    edges = np.linspace(a, b, panels + 1)
    half = 0.5 * (edges[1:] - edges[:-1])
    mid = 0.5 * (edges[1:] + edges[:-1])
    x = mid[:, None] + half[:, None] * _GL_X[None, :]
    w = half[:, None] * _GL_W[None, :]
    f = np.exp(coordinate_log_density(x, d)) * w
    return float(f.sum()), float((x * f).sum()), float((x * x * f).sum())


def _cells(boundaries: np.ndarray, d: int) -> list[tuple[float, float]]:
    lim = _support(d)
    edges = np.concatenate([[-lim], np.clip(boundaries, -lim, lim), [lim]])
    return [(edges[j], edges[j + 1]) for j in range(len(edges) - 1)]


def _panels(a: float, b: float, d: int, total: int = 2000) -> int:
    return max(16, int(np.ceil(total * (b - a) / (2.0 * _support(d)))))


def beta_quantiles(d: int, probs: np.ndarray, grid: int = 200001) -> np.ndarray:
    """Quantiles of f_d by a fine trapezoidal CDF (used only to start Lloyd)."""
    lim = _support(d)
    x = np.linspace(-lim, lim, grid)
    f = np.exp(coordinate_log_density(np.clip(x, -1 + 1e-15, 1 - 1e-15), d))
    cdf = np.concatenate([[0.0], np.cumsum(0.5 * (f[1:] + f[:-1]) * np.diff(x))])
    cdf /= cdf[-1]
    return np.interp(probs, cdf, x)


def lloyd_max_beta(d: int, bits: int, tol: float = 1e-13, max_iter: int = 10000) -> Codebook:
    """Lloyd-Max quantiser for a coordinate of a random unit vector in R^d."""
    if d < 3:
        raise ValueError("the coordinate law needs d >= 3")
    n = 1 << bits
    c = beta_quantiles(d, (np.arange(n) + 0.5) / n)
    it = 0
    for it in range(1, max_iter + 1):
        t = 0.5 * (c[1:] + c[:-1])
        new = c.copy()
        for j, (a, b) in enumerate(_cells(t, d)):
            m0, m1, _ = _cell_moments(a, b, d, _panels(a, b, d))
            if m0 > 0.0:
                new[j] = m1 / m0
        moved = np.max(np.abs(new - c))
        c = new
        if moved < tol:
            break
    c = 0.5 * (c - c[::-1])   # exact symmetry of the symmetric law
    t = 0.5 * (c[1:] + c[:-1])
    return Codebook(centroids=c, boundaries=t, mse=beta_distortion(d, c, t), iterations=it)


def beta_distortion(d: int, centroids: np.ndarray, boundaries: np.ndarray) -> float:
    """E[(x - c_cell(x))^2] under f_d, by the same quadrature."""
    num = 0.0
    den = 0.0
    for j, (a, b) in enumerate(_cells(boundaries, d)):
        m0, m1, m2 = _cell_moments(a, b, d, _panels(a, b, d))
        cj = centroids[j]
        num += m2 - 2.0 * cj * m1 + cj * cj * m0
        den += m0
    return num / den


def cell_means_beta(d: int, boundaries: np.ndarray) -> np.ndarray:
    """Conditional mean of x in every cell (for the optimality invariant)."""
    out = []
    for a, b in _cells(boundaries, d):
        m0, m1, _ = _cell_moments(a, b, d, _panels(a, b, d))
        out.append(m1 / m0)
    return np.asarray(out)


# --------------------------------------------------------------------------
# Empirical Lloyd on samples (dual K/V tables fitted to calibration data).
# --------------------------------------------------------------------------
def lloyd_step(samples: np.ndarray, levels: np.ndarray) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """One Lloyd iteration exactly as the worked example runs it.

    Returns (boundaries, cell index of every sample, new levels). A sample equal
    to a boundary stays in the lower cell; an empty cell keeps its level."""
    t = 0.5 * (levels[1:] + levels[:-1])
    cell = np.array([int(np.sum(x > t)) for x in samples]) if samples.size < 64 else \
        np.searchsorted(t, samples, side="left")
    new = levels.astype(np.float64).copy()
    for j in range(len(levels)):
        members = samples[cell == j]
        if members.size:
            new[j] = members.mean()
    return t, cell, new


def lloyd_empirical(samples: np.ndarray, bits: int, init: np.ndarray | None = None,
                    max_iter: int = 10000) -> Codebook:
    """Lloyd iteration on a finite sample until no sample changes cell."""
    x = np.sort(np.asarray(samples, dtype=np.float64).ravel())
    n = 1 << bits
    if init is None:
        c = np.quantile(x, (np.arange(n) + 0.5) / n)
    else:
        c = np.asarray(init, dtype=np.float64).copy()
    prefix = np.concatenate([[0.0], np.cumsum(x)])
    prev_edges = None
    it = 0
    for it in range(1, max_iter + 1):
        t = 0.5 * (c[1:] + c[:-1])
        # cell j holds samples with t_{j-1} < x <= t_j
        edges = np.concatenate([[0], np.searchsorted(x, t, side="right"), [x.size]])
        counts = np.diff(edges)
        sums = prefix[edges[1:]] - prefix[edges[:-1]]
        c = np.where(counts > 0, sums / np.maximum(counts, 1), c)
        if prev_edges is not None and np.array_equal(edges, prev_edges):
            break
        prev_edges = edges
    t = 0.5 * (c[1:] + c[:-1])
    cell = np.searchsorted(t, x, side="left")
    mse = float(np.mean((x - c[cell]) ** 2))
    return Codebook(centroids=c, boundaries=t, mse=mse, iterations=it)
