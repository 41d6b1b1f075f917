"""TurboESM's one-bit residual correction, and the layouts it implies (oracle, fp64).

Test infrastructure only. Sources:
  * gist.science "TurboESM ..." section 2D: besides the 3-bit index, only the
    sign of the quantisation residual x - x_hat is stored, one extra bit; the
    decoder adds a first-order correction x_tilde = x_hat + sign * e_bar, with
    e_bar the mean residual magnitude calibrated beforehand.
  * the same pages, section 3 (results): a 1024-token ESM-2 650M cache goes
    from 330 MB (fp32 K and V) to 47 MB, 7.1x.
  * 7minutos.es "KV cache ... TurboQuant", Etapa 1 (Note): TurboQuant itself
    keeps b - 1 index bits per coordinate plus the one-bit QJL correction, b
    bits in all.

Readings (the pages leave them open):
  * the residual and its sign are taken per rotated coordinate, where the
    codes live: r_i = y_i - ||x|| c[code_i], sign_i = (r_i >= 0) (a zero
    residual counts as positive, as for the QJL signs);
  * e_bar is one number per codebook, in unit-vector coordinates: the mean of
    |u - c[code(u)]| over the calibration coordinates u (rotated unit
    vectors), so vector x is corrected by ||x|| e_bar (2 sign - 1);
  * the stored vector is its codes, its d sign bits and ||x||: 36 bytes at
    d = 64 and 3 bits, which is the budget that reproduces 330 MB -> 47 MB.
"""
from __future__ import annotations

import numpy as np

from .codebook import _cell_moments, _cells, _panels, coordinate_log_density
from .quantize import bucketize, row_bytes, unpack_codes, unpack_signs


def residual_mean_magnitude(u: np.ndarray, centroids: np.ndarray, boundaries: np.ndarray) -> float:
    """e_bar = mean |u - c[code(u)]| over the sample coordinates u."""
    u = np.asarray(u, dtype=np.float64).ravel()
    c = np.asarray(centroids, dtype=np.float64)
    return float(np.mean(np.abs(u - c[bucketize(u, np.asarray(boundaries, dtype=np.float64))])))


def residual_mean_magnitude_beta(d: int, centroids: np.ndarray, boundaries: np.ndarray) -> float:
    """E|u - c[code(u)]| under the coordinate law f_d of a random unit vector.

    Per cell [a, b] with level c: int |u - c| f = (int_c^b (u - c) f) + (int_a^c (c - u) f),
    each part by the codebook's own quadrature of (int f, int u f)."""
    c = np.asarray(centroids, dtype=np.float64)
    num = den = 0.0
    for j, (a, b) in enumerate(_cells(np.asarray(boundaries, dtype=np.float64), d)):
        cj = min(max(c[j], a), b)
        m0a, m1a, _ = _cell_moments(a, cj, d, _panels(a, cj, d))
        m0b, m1b, _ = _cell_moments(cj, b, d, _panels(cj, b, d))
        num += (m1b - c[j] * m0b) + (c[j] * m0a - m1a)
        den += m0a + m0b
    return num / den


def residual_signs(codes: np.ndarray, y: np.ndarray, norm: np.ndarray, centroids: np.ndarray) -> np.ndarray:
    """sign_i = (y_i - ||x|| c[code_i] >= 0), [n, d] bool."""
    r = np.asarray(y, dtype=np.float64) - np.asarray(norm, dtype=np.float64)[:, None] * \
        np.asarray(centroids, dtype=np.float64)[codes]
    return r >= 0.0


def reconstruct(idx_plane: np.ndarray, sign_plane: np.ndarray, norm: np.ndarray, Pi: np.ndarray,
                centroids: np.ndarray, e_bar: float, bits: int, d: int) -> np.ndarray:
    """x_tilde = Pi^T ||x|| (c[code] + e_bar (2 sign - 1)), rows [n, d]."""
    codes = unpack_codes(idx_plane, bits, d)
    pm = np.where(unpack_signs(sign_plane, d), 1.0, -1.0)
    rot = np.asarray(norm, dtype=np.float64)[:, None] * (np.asarray(centroids, dtype=np.float64)[codes] + e_bar * pm)
    return rot @ np.asarray(Pi, dtype=np.float64)


def snr_db(x: np.ndarray, x_rec: np.ndarray) -> float:
    """10 log10( sum ||x||^2 / sum ||x - x_rec||^2 )."""
    x = np.asarray(x, dtype=np.float64)
    e = x - np.asarray(x_rec, dtype=np.float64)
    return float(10.0 * np.log10(np.sum(x * x) / np.sum(e * e)))


def bytes_per_vector(d: int, bits: int, layout: str) -> int:
    """Stored bytes of one vector.

    "qjl_key"   codes + d QJL signs + ||x|| + ||r||   (the configs' keys)
    "value"     codes + ||x||                          (the configs' values)
    "sign_mean" codes + d residual signs + ||x||       (TurboESM section 2D)"""
    signs = (d + 31) // 32 * 4
    return {"qjl_key": row_bytes(d, bits) + signs + 8,
            "value": row_bytes(d, bits) + 4,
            "sign_mean": row_bytes(d, bits) + signs + 4}[layout]
