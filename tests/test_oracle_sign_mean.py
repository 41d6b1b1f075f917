"""Pins of the oracle's TurboESM sign-correction functions (CPU).

* d = 3: a coordinate of a random unit vector in R^3 is uniform on [-1, 1]
  (Archimedes), so the b-bit Lloyd-Max quantiser is uniform with cells of
  width 2^(1-b) and |u - c| is uniform on [0, 2^-b]: e_bar = 2^-(b+1) exactly.
* d = 128: the quadrature value matches the sample mean over coordinates of
  random unit vectors (within sampling error).
* On unit vectors with e_bar calibrated on the same coordinates, the
  correction removes exactly e_bar^2 per coordinate from the squared error:
  sum (|r| - e_bar)^2 = sum r^2 - n e_bar^2 when e_bar = mean |r|. A dropped
  norm, a flipped sign or a missing Pi^T in `reconstruct` breaks it.
* The stored bytes of the layouts (36 B at d = 64 is the 7.1x budget).
"""
import numpy as np
import pytest

import synth
from oracle import codebook as ocb
from oracle import quantize as oq
from oracle import sign_mean as osm


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_e_bar_closed_form_d3(bits):
    b = ocb.lloyd_max_beta(3, bits)
    t = 0.5 * (b.centroids[1:] + b.centroids[:-1])
    assert abs(osm.residual_mean_magnitude_beta(3, b.centroids, t) - 2.0 ** -(bits + 1)) < 1e-9
    u = np.random.default_rng(bits).uniform(-1.0, 1.0, 400000)
    assert abs(osm.residual_mean_magnitude(u, b.centroids, t) - 2.0 ** -(bits + 1)) < 5e-4


def test_e_bar_quadrature_matches_unit_vector_samples_d128():
    d, bits = 128, 3
    b = ocb.lloyd_max_beta(d, bits)
    t = 0.5 * (b.centroids[1:] + b.centroids[:-1])
    x = np.random.default_rng(3).standard_normal((20000, d))
    u = x / np.linalg.norm(x, axis=1, keepdims=True)
    e_q = osm.residual_mean_magnitude_beta(d, b.centroids, t)
    e_s = osm.residual_mean_magnitude(u, b.centroids, t)
    assert abs(e_s - e_q) < 3e-3 * e_q, (e_s, e_q)
    # a quarter of a cell width is the right scale (cells are ~0.4 sigma wide here)
    assert 0.01 < e_q * np.sqrt(d) < 0.2


def test_correction_removes_e_bar_squared_per_coordinate():
    d, bits, n = 64, 3, 3000
    b = ocb.lloyd_max_beta(d, bits)
    c = b.centroids
    t = 0.5 * (c[1:] + c[:-1])
    Pi = synth.random_rotation(d, 9).astype(np.float64)
    x = np.random.default_rng(4).standard_normal((n, d))
    x /= np.linalg.norm(x, axis=1, keepdims=True)           # unit vectors: errors need no weights
    q = oq.quantize(x, Pi, c, t, bits)
    signs = osm.residual_signs(q.codes, q.y, q.norm64, c)
    e_bar = osm.residual_mean_magnitude(q.u, c, t)
    sign_plane = oq.pack_signs(signs)
    x_tilde = osm.reconstruct(q.idx_plane, sign_plane, q.norm64, Pi, c, e_bar, bits, d)
    x_hat = osm.reconstruct(q.idx_plane, sign_plane, q.norm64, Pi, c, 0.0, bits, d)
    err_hat = np.sum((x - x_hat) ** 2)
    err_tilde = np.sum((x - x_tilde) ** 2)
    # (1e-6: Pi is an fp32 rotation, orthogonal to ~1e-7)
    assert abs(err_tilde - (err_hat - n * d * e_bar ** 2)) < 1e-6 * err_hat
    assert osm.snr_db(x, x_tilde) > osm.snr_db(x, x_hat)


def test_layout_bytes():
    assert osm.bytes_per_vector(64, 3, "sign_mean") == 36
    assert osm.bytes_per_vector(64, 3, "qjl_key") == 40
    assert osm.bytes_per_vector(64, 3, "value") == 28
    assert osm.bytes_per_vector(128, 2, "qjl_key") == 32 + 16 + 8     # TurboQuant's (b-1)+1 at b = 3
