"""Pins for the oracle's Lloyd-Max codebooks (no GPU).

* d = 3: the coordinate law (1-x^2)^0 is uniform on [-1, 1], whose Lloyd-Max
  quantiser is the uniform one: levels -1 + (2j+1)/2^b, distortion
  (2/2^b)^2 / 12.
* d -> infinity: sqrt(d) x tends to N(0, 1); the levels must approach
  Max (1960)'s printed Gaussian table.
* Optimality (7minutos.es, Etapa 1): every level is the mean of its cell and
  every boundary is the midpoint of its two levels.
* The printed 1-bit worked example of the same page.
"""
import json
import os

import numpy as np
import pytest

from oracle import codebook as cb

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_uniform_law_at_d3_is_the_uniform_quantiser(bits):
    book = cb.lloyd_max_beta(3, bits)
    n = 1 << bits
    expect = -1.0 + (2.0 * np.arange(n) + 1.0) / n
    np.testing.assert_allclose(book.centroids, expect, atol=1e-12)
    np.testing.assert_allclose(book.boundaries, -1.0 + 2.0 * np.arange(1, n) / n, atol=1e-12)
    assert abs(book.mse - (2.0 / n) ** 2 / 12.0) < 1e-12


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_large_d_tends_to_max_gaussian_table(bits):
    g = _golden("max1960_gaussian.json")
    row = g["levels"][str(bits)]
    d = 1_000_000
    book = cb.lloyd_max_beta(d, bits)
    pos = np.sqrt(d) * book.centroids[len(book.centroids) // 2:]
    tol = g["table_precision"]
    np.testing.assert_allclose(pos, row["positive_levels"], atol=tol, rtol=5e-4)
    assert abs(d * book.mse - row["mse"]) <= 5e-4 * row["mse"] + 5e-6


def test_scaled_levels_converge_monotonically_in_d():
    ref = np.array(_golden("max1960_gaussian.json")["levels"]["3"]["positive_levels"])
    errs = []
    for d in (16, 64, 256, 4096):
        book = cb.lloyd_max_beta(d, 3)
        errs.append(np.max(np.abs(np.sqrt(d) * book.centroids[4:] - ref)))
    assert all(a > b for a, b in zip(errs, errs[1:])), errs


@pytest.mark.parametrize("d", [64, 128, 200])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_lloyd_max_optimality_invariants(d, bits):
    book = cb.lloyd_max_beta(d, bits)
    c, t = book.centroids, book.boundaries
    assert np.all(np.diff(c) > 0)
    np.testing.assert_allclose(t, 0.5 * (c[1:] + c[:-1]), atol=0, rtol=0)
    np.testing.assert_allclose(c, -c[::-1], atol=0)
    np.testing.assert_allclose(cb.cell_means_beta(d, t), c, atol=1e-12 / np.sqrt(d))
    # The middle boundary of the symmetric law sits exactly at zero.
    assert t[len(t) // 2] == 0.0


def test_distortion_decreases_with_bits_and_matches_gaussian_scale():
    d = 128
    mses = [cb.lloyd_max_beta(d, b).mse * d for b in (2, 3, 4)]
    assert mses[0] > mses[1] > mses[2]
    # Roughly the Gaussian values 0.1175, 0.0345, 0.0095 at this d.
    np.testing.assert_allclose(mses, [0.1175, 0.03454, 0.009497], rtol=0.05)


def test_codebook_depends_only_on_d_and_bits():
    a = cb.lloyd_max_beta(128, 3)
    b = cb.lloyd_max_beta(128, 3)
    assert np.array_equal(a.centroids, b.centroids)


def test_printed_worked_example_first_iteration():
    g = _golden("lloyd_worked_example.json")
    x = np.array(g["samples"])
    levels = np.array(g["init_levels"])
    t, cell, new = cb.lloyd_step(x, levels)
    p = g["printed"]
    tol = p["rounding_tol"]
    assert abs(t[0] - p["first_boundary"]) < 1e-15
    np.testing.assert_array_equal(levels[cell], p["first_quantized_values"])
    np.testing.assert_allclose(new, p["second_levels"], atol=tol)
    assert abs(0.5 * (new[0] + new[1]) - p["second_boundary"]) < tol


def test_worked_example_runs_to_its_fixed_point():
    g = _golden("lloyd_worked_example.json")
    book = cb.lloyd_empirical(np.array(g["samples"]), 1, init=np.array(g["init_levels"]))
    # {-0.85} | {0.97, 1.42, 2.31}: levels -0.85 and 4.70/3, boundary between them.
    np.testing.assert_allclose(book.centroids, [-0.85, (0.97 + 1.42 + 2.31) / 3.0], atol=1e-15)
    t, cell, new = cb.lloyd_step(np.array(g["samples"]), book.centroids)
    np.testing.assert_allclose(new, book.centroids, atol=1e-15)


def test_empirical_lloyd_on_sphere_samples_matches_analytic():
    # Coordinates of uniformly random unit vectors follow f_d exactly.
    d = 64
    g = np.random.default_rng(123).standard_normal((40000, d))
    u = (g / np.linalg.norm(g, axis=1, keepdims=True)).ravel()
    emp = cb.lloyd_empirical(u, 3)
    ana = cb.lloyd_max_beta(d, 3)
    np.testing.assert_allclose(emp.centroids, ana.centroids, atol=2e-3 / np.sqrt(d) * 3)
    assert abs(emp.mse - ana.mse) < 0.01 * ana.mse


def test_empirical_fixed_point_levels_are_cell_means():
    x = np.random.default_rng(5).standard_normal(5000) * 0.1
    book = cb.lloyd_empirical(x, 3)
    cell = np.searchsorted(book.boundaries, x, side="left")
    for j in range(8):
        assert abs(x[cell == j].mean() - book.centroids[j]) < 1e-14
