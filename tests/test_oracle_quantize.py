"""Pins for the oracle's quantiser (no GPU).

* Pi from the seeded generator is orthogonal and preserves inner products
  (gist.science TurboESM, section 2A: Pi^T Pi = I).
* RoPE is a rotation with the relative-position property the same section's
  equation relies on: (R_i q)^T (R_j k) = q^T R_i^T R_j k depends on j - i.
* The strict-boundary bucketize equals brute force over all centroids.
* Packing round-trips; the documented bit order gives a fixed byte pattern.
* The empirical per-coordinate MSE of Gaussian vectors equals the Lloyd-Max
  distortion from integration (7minutos.es, Etapa 1).
* The QJL estimate is unbiased: its mean over many draws of S is the true
  inner product (7minutos.es, Etapa 2: the sqrt(pi/2)/d factor removes the
  bias); with q = r the mean is ||r||^2.
"""
import math

import numpy as np
import pytest

import synth
from oracle import attention as oa
from oracle import codebook as cb
from oracle import quantize as oq


def test_generated_rotation_is_orthogonal_and_preserves_inner_products():
    for d in (64, 128, 200):
        Pi = synth.random_rotation(d, 0).astype(np.float64)
        assert np.max(np.abs(Pi.T @ Pi - np.eye(d))) <= 2e-6
        a, b = np.random.default_rng(1).standard_normal((2, d))
        assert abs((Pi @ a) @ (Pi @ b) - a @ b) <= 1e-5 * np.linalg.norm(a) * np.linalg.norm(b)


def test_rope_is_a_rotation_with_relative_position_property():
    d, base = 64, 10000.0
    rg = np.random.default_rng(2)
    q, k = rg.standard_normal((2, d))
    for pos in (0, 1, 17, 255):
        assert abs(np.linalg.norm(oq.rope(q, pos, base)) - np.linalg.norm(q)) < 1e-12
    np.testing.assert_allclose(oq.rope(q, 0, base), q, atol=0)
    ref = oq.rope(q, 0, base) @ oq.rope(k, 5, base)
    for m in (1, 7, 100, 250):
        assert abs(oq.rope(q, m, base) @ oq.rope(k, m + 5, base) - ref) < 1e-11


def test_rope_literal_values_of_the_published_definition():
    # Rotate-half RoPE as published (RoFormer, Su et al., section 3.4.2, with
    # theta_i = base^(-2(i-1)/d) for 1-based pair index i; the pairing of
    # channel i with channel i + d/2 is the rotate-half convention). Worked by
    # hand at d = 4, base = 1e4, position 1: the two pair angles are 1 and
    # 1e4^(-1/2) = 0.01, so e_0 -> (cos 1, 0, sin 1, 0), e_1 -> (0, cos .01, 0,
    # sin .01), e_2 -> (-sin 1, 0, cos 1, 0), e_3 -> (0, -sin .01, 0, cos .01).
    c1, s1 = 0.5403023058681398, 0.8414709848078965          # cos 1, sin 1
    c2, s2 = 0.9999500004166653, 0.009999833334166664        # cos .01, sin .01
    expect = np.array([[c1, 0.0, s1, 0.0],
                       [0.0, c2, 0.0, s2],
                       [-s1, 0.0, c1, 0.0],
                       [0.0, -s2, 0.0, c2]])
    np.testing.assert_allclose(oq.rope(np.eye(4), np.ones(4), 1e4), expect, atol=1e-15)
    # d = 8, position 3: angles 3, 0.3, 0.03, 0.003 (exponents 0, -1/4, -1/2,
    # -3/4 of 1e4). A wrong exponent such as -i/d or -2(i+1)/d moves them.
    ang = np.array([3.0, 0.3, 0.03, 0.003])
    out = oq.rope(np.eye(8)[:4], np.full(4, 3), 1e4)
    for i in range(4):
        want = np.zeros(8)
        want[i], want[i + 4] = math.cos(ang[i]), math.sin(ang[i])
        np.testing.assert_allclose(out[i], want, atol=1e-14)


def test_rope_then_rotation_preserves_scores():
    # (Pi R_i q)^T (Pi R_j k) = q^T R_i^T R_j k.
    d = 64
    rg = np.random.default_rng(3)
    Pi, _ = np.linalg.qr(rg.standard_normal((d, d)))   # orthogonal to fp64 rounding
    q, k = rg.standard_normal((2, d))
    lhs = (Pi @ oq.rope(q, 40, 1e4)) @ (Pi @ oq.rope(k, 9, 1e4))
    rhs = oq.rope(q, 40, 1e4) @ oq.rope(k, 9, 1e4)
    assert abs(lhs - rhs) < 1e-12 * max(1.0, abs(rhs))


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_strict_bucketize_equals_brute_force_nearest_centroid(bits):
    d = 64
    book = cb.lloyd_max_beta(d, bits)
    c32 = book.centroids.astype(np.float32).astype(np.float64)
    t32 = (0.5 * (c32[1:] + c32[:-1]))
    u = np.random.default_rng(bits).standard_normal((5000, 8)) / np.sqrt(d)
    np.testing.assert_array_equal(oq.bucketize(u, t32), oq.nearest_centroid(u, c32))
    # Exact ties go to the lower code under both rules.
    np.testing.assert_array_equal(oq.bucketize(t32, t32), np.arange(len(t32)))
    np.testing.assert_array_equal(oq.nearest_centroid(t32, c32), np.arange(len(t32)))


def test_packing_bit_order_fixture_and_round_trip():
    codes = np.arange(8)[None, :]
    # sum_j j << 3j = 0xFAC688, little-endian bytes.
    np.testing.assert_array_equal(oq.pack_codes(codes, 3)[0], [0x88, 0xC6, 0xFA])
    np.testing.assert_array_equal(oq.pack_codes(np.array([[3, 2, 1, 0, 1, 2, 3, 0]]), 2)[0],
                                  [3 | 2 << 2 | 1 << 4, 1 | 2 << 2 | 3 << 4])
    rg = np.random.default_rng(4)
    for bits in (2, 3, 4):
        for d in (64, 128, 200):
            x = rg.integers(0, 1 << bits, (7, d))
            p = oq.pack_codes(x, bits)
            assert p.shape == (7, d * bits // 8)
            np.testing.assert_array_equal(oq.unpack_codes(p, bits, d), x)
    s = rg.random((5, 200)) < 0.5
    sp = oq.pack_signs(s)
    assert sp.shape == (5, 7) and sp.dtype == np.uint32
    np.testing.assert_array_equal(oq.unpack_signs(sp, 200), s)
    one = np.zeros((1, 64), dtype=bool)
    one[0, 33] = True
    np.testing.assert_array_equal(oq.pack_signs(one)[0], [0, 2])
    # Pad bits of the last word stay zero.
    assert (oq.pack_signs(np.ones((1, 200), dtype=bool))[0, 6] >> 8) == 0


@pytest.mark.parametrize("d,bits", [(64, 3), (128, 2), (128, 3), (128, 4)])
def test_per_coordinate_mse_matches_lloyd_max_distortion(d, bits):
    book = cb.lloyd_max_beta(d, bits)
    Pi = synth.random_rotation(d, 7)
    x = np.random.default_rng(11).standard_normal((20000, d))
    q = oq.quantize(x, Pi, book.centroids, book.boundaries, bits)
    err = (q.u - book.centroids[q.codes]) ** 2
    per_vec = err.mean(axis=1)
    se = per_vec.std(ddof=1) / math.sqrt(per_vec.size)
    assert abs(per_vec.mean() - book.mse) <= 4.0 * se, (per_vec.mean(), book.mse, se)


def test_zero_vector_reading():
    d, bits = 64, 3
    book = cb.lloyd_max_beta(d, bits)
    q = oq.quantize(np.zeros((1, d)), np.eye(d), book.centroids, book.boundaries, bits, S=np.eye(d))
    assert np.all(q.codes == (1 << (bits - 1)) - 1)
    assert q.norm[0] == 0 and q.rnorm[0] == 0 and np.all(q.signs)


def test_residual_and_signs_definition_consistency():
    d, bits = 64, 3
    book = cb.lloyd_max_beta(d, bits)
    Pi = synth.random_rotation(d, 1)
    S = synth.gaussian_projection(d, 1)
    x = np.random.default_rng(8).standard_normal((50, d))
    q = oq.quantize(x, Pi, book.centroids, book.boundaries, bits, S=S)
    # ||y|| = ||x|| (Pi orthogonal up to fp32 storage) and the residual is what is left of y.
    np.testing.assert_allclose(np.linalg.norm(q.y, axis=1), q.norm64, rtol=3e-6)
    np.testing.assert_allclose(q.y - q.r, q.norm64[:, None] * book.centroids[q.codes], atol=1e-12)
    assert np.all((q.p >= 0) == q.signs)


def _qjl_estimates(q, k, seeds, d, bits=3):
    book = cb.lloyd_max_beta(d, bits)
    Pi = synth.random_rotation(d, 0)
    est = []
    for s in seeds:
        S = synth.gaussian_projection(d, s)
        kq = oq.quantize(k[None, :], Pi, book.centroids, book.boundaries, bits, S=S)
        kp = oa.KeyPlanes(kq.idx_plane, kq.sign_plane, kq.norm64, kq.rnorm64, bits)
        q_rot = oa.rotate_query(q[None, :], Pi)
        est.append(oa.key_scores(q_rot, kp, S, book.centroids, 1.0)[0, 0])
    return np.array(est), book, Pi


def test_qjl_estimate_is_unbiased_over_projection_draws():
    d = 32
    rg = np.random.default_rng(21)
    q, k = rg.standard_normal((2, d))
    est, _, _ = _qjl_estimates(q, k, range(100, 4100), d)
    se = est.std(ddof=1) / math.sqrt(est.size)
    assert abs(est.mean() - q @ k) <= 4.0 * se, (est.mean(), q @ k, se)


def test_qjl_special_case_q_equals_residual():
    # E[sqrt(pi/2)/d ||r|| <S r, sign(S r)>] = ||r||^2.
    d = 32
    rg = np.random.default_rng(22)
    r = rg.standard_normal(d)
    vals = []
    for s in range(200, 3200):
        S = synth.gaussian_projection(d, s).astype(np.float64)
        p = S @ r
        vals.append(oa.qjl_scale(d) * np.linalg.norm(r) * (p @ np.where(p >= 0, 1.0, -1.0)))
    vals = np.array(vals)
    se = vals.std(ddof=1) / math.sqrt(vals.size)
    assert abs(vals.mean() - r @ r) <= 4.0 * se


def test_dequantized_key_is_unbiased_over_projection_draws():
    d, bits = 32, 3
    book = cb.lloyd_max_beta(d, bits)
    Pi = synth.random_rotation(d, 0)
    k = np.random.default_rng(23).standard_normal(d)
    rec = []
    for s in range(300, 2300):
        S = synth.gaussian_projection(d, s)
        kq = oq.quantize(k[None, :], Pi, book.centroids, book.boundaries, bits, S=S)
        kp = oa.KeyPlanes(kq.idx_plane, kq.sign_plane, kq.norm64, kq.rnorm64, bits)
        rec.append(oa.dequantize_keys(kp, Pi, S, book.centroids, d)[0])
    rec = np.array(rec)
    se = rec.std(axis=0, ddof=1) / math.sqrt(rec.shape[0])
    assert np.all(np.abs(rec.mean(axis=0) - k) <= 4.5 * se)
