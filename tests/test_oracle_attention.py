"""Pins for the oracle's attention, dequantisation, calibration and search.

* Two independent routes agree: scoring the packed planes in rotated space
  equals <q, dequantised key> in the original space (7minutos.es, Etapa 1-2:
  K_tilde = R^T c[idx] + sqrt(pi/2)/d ||eps|| S^T QJL), and accumulating V in
  rotated space then applying Pi_V^T equals attending over dequantised values
  (gist.science TurboESM section 2E: Pi^T inside the fused kernel).
* RoPE-first invariance (TurboESM section 2A): unquantised attention through
  Pi equals plain attention ("prefill cosine 1.0000").
* Softmax special cases.
* Memory arithmetic of the ESM-2 650M example (TurboESM results: 330 MB fp32).
* SVD calibration: singular basis is orthonormal, diagonalises X^T X.
* Search: exact top-k equals brute-force sort; estimated scores equal
  inner products with dequantised vectors.
"""
import json
import math
import os

import numpy as np
import pytest

import synth
from oracle import attention as oa
from oracle import calib as oc
from oracle import codebook as cb
from oracle import quantize as oq
from oracle import search as osr


def _cache(n=96, d=64, bits=3, seed=0, spikes=True):
    rg = np.random.default_rng(seed)
    K = rg.standard_normal((n, d))
    V = rg.standard_normal((n, d))
    if spikes:
        K[:, 3] *= 20
        V[:, 17] *= 20
    Pi = synth.random_rotation(d, seed)
    S = synth.gaussian_projection(d, seed)
    book = cb.lloyd_max_beta(d, bits)
    c = book.centroids.astype(np.float32)
    t = (0.5 * (c[1:].astype(np.float64) + c[:-1]))
    kq = oq.quantize(K, Pi, c, t, bits, S=S)
    vq = oq.quantize(V, Pi, c, t, bits)
    kp = oa.KeyPlanes(kq.idx_plane, kq.sign_plane, kq.norm, kq.rnorm, bits)
    vp = oa.ValuePlanes(vq.idx_plane, vq.norm, bits)
    return K, V, Pi, S, c, kp, vp


def test_scores_equal_inner_product_with_dequantised_keys():
    K, V, Pi, S, c, kp, vp = _cache()
    d = K.shape[1]
    q = np.random.default_rng(9).standard_normal((5, d))
    scale = 1.0 / math.sqrt(d)
    s1 = oa.key_scores(oa.rotate_query(q, Pi), kp, S, c, scale)
    Kt = oa.dequantize_keys(kp, Pi, S, c, d)
    # Pi is orthogonal only to float32 storage precision.
    s2 = scale * q @ Kt.T
    np.testing.assert_allclose(s1, s2, atol=2e-5 * np.abs(s2).max())
    # With an exactly orthogonal Pi the two routes agree to rounding.
    P64, _ = np.linalg.qr(np.random.default_rng(1).standard_normal((d, d)))
    s3 = oa.key_scores(oa.rotate_query(q, P64), kp, S, c, scale)
    s4 = scale * q @ oa.dequantize_keys(kp, P64, S, c, d).T
    np.testing.assert_allclose(s3, s4, atol=1e-11 * np.abs(s4).max())


def test_attention_equals_attention_over_dequantised_cache():
    K, V, _, S, c, kp, vp = _cache()
    d = K.shape[1]
    P64, _ = np.linalg.qr(np.random.default_rng(2).standard_normal((d, d)))
    q = np.random.default_rng(10).standard_normal((4, d))
    res = oa.attention(q, kp, vp, P64, P64, S, c, c)
    Kt = oa.dequantize_keys(kp, P64, S, c, d)
    Vh = oa.dequantize_values(vp, P64, c, d)
    ref = oa.plain_attention(q, Kt, Vh)
    np.testing.assert_allclose(res.out, ref, atol=1e-11 * np.abs(ref).max())
    np.testing.assert_allclose(res.probs.sum(axis=1), 1.0, atol=1e-14)


def test_rope_first_pipeline_preserves_unquantised_attention():
    # Attention computed on (Pi R q, Pi R k, Pi v) and turned back by Pi^T is plain attention.
    th = synth.tiny_head(0)
    P64, _ = np.linalg.qr(np.random.default_rng(3).standard_normal((th.d, th.d)))
    qr = oq.rope(th.Q, th.q_pos, th.rope_base)
    kr = oq.rope(th.K, th.k_pos, th.rope_base)
    ref = oa.plain_attention(qr, kr, th.V)
    rot = oa.plain_attention(qr @ P64.T, kr @ P64.T, th.V @ P64.T) @ P64
    err = np.abs(rot - ref).max() / np.abs(ref).max()
    assert err <= 1e-9, err


def test_softmax_special_cases():
    K, V, Pi, S, c, kp, vp = _cache(n=1)
    d = K.shape[1]
    q = np.random.default_rng(4).standard_normal((2, d))
    res = oa.attention(q, kp, vp, Pi, Pi, S, c, c)
    np.testing.assert_allclose(res.out, np.repeat(oa.dequantize_values(vp, Pi, c, d), 2, 0), atol=1e-12)
    # A zero query gives equal scores: the output is the mean dequantised value.
    K, V, Pi, S, c, kp, vp = _cache(n=7)
    res = oa.attention(np.zeros((1, d)), kp, vp, Pi, Pi, S, c, c)
    np.testing.assert_allclose(res.out[0], oa.dequantize_values(vp, Pi, c, d).mean(0), atol=1e-12)


def test_quantised_attention_tracks_exact_attention():
    # Not a parity pin: a sanity bound that the 3-bit + QJL cache stays close
    # to exact attention on Gaussian keys (the TurboESM pages report a mean
    # decode cosine above 0.96 on real activations). With the x20 spikes the
    # softmax is nearly one-hot and single-query cosines vary much more.
    th = synth.tiny_head(0, spike_scale=1.0, nq=16)
    d, bits = th.d, 3
    book = cb.lloyd_max_beta(d, bits)
    c = book.centroids.astype(np.float32)
    t = 0.5 * (c[1:].astype(np.float64) + c[:-1])
    kq = oq.quantize(th.K, th.Pi, c, t, bits, S=th.S, positions=th.k_pos, rope_base=th.rope_base)
    vq = oq.quantize(th.V, th.Pi, c, t, bits)
    kp = oa.KeyPlanes(kq.idx_plane, kq.sign_plane, kq.norm, kq.rnorm, bits)
    vp = oa.ValuePlanes(vq.idx_plane, vq.norm, bits)
    res = oa.attention(th.Q, kp, vp, th.Pi, th.Pi, th.S, c, c, q_positions=th.q_pos, rope_base=th.rope_base)
    ref = oa.plain_attention(oq.rope(th.Q, th.q_pos, th.rope_base), oq.rope(th.K, th.k_pos, th.rope_base), th.V)
    cos = np.sum(res.out * ref, 1) / np.linalg.norm(res.out, axis=1) / np.linalg.norm(ref, axis=1)
    assert np.all(cos > 0.9) and cos.mean() > 0.95, cos


def test_memory_arithmetic_of_the_esm2_example():
    with open(os.path.join(os.path.dirname(__file__), "golden", "turboesm_memory.json")) as f:
        g = json.load(f)
    n_vec = g["layers"] * g["heads"] * g["tokens"]
    d = g["head_dim_reading"]
    fp32 = n_vec * 2 * d * g["fp32_bytes_per_element"]
    assert round(fp32 / 2 ** 20) == g["printed_fp32_MB"]
    # This layout: K = codes + signs + ||k|| + ||r||, V = codes + ||v||.
    k_bytes = oq.row_bytes(d, 3) + 4 * oq.sign_words(d) + 4 + 4
    v_bytes = oq.row_bytes(d, 3) + 4
    assert (k_bytes, v_bytes) == (40, 28)
    ours = n_vec * (k_bytes + v_bytes)
    assert abs(fp32 / ours - 7.53) < 0.01
    # The page's 7.1x is what K and V at 36 B each give (codes + signs + one
    # scalar): 46.4 MiB, within a megabyte of the printed 47 MB.
    page = n_vec * 2 * (oq.row_bytes(d, 3) + 4 * oq.sign_words(d) + 4)
    assert abs(page / 2 ** 20 - g["printed_compressed_MB"]) < 1.0
    assert round(fp32 / page, 1) == g["printed_ratio"]


def test_svd_basis_orthonormal_and_diagonalising():
    X = np.random.default_rng(5).standard_normal((256, 64))
    X[:, 7] *= 30
    V = oc.right_singular_basis(X)
    np.testing.assert_allclose(V.T @ V, np.eye(64), atol=1e-12)
    G = (X @ V).T @ (X @ V)
    off = G - np.diag(np.diag(G))
    assert np.abs(off).max() <= 1e-9 * np.abs(G).max()
    assert np.all(np.diff(np.diag(G)) <= 1e-9 * G[0, 0])      # decreasing singular values
    for j in range(64):
        assert V[np.argmax(np.abs(V[:, j])), j] > 0
    Pi_h = oc.head_rotation(synth.random_rotation(64, 0), X)
    np.testing.assert_allclose(Pi_h.T @ Pi_h, np.eye(64), atol=3e-6)


def test_dual_codebooks_are_lloyd_fixed_points_of_their_samples():
    rg = np.random.default_rng(6)
    cK = [rg.standard_normal((64, 32)) for _ in range(3)]
    cV = [rg.standard_normal((64, 32)) * 0.5 for _ in range(3)]
    P = [synth.random_rotation(32, i).astype(np.float64) for i in range(3)]
    bk, bv = oc.dual_codebooks(cK, cV, P, P, 3)
    for book, cal in ((bk, cK), (bv, cV)):
        u = np.concatenate([oc.rotated_unit_coordinates(X, Pm) for X, Pm in zip(cal, P)])
        cell = np.searchsorted(book.boundaries, u, side="left")
        for j in range(8):
            assert abs(u[cell == j].mean() - book.centroids[j]) < 1e-13


def test_exact_top_k_matches_full_sort_and_tie_rule():
    rg = np.random.default_rng(7)
    X = rg.standard_normal((1000, 16))
    Q = rg.standard_normal((6, 16))
    got = osr.exact_top_k(Q, X, 10, block=128)
    full = np.argsort(-(Q @ X.T), axis=1, kind="stable")[:, :10]
    np.testing.assert_array_equal(got, full)
    sc = np.array([[1.0, 3.0, 3.0, 2.0, 3.0]])
    np.testing.assert_array_equal(osr.top_k(sc, 3), [[1, 2, 4]])
    assert osr.recall_at_k(np.array([[1, 2, 3]]), np.array([[3, 4, 1]])) == pytest.approx(2 / 3)


def test_estimated_search_scores_are_inner_products_with_dequantised_vectors():
    d, bits = 200, 3
    rg = np.random.default_rng(8)
    X = rg.standard_normal((300, d))
    X /= np.linalg.norm(X, axis=1, keepdims=True)
    Q = rg.standard_normal((4, d))
    P64, _ = np.linalg.qr(rg.standard_normal((d, d)))
    S = synth.gaussian_projection(d, 0)
    book = cb.lloyd_max_beta(d, bits)
    c = book.centroids.astype(np.float32)
    t = 0.5 * (c[1:].astype(np.float64) + c[:-1])
    xq = oq.quantize(X, P64, c, t, bits, S=S)
    kp = oa.KeyPlanes(xq.idx_plane, xq.sign_plane, xq.norm, xq.rnorm, bits)
    est = osr.estimated_scores(Q, kp, P64, S, c)
    ref = Q @ oa.dequantize_keys(kp, P64, S, c, d).T
    np.testing.assert_allclose(est, ref, atol=1e-11 * np.abs(ref).max())
