"""libtq.so on the host (no GPU): exports, sizes, codebook, validation.

* The shared library loads and exports every function include/tq.h declares.
* tq_make_codebook (the library's own C++ Lloyd-Max) matches the oracle's
  codebook for every (d, bits) the workloads use, analytic and empirical.
* Argument errors are rejected on the host with TQ_ERR_INVALID_ARG and a
  message, before anything is launched.
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import kv_cache_vector_rope_b200 as tq
from oracle import codebook as ocb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol():
    declared = _declared_symbols()
    assert {"tq_make_codebook", "tq_quantize_kv", "tq_decode_attention", "tq_dequantize"} <= declared
    lib = ctypes.CDLL(tq.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", tq.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (tq_[a-z0-9_]+)$", out, flags=re.M))
    assert declared <= exported, declared - exported
    assert declared == set(tq.exported_symbols()) | (declared - set(tq.exported_symbols()))
    assert "sm_100a" in tq.tq_version()


def test_layout_sizes():
    assert tq.tq_idx_row_bytes(128, 3) == 48 and tq.tq_idx_row_bytes(64, 3) == 24
    assert tq.tq_idx_row_bytes(200, 3) == 75 and tq.tq_idx_row_bytes(128, 2) == 32
    assert tq.tq_sign_words(128) == 4 and tq.tq_sign_words(200) == 7 and tq.tq_sign_words(64) == 2
    lay = tq.layout(128, 3, 3)
    assert tq.tq_packed_bytes(lay, 1, True) == 48 + 16 + 4 + 4
    assert tq.tq_packed_bytes(lay, 1, False) == 48 + 4
    assert tq.tq_packed_bytes(tq.layout(64, 3, 3), 10, True) == 400
    assert tq.tq_packed_bytes(tq.layout(7, 3, 3), 1, True) == -1


@pytest.mark.parametrize("d", [64, 128, 200])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_host_codebook_matches_oracle(d, bits):
    c, t, mse = tq.tq_make_codebook(d, bits, 0)
    ref = ocb.lloyd_max_beta(d, bits)
    # Two independent quadratures; both converge to 1e-13 in the level.
    np.testing.assert_allclose(c.astype(np.float64), ref.centroids, rtol=0, atol=2e-7 / np.sqrt(d))
    np.testing.assert_allclose(t.astype(np.float64), ref.boundaries, rtol=0, atol=2e-7 / np.sqrt(d))
    assert abs(mse - ref.mse) < 1e-9 * ref.mse
    assert np.all(np.diff(c) > 0) and np.all(np.diff(t) > 0)
    assert np.array_equal(c, -c[::-1])


def test_host_codebook_d3_closed_form():
    c, t, mse = tq.tq_make_codebook(3, 3, 0)
    np.testing.assert_allclose(c, -1.0 + (2.0 * np.arange(8) + 1.0) / 8, atol=1e-7)
    assert abs(mse - 1.0 / 192.0) < 1e-12


def test_host_empirical_codebook_matches_oracle():
    rg = np.random.default_rng(3)
    x = (rg.standard_normal(200000) * 0.1).astype(np.float32)
    x[:1000] *= 8.0
    c, t, mse = tq.tq_make_codebook(0, 3, 1, x)
    ref = ocb.lloyd_empirical(x.astype(np.float64), 3)
    np.testing.assert_allclose(c, ref.centroids, rtol=2e-7, atol=1e-9)
    assert abs(mse - ref.mse) < 1e-9


def test_host_empirical_codebook_worked_example_fixed_point():
    # The 1-bit worked example of the TurboQuant Lloyd-Max section (quantile start).
    c, t, mse = tq.tq_make_codebook(0, 1, 1, np.array([1.42, -0.85, 2.31, 0.97], dtype=np.float32))
    ref = ocb.lloyd_empirical(np.array([1.42, -0.85, 2.31, 0.97], dtype=np.float32).astype(np.float64), 1)
    np.testing.assert_allclose(c, ref.centroids, rtol=1e-6)


def test_codebook_argument_errors():
    with pytest.raises(tq.TQError) as e:
        tq.tq_make_codebook(64, 5, 0)
    assert e.value.status == tq.TQ_ERR_INVALID_ARG
    with pytest.raises(tq.TQError):
        tq.tq_make_codebook(2, 3, 0)
    with pytest.raises(tq.TQError):
        tq.tq_make_codebook(64, 3, 1, None)
    with pytest.raises(tq.TQError):
        tq.tq_make_codebook(64, 3, 7)
    with pytest.raises(tq.TQError):
        tq.tq_make_codebook(0, 2, 1, np.array([0.0, np.nan, 1.0, 2.0, 3.0], dtype=np.float32))


def _raw_quantize(lay, is_key=1, x=0x1000, n=4, row_stride=128, Pi=0x2000, vpp=1, pis=0, S=0x3000,
                  c=0x4000, t=0x5000, planes=None):
    planes = planes or tq._Planes(0x6000, 0x7000, 0x8000, 0x9000)
    return tq._lib.tq_quantize_kv(ctypes.byref(lay), is_key, x, 0, n, row_stride, None, 0.0, Pi, vpp, pis, S, c, t,
                                  ctypes.byref(planes), None, None)


def test_quantize_host_validation():
    bad = tq.layout(100, 3, 3)
    assert _raw_quantize(bad) == tq.TQ_ERR_INVALID_ARG
    assert "multiple of 8" in tq.tq_last_error_string()
    assert _raw_quantize(tq.layout(128, 5, 3)) == tq.TQ_ERR_INVALID_ARG
    lay = tq.layout(128, 3, 3)
    assert _raw_quantize(lay, n=-1) == tq.TQ_ERR_INVALID_ARG
    assert _raw_quantize(lay, n=0) == tq.TQ_OK           # nothing to do, nothing launched
    assert _raw_quantize(lay, row_stride=64) == tq.TQ_ERR_INVALID_ARG
    assert _raw_quantize(lay, S=0) == tq.TQ_ERR_INVALID_ARG
    assert _raw_quantize(lay, x=0) == tq.TQ_ERR_INVALID_ARG
    assert _raw_quantize(lay, Pi=0x2004) == tq.TQ_ERR_INVALID_ARG   # misaligned
    assert _raw_quantize(lay, pis=-4) == tq.TQ_ERR_INVALID_ARG
    assert _raw_quantize(lay, pis=16384, vpp=0) == tq.TQ_ERR_INVALID_ARG
    assert _raw_quantize(lay, is_key=1, planes=tq._Planes(0x6000, 0, 0x8000, 0x9000)) == tq.TQ_ERR_INVALID_ARG


def _raw_append(lay, is_key=1, x=0x1000, n=4, row_stride=128, Pi=0x2000, S=0x3000, ctx_stride=100, slot=7,
                planes=None):
    planes = planes or tq._Planes(0x6000, 0x7000, 0x8000, 0x9000)
    return tq._lib.tq_append_kv(ctypes.byref(lay), is_key, x, 0, n, row_stride, None, 0.0, Pi, S, 0x4000, 0x5000,
                                ctypes.byref(planes), ctx_stride, slot, None, None)


def test_append_host_validation():
    lay = tq.layout(128, 3, 3)
    assert _raw_append(lay, n=0) == tq.TQ_OK             # nothing to do, nothing launched
    assert _raw_append(lay, n=-1) == tq.TQ_ERR_INVALID_ARG
    assert _raw_append(lay, slot=100) == tq.TQ_ERR_INVALID_ARG      # slot must be < ctx_stride
    assert "slot" in tq.tq_last_error_string()
    assert _raw_append(lay, slot=-1) == tq.TQ_ERR_INVALID_ARG
    assert _raw_append(lay, ctx_stride=0, slot=0) == tq.TQ_ERR_INVALID_ARG
    assert _raw_append(lay, S=0) == tq.TQ_ERR_INVALID_ARG
    assert _raw_append(lay, row_stride=100) == tq.TQ_ERR_INVALID_ARG
    assert _raw_append(lay, Pi=0x2004) == tq.TQ_ERR_INVALID_ARG
    assert _raw_append(tq.layout(96, 3, 3), row_stride=96) == tq.TQ_ERR_UNSUPPORTED


def _raw_decode(lay, hq=32, hkv=8, nq=1, n_ctx=1024, ctx_stride=0, ws=0x10000, ws_bytes=1 << 30, kp=None):
    kp = kp or tq._Planes(0x1000, 0x2000, 0x3000, 0x4000)
    vp = tq._Planes(0x5000, 0, 0x6000, 0)
    return tq._lib.tq_decode_attention(ctypes.byref(lay), 0x100, 1, 1, hq, hkv, nq, n_ctx, ctx_stride, None, 0.0,
                                       ctypes.byref(kp), ctypes.byref(vp), 0x7000, 0x8000, 0, 0x9000, 0xa000, 0xb000,
                                       0.1, 0xc000, 0, None, ws, ws_bytes, None, None)


def test_decode_host_validation():
    lay = tq.layout(128, 3, 3)
    assert _raw_decode(lay, hq=30) == tq.TQ_ERR_INVALID_ARG          # hq not a multiple of hkv
    assert _raw_decode(lay, n_ctx=0) == tq.TQ_ERR_INVALID_ARG
    assert "empty" in tq.tq_last_error_string()
    assert _raw_decode(lay, ctx_stride=100) == tq.TQ_ERR_INVALID_ARG
    assert _raw_decode(lay, ws_bytes=16) == tq.TQ_ERR_WORKSPACE
    assert _raw_decode(lay, ws=0x10010) == tq.TQ_ERR_INVALID_ARG      # workspace alignment
    assert _raw_decode(lay, kp=tq._Planes(0x1001, 0x2000, 0x3000, 0x4000)) == tq.TQ_ERR_INVALID_ARG
    assert _raw_decode(lay, kp=tq._Planes(0x1000, 0, 0x3000, 0x4000)) == tq.TQ_ERR_INVALID_ARG
    need = tq.tq_decode_workspace_bytes(lay, 1, 32, 8, 1, 1024)
    assert need > 0 and tq.tq_decode_workspace_bytes(tq.layout(128, 3, 3), 1, 32, 8, 1, 0) == 0


def test_dequantize_host_validation():
    lay = tq.layout(128, 3, 3)
    p = tq._Planes(0x1000, 0x2000, 0x3000, 0x4000)
    f = tq._lib.tq_dequantize
    assert f(ctypes.byref(lay), 1, 10, ctypes.byref(p), 0x5000, 1, 0, None, 0x6000, 0x7000, 0, 128, None) \
        == tq.TQ_ERR_INVALID_ARG     # keys need S
    assert f(ctypes.byref(lay), 0, 10, ctypes.byref(p), 0x5000, 1, 0, None, 0x6000, 0x7000, 0, 64, None) \
        == tq.TQ_ERR_INVALID_ARG     # out_stride < d
    assert f(ctypes.byref(lay), 0, 0, ctypes.byref(p), 0x5000, 1, 0, None, 0x6000, 0x7000, 0, 128, None) == tq.TQ_OK


def test_fit_rotation_matches_oracle_svd_basis():
    from oracle import calib as oc
    import synth
    rg = np.random.default_rng(41)
    for d in (64, 128):
        X = rg.standard_normal((256, d))
        X[:, rg.choice(d, 4, replace=False)] *= rg.lognormal(2.0, 1.0, 4)
        X32 = X.astype(np.float32)
        Pr = synth.random_rotation(d, 5)
        got = tq.tq_fit_rotation(X32, Pr)
        ref = oc.head_rotation(Pr, X32.astype(np.float64))
        np.testing.assert_allclose(got, ref, atol=2e-6)
        np.testing.assert_allclose(got.astype(np.float64).T @ got, np.eye(d), atol=5e-6)


def test_rotate_normalize_matches_oracle_and_skips_zero_rows():
    from oracle import calib as oc
    import synth
    rg = np.random.default_rng(42)
    X = rg.standard_normal((50, 64)).astype(np.float32)
    X[7] = 0.0
    P = synth.random_rotation(64, 1)
    got = tq.tq_rotate_normalize(X, P)
    assert got.shape == (49, 64)
    ref = oc.rotated_unit_coordinates(X.astype(np.float64), P).reshape(-1, 64)
    np.testing.assert_allclose(got, ref, atol=1e-7)


def test_calibration_argument_errors():
    with pytest.raises(tq.TQError):
        tq.tq_fit_rotation(np.zeros((0, 64), np.float32), np.eye(64, dtype=np.float32))
    with pytest.raises(tq.TQError):
        tq.tq_fit_rotation(np.full((4, 64), np.nan, np.float32), np.eye(64, dtype=np.float32))


def test_residual_mean_matches_oracle_and_validates():
    from oracle import sign_mean as osm
    b = ocb.lloyd_max_beta(64, 3)
    c = b.centroids.astype(np.float32)
    t = (0.5 * (b.centroids[1:] + b.centroids[:-1])).astype(np.float32)
    u = (np.random.default_rng(8).standard_normal(50000) / 8).astype(np.float32)
    u[:7] = t[:7]                                        # ties take the lower code on both sides
    e = tq.tq_residual_mean(u, c, t, 3)
    ref = osm.residual_mean_magnitude(u.astype(np.float64), c.astype(np.float64), t.astype(np.float64))
    assert abs(e - ref) <= 1e-12 * ref
    with pytest.raises(tq.TQError):
        tq.tq_residual_mean(u, c, t[::-1].copy(), 3)     # boundaries must increase
    with pytest.raises(tq.TQError):
        tq.tq_residual_mean(u[:0], c, t, 3)


def test_search_merge_host_validation():
    f = tq._lib.tq_search_merge_topk
    p = 0x1000
    assert f(0, 10, p, p, 0, p, p, 0, p, p, None) == tq.TQ_OK              # nothing to merge
    assert f(4, 33, p, p, 0, p, p, 0, p, p, None) == tq.TQ_ERR_INVALID_ARG  # k above 32
    assert f(4, 0, p, p, 0, p, p, 0, p, p, None) == tq.TQ_ERR_INVALID_ARG
    assert f(4, 10, p, p, -1, p, p, 0, p, p, None) == tq.TQ_ERR_INVALID_ARG
    assert f(4, 10, 0, p, 0, p, p, 0, p, p, None) == tq.TQ_ERR_INVALID_ARG
    lay = tq.layout(128, 3, 3)
    one = tq._lib.tq_search_workspace_bytes(ctypes.byref(lay), 1, 100000, 10)
    many = tq._lib.tq_search_workspace_bytes(ctypes.byref(lay), 100000, 100000, 10)
    cap = tq._lib.tq_search_workspace_bytes(ctypes.byref(lay), 16384, 100000, 10)
    assert 0 < one < cap == many                       # one pass holds at most 16,384 queries
