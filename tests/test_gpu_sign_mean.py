"""TurboESM's one-bit residual correction on the GPU against the oracle.

Keys and values of a small per-head-rotated cache (d = 64, four heads of 256
vectors, outlier channels) are quantised with S = identity, so the sign plane
holds the signs of the rotated residual coordinates; e_bar is calibrated on
separate tokens (tq_residual_mean, checked against the oracle); and
tq_dequantize_sign_mean must rebuild x_tilde = Pi^T ||x|| (c + e_bar (2s - 1))
as the oracle does from the GPU's own planes. The correction must also lower
the squared error of the plain reconstruction.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import codebook as ocb
from oracle import quantize as oq
from oracle import sign_mean as osm

from . import parity as P

pytestmark = pytest.mark.gpu
tq = pytest.importorskip("kv_cache_vector_rope_b200")


def _dev(x):
    return torch.as_tensor(np.ascontiguousarray(x), device="cuda", dtype=torch.float32)


@pytest.mark.parametrize("bits", [2, 3])
def test_sign_mean_reconstruction(bits):
    d, heads, per = 64, 4, 256
    n = heads * per
    rg = np.random.default_rng(20 + bits)
    X = rg.standard_normal((n + heads * 128, d))
    X[:, rg.choice(d, 4, replace=False)] *= 6.0
    Xb = synth.to_bf16(X.astype(np.float32))
    X64 = Xb.float().numpy().astype(np.float64)
    data, calib = X64[:n], X64[n:]
    Pis = np.stack([synth.random_rotation(d, 70 + h) for h in range(heads)])
    book = ocb.lloyd_max_beta(d, bits)
    c = book.centroids.astype(np.float32)
    t = (0.5 * (book.centroids[1:] + book.centroids[:-1])).astype(np.float32)
    # e_bar on separate calibration tokens of every head
    u = np.concatenate([tq.tq_rotate_normalize(calib[h * 128:(h + 1) * 128], Pis[h]).ravel() for h in range(heads)])
    e_bar = tq.tq_residual_mean(u, c, t, bits)
    assert abs(e_bar - osm.residual_mean_magnitude(u.astype(np.float64), c.astype(np.float64),
                                                   t.astype(np.float64))) <= 1e-12 * e_bar
    lay = tq.layout(d, bits, bits)
    planes = tq.alloc_planes(n, d, bits, True)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_quantize_kv(lay, True, Xb[:n].cuda(), planes, _dev(Pis.reshape(heads * d, d)), _dev(c), _dev(t),
                      S=_dev(np.eye(d)), vectors_per_pi=per, pi_stride=d * d, d_status=st)
    out = torch.empty((n, d), device="cuda")
    tq.tq_dequantize_sign_mean(lay, True, planes, n, _dev(Pis.reshape(heads * d, d)), _dev(c), e_bar, out,
                               vectors_per_pi=per, pi_stride=d * d)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    group = np.arange(n) // per
    ref_q = oq.quantize(data, Pis, c.astype(np.float64), t.astype(np.float64), bits, S=np.eye(d), pi_group=group)
    h = P.host_planes(planes)
    P.compare_quantized(h, ref_q, d, bits, True)          # the signs are those of the residual coordinates
    ref = np.concatenate([osm.reconstruct(h["idx"][g * per:(g + 1) * per], h["sign"][g * per:(g + 1) * per],
                                          h["norm"][g * per:(g + 1) * per], Pis[g], c, e_bar, bits, d)
                          for g in range(heads)])
    got = out.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(got, ref, atol=2e-6 * np.abs(ref).max())
    plain = np.concatenate([osm.reconstruct(h["idx"][g * per:(g + 1) * per], h["sign"][g * per:(g + 1) * per],
                                            h["norm"][g * per:(g + 1) * per], Pis[g], c, 0.0, bits, d)
                            for g in range(heads)])
    assert osm.snr_db(data, got) > osm.snr_db(data, plain) + 0.5
