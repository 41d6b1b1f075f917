"""The near-boundary input builder lands where it says (CPU, against the oracle).

Each code row must put the oracle's u_i at t_j + delta sigma_d and each sign
row the oracle's (S r)_i at delta ||r||, to within 1e-3 |delta| (1e-11 for
delta = 0); wide rows carry one channel four orders above the rest. The GPU
tests on these rows then probe the quantisers exactly where fp32 arithmetic
could pick a different code or sign than the fp64 definition.
"""
import numpy as np
import pytest

import synth
from oracle import codebook as ocb
from oracle import quantize as oq

from . import boundary as bd


def _book(d, bits):
    b = ocb.lloyd_max_beta(d, bits)
    c = b.centroids.astype(np.float32).astype(np.float64)
    t = (0.5 * (b.centroids[1:] + b.centroids[:-1])).astype(np.float32).astype(np.float64)
    return c, t


@pytest.mark.parametrize("d,bits", [(128, 3), (64, 3), (128, 2), (128, 4)])
def test_rows_sit_at_their_targets(d, bits):
    c, t = _book(d, bits)
    Pi = synth.random_rotation(d, 0).astype(np.float64)
    S = synth.gaussian_projection(d, 0).astype(np.float64)
    X, kind, delta, coord, target = bd.build(d, bits, Pi, S, c, t, seed=d + bits)
    assert np.array_equal(bd.to_bf16(X), X.astype(np.float64))          # bf16-exact inputs
    q = oq.quantize(X.astype(np.float64), Pi, c, t, bits, S=S)
    sigma = 1.0 / np.sqrt(d)
    code = np.where(kind == "code")[0]
    assert len(code) == len(t) * len(bd.DELTAS)
    off = (q.u[code, coord[code]] - target[code]) / sigma
    tol = np.maximum(1e-3 * np.abs(delta[code]), 1e-11)
    assert np.all(np.abs(off - delta[code]) <= tol), np.abs(off - delta[code]).max()
    sign = np.where(kind == "sign")[0]
    offs = q.p[sign, coord[sign]] / q.rnorm64[sign]
    tol = np.maximum(1e-3 * np.abs(delta[sign]), 1e-11)
    assert np.all(np.abs(offs - delta[sign]) <= tol), np.abs(offs - delta[sign]).max()
    wide = np.where(kind == "wide")[0]
    a = np.abs(X[wide])
    assert np.all(a.max(axis=1) >= 1e2 * np.median(a, axis=1))
