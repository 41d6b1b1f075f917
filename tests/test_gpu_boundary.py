"""The quantisers on inputs built at and beside their decision points.

Rows from tests/boundary.py put a rotated coordinate at t_j + delta sigma_d or
a projected residual at delta ||r|| (delta in {0, +-1e-9, +-1e-7, +-1e-6,
+-2e-6}), plus rows with one channel x1e4. The tensor-core quantiser (bf16
input), the CUDA-core quantiser (bf16 and fp32 input) and the exact per-vector
kernel that small calls use (bf16 input) must reproduce the
oracle's codes and signs exactly: their guard bands send every such row to
the fp64 fixup; the exact per-vector kernel (small calls) decides everything in
fp64. The only differences allowed are where the oracle's own fp64
value is within 1e-12 (sigma_d for codes, ||r|| for signs) of the decision
point, below the resolution two fp64 summation orders can agree on.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import codebook as ocb
from oracle import quantize as oq

from . import boundary as bd
from . import parity as P

pytestmark = pytest.mark.gpu
tq = pytest.importorskip("kv_cache_vector_rope_b200")

FP64_RES = 1e-12


def _book(d, bits):
    b = ocb.lloyd_max_beta(d, bits)
    c = b.centroids.astype(np.float32)
    t = (0.5 * (b.centroids[1:] + b.centroids[:-1])).astype(np.float32)
    return c, t


def _dev(x):
    return torch.as_tensor(np.ascontiguousarray(x), device="cuda", dtype=torch.float32)


@pytest.mark.parametrize("d,bits", [(128, 3), (64, 3), (128, 2), (128, 4)])
@pytest.mark.parametrize("path", ["tensor-core", "cuda-core-bf16", "cuda-core-fp32", "exact-bf16"])
def test_quantizers_exact_at_decision_points(d, bits, path, monkeypatch):
    c, t = _book(d, bits)
    Pi = synth.random_rotation(d, 0)
    S = synth.gaussian_projection(d, 0)
    X, kind, delta, coord, target = bd.build(d, bits, Pi.astype(np.float64), S.astype(np.float64),
                                             c.astype(np.float64), t.astype(np.float64), seed=d + bits)
    X = np.concatenate([X, X[:37]])                   # several tiles' worth plus a ragged tail
    if path == "tensor-core":
        monkeypatch.setenv("TQ_QUANTIZE_PATH", "tensor-core")
    elif path.startswith("exact"):
        monkeypatch.delenv("TQ_QUANTIZE_PATH", raising=False)     # a small call: the exact per-vector kernel
    else:
        monkeypatch.setenv("TQ_QUANTIZE_PATH", "cuda-core")
    x = torch.as_tensor(X, device="cuda")
    x = x.float() if path.endswith("fp32") else x.to(torch.bfloat16)
    lay = tq.layout(d, bits, bits)
    sigma = 1.0 / np.sqrt(d)
    worst = {}
    for is_key in (True, False):
        ref = oq.quantize(X.astype(np.float64), Pi, c.astype(np.float64), t.astype(np.float64), bits,
                          S=S if is_key else None)
        planes = tq.alloc_planes(X.shape[0], d, bits, is_key)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        tq.tq_quantize_kv(lay, is_key, x, planes, _dev(Pi), _dev(c), _dev(t), S=_dev(S) if is_key else None,
                          d_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        h = P.host_planes(planes)
        codes = oq.unpack_codes(h["idx"], bits, d)
        diff = codes != ref.codes
        allowed = ref.code_margin <= FP64_RES * sigma
        assert not (diff & ~allowed).any(), (path, is_key, np.argwhere(diff & ~allowed)[:5])
        np.testing.assert_allclose(h["norm"], ref.norm64, rtol=P.NORM_RTOL)
        worst["codes_differing"] = worst.get("codes_differing", 0) + int(diff.sum())
        if is_key:
            signs = oq.unpack_signs(h["sign"], d)
            sd = signs != ref.signs
            near = np.abs(ref.p) <= FP64_RES * ref.rnorm64[:, None]
            ok = sd & (near | diff.any(axis=1)[:, None])
            assert not (sd & ~ok).any(), (path, np.argwhere(sd & ~ok)[:5])
            worst["signs_differing"] = int(sd.sum())
            keep = ~diff.any(axis=1) & (ref.rnorm64 > 0)
            rn = np.abs(h["rnorm"][keep].astype(np.float64) - ref.rnorm64[keep]) / ref.rnorm64[keep]
            assert rn.max() <= P.RNORM_RTOL
    print(f"{path} d={d} bits={bits}: {worst}")
