"""Every decode kernel family against the oracle, and the bounded-wait path.

Decode: d=128, GQA group 8, one and two queries per head, value bits 2, 3
and 4, with TQ_DECODE_PATH unset, "v1" (the general CUDA-core kernel) and "v2"
(the table kernel for 3-bit values). Group 8 is outside the tensor-core
decode (group 4, one query, 3-bit values; its own tests are elsewhere), so
these cases pin the CUDA-core kernels that serve every other shape.

Bounded waits: with TQ_TEST_WAIT_NS=0 the pipeline waits of both tensor-core
kernels give up at their first unmet wait; the call must come back with
TQ_DEV_TIMEOUT in the device status (no fault, no hang), and the next call with
the normal limit must reproduce the earlier results bit for bit.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import attention as oa
from oracle import codebook as ocb

from . import parity as P

pytestmark = pytest.mark.gpu
tq = pytest.importorskip("kv_cache_vector_rope_b200")


def _book(d, bits):
    b = ocb.lloyd_max_beta(d, bits)
    return (b.centroids.astype(np.float32), (0.5 * (b.centroids[1:] + b.centroids[:-1])).astype(np.float32))


def _dev(x):
    return torch.as_tensor(np.ascontiguousarray(x), device="cuda", dtype=torch.float32)


def _cache(seed, b, hkv, n, d, kbits, vbits):
    rg = np.random.default_rng(seed)
    K = rg.standard_normal((b * hkv * n, d))
    V = rg.standard_normal((b * hkv * n, d))
    ch = rg.choice(d, 3, replace=False)
    K[:, ch] *= 10.0
    V[:, ch] *= 10.0
    Kb = synth.to_bf16(K.astype(np.float32)).cuda()
    Vb = synth.to_bf16(V.astype(np.float32)).cuda()
    Pi = synth.random_rotation(d, seed)
    S = synth.gaussian_projection(d, seed)
    (cK, tK), (cV, tV) = _book(d, kbits), _book(d, vbits)
    lay = tq.layout(d, kbits, vbits)
    kp = tq.alloc_planes(Kb.shape[0], d, kbits, True)
    vp = tq.alloc_planes(Vb.shape[0], d, vbits, False)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_quantize_kv(lay, True, Kb, kp, _dev(Pi), _dev(cK), _dev(tK), S=_dev(S), d_status=st)
    tq.tq_quantize_kv(lay, False, Vb, vp, _dev(Pi), _dev(cV), _dev(tV), d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return lay, kp, vp, Pi, S, cK, cV


@pytest.mark.parametrize("vbits", [2, 3, 4])
@pytest.mark.parametrize("nq", [1, 2])
@pytest.mark.parametrize("path", [None, "v1", "v2"])
def test_decode_paths_gqa8(vbits, nq, path, monkeypatch):
    b, hkv, G, n, d, kbits = 2, 2, 8, 777, 128, 3
    hq = hkv * G
    if path is None:
        monkeypatch.delenv("TQ_DECODE_PATH", raising=False)
    else:
        monkeypatch.setenv("TQ_DECODE_PATH", path)
    lay, kp, vp, Pi, S, cK, cV = _cache(vbits, b, hkv, n, d, kbits, vbits)
    Q = synth.to_bf16(np.random.default_rng(9).standard_normal((b, hq, nq, d)).astype(np.float32))
    out = torch.empty((b, hq, nq, d), dtype=torch.float32, device="cuda")
    scores = torch.empty((b, hq, nq, n), device="cuda")
    ws = tq.decode_workspace(lay, b, hq, hkv, nq, n)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_decode_attention(lay, Q.cuda(), kp, vp, hkv, n, _dev(Pi), _dev(Pi), _dev(S), _dev(cK), _dev(cV), out, ws,
                           scores_out=scores, d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    hk, hv = P.host_planes(kp), P.host_planes(vp)
    Qn = Q.float().numpy().astype(np.float64)
    for bi in range(b):
        for kv in range(hkv):
            rows = slice((bi * hkv + kv) * n, (bi * hkv + kv + 1) * n)
            kpl = P.key_planes({k: v[rows] for k, v in hk.items()}, kbits)
            vpl = P.value_planes({k: v[rows] for k, v in hv.items()}, vbits)
            for h in range(kv * G, (kv + 1) * G):
                ref = oa.attention(Qn[bi, h], kpl, vpl, Pi, Pi, S, cK, cV)
                P.check_scores(scores[bi, h].cpu().numpy(), ref.scores, np.linalg.norm(Qn[bi, h], axis=1),
                               hk["norm"][rows], d)
                P.check_out(out[bi, h], ref.out)


def test_bounded_wait_timeout_is_reported_and_the_next_call_is_exact(monkeypatch):
    b, hkv, G, n, d = 1, 2, 4, 4096, 128
    hq = hkv * G
    monkeypatch.delenv("TQ_TEST_WAIT_NS", raising=False)
    monkeypatch.delenv("TQ_DECODE_PATH", raising=False)
    monkeypatch.delenv("TQ_QUANTIZE_PATH", raising=False)
    rg = np.random.default_rng(3)
    K = synth.to_bf16(rg.standard_normal((b * hkv * n, d)).astype(np.float32)).cuda()
    V = synth.to_bf16(rg.standard_normal((b * hkv * n, d)).astype(np.float32)).cuda()
    Pi, S = _dev(synth.random_rotation(d, 3)), _dev(synth.gaussian_projection(d, 3))
    c, t = (_dev(x) for x in _book(d, 3))
    lay = tq.layout(d, 3, 3)
    q = torch.randn((b, hq, 1, d), device="cuda")
    ws = tq.decode_workspace(lay, b, hq, hkv, 1, n)

    def run(kp, vp, out):
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        tq.tq_quantize_kv(lay, True, K, kp, Pi, c, t, S=S, d_status=st)
        tq.tq_quantize_kv(lay, False, V, vp, Pi, c, t, d_status=st)
        tq.tq_decode_attention(lay, q, kp, vp, hkv, n, Pi, Pi, S, c, c, out, ws, d_status=st)
        torch.cuda.synchronize()
        return int(st.item())

    def fresh():
        return (tq.alloc_planes(K.shape[0], d, 3, True), tq.alloc_planes(V.shape[0], d, 3, False),
                torch.empty((b, hq, 1, d), device="cuda"))

    kp0, vp0, out0 = fresh()
    assert run(kp0, vp0, out0) == 0
    # Each kernel alone with the short limit: the key quantiser, then decode
    # over a good cache.
    monkeypatch.setenv("TQ_TEST_WAIT_NS", "0")
    seen_q = seen_d = False
    for _ in range(10):
        kp1, _, _ = fresh()
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        tq.tq_quantize_kv(lay, True, K, kp1, Pi, c, t, S=S, d_status=st)
        torch.cuda.synchronize()
        seen_q |= bool(int(st.item()) & tq.TQ_DEV_TIMEOUT)
        out1 = torch.empty_like(out0)
        st.zero_()
        tq.tq_decode_attention(lay, q, kp0, vp0, hkv, n, Pi, Pi, S, c, c, out1, ws, d_status=st)
        torch.cuda.synchronize()
        seen_d |= bool(int(st.item()) & tq.TQ_DEV_TIMEOUT)
        if seen_q and seen_d:
            break
    assert seen_q and seen_d, (seen_q, seen_d)
    # Back to the normal limit: the same results, bit for bit.
    monkeypatch.delenv("TQ_TEST_WAIT_NS")
    kp2, vp2, out2 = fresh()
    assert run(kp2, vp2, out2) == 0
    for a0, a2 in ((kp0.idx, kp2.idx), (kp0.sign, kp2.sign), (kp0.norm, kp2.norm), (kp0.rnorm, kp2.rnorm),
                   (vp0.idx, vp2.idx), (vp0.norm, vp2.norm)):
        assert torch.equal(a0, a2)
    assert torch.equal(out0, out2)
