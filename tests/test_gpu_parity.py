"""GPU parity: the CUDA library against the oracle, through the C ABI.

Rules are in tests/parity.py. Sizes span several tiles plus a ragged tail
(quantize tiles 32 vectors, decode tiles 128 tokens), the tiny RoPE head, a
Llama-shaped GQA slice at 2/3/4 key bits, edge cases, and the full-size
Llama-shaped layer (sampled) in the launch configuration the benchmark uses.
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import attention as oa
from oracle import codebook as ocb
from oracle import quantize as oq

from . import parity as P

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("kv_cache_vector_rope_b200")

_BOOKS = {}


def book(d, bits):
    key = (d, bits)
    if key not in _BOOKS:
        b = ocb.lloyd_max_beta(d, bits)
        c32 = b.centroids.astype(np.float32)
        t32 = (0.5 * (b.centroids[1:] + b.centroids[:-1])).astype(np.float32)
        _BOOKS[key] = (c32, t32)
    return _BOOKS[key]


def dev(x, dtype=torch.float32):
    return torch.as_tensor(np.ascontiguousarray(x), device="cuda").to(dtype)


def quantize_gpu(x_dev, d, bits, is_key, Pi, S=None, positions=None, rope_base=0.0, vpp=1, pi_stride=0):
    lay = tq.layout(d, bits, bits)
    n = x_dev.shape[0]
    c, t = book(d, bits)
    planes = tq.alloc_planes(n, d, bits, is_key)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_quantize_kv(lay, is_key, x_dev, planes, dev(Pi), dev(c), dev(t), S=None if S is None else dev(S),
                      positions=positions, rope_base=rope_base, vectors_per_pi=vpp, pi_stride=pi_stride, d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return planes


def quantize_ref(x_np, d, bits, is_key, Pi, S=None, positions=None, rope_base=0.0, pi_group=None):
    c, t = book(d, bits)
    return oq.quantize(x_np, Pi, c.astype(np.float64), t.astype(np.float64), bits, S=S if is_key else None,
                       positions=positions, rope_base=rope_base, pi_group=pi_group)


# ---------------------------------------------------------------------------
# Workload 1: tiny single head with RoPE (full size).
# ---------------------------------------------------------------------------
@pytest.fixture(scope="module")
def tiny():
    th = synth.tiny_head(0)
    d = th.d
    kpos = torch.as_tensor(th.k_pos, device="cuda")
    kp = quantize_gpu(dev(th.K), d, 3, True, th.Pi, th.S, positions=kpos, rope_base=th.rope_base)
    vp = quantize_gpu(dev(th.V), d, 3, False, th.Pi)
    return th, kp, vp


def test_tiny_head_quantize_parity(tiny):
    th, kp, vp = tiny
    rk = quantize_ref(th.K, th.d, 3, True, th.Pi, th.S, positions=th.k_pos, rope_base=th.rope_base)
    rv = quantize_ref(th.V, th.d, 3, False, th.Pi)
    sk = P.compare_quantized(P.host_planes(kp), rk, th.d, 3, True)
    sv = P.compare_quantized(P.host_planes(vp), rv, th.d, 3, False)
    assert sk["excused_codes"] + sk["excused_signs"] + sv["excused_codes"] == 0


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_tiny_head_decode_parity(tiny, out_dtype):
    th, kp, vp = tiny
    d, n, nq = th.d, th.K.shape[0], th.Q.shape[0]
    lay = tq.layout(d, 3, 3)
    c, _ = book(d, 3)
    q = dev(th.Q).reshape(1, 1, nq, d)
    qpos = torch.as_tensor(th.q_pos, device="cuda")
    out = torch.empty((1, 1, nq, d), dtype=out_dtype, device="cuda")
    scores = torch.empty((1, 1, nq, n), dtype=torch.float32, device="cuda")
    ws = tq.decode_workspace(lay, 1, 1, 1, nq, n)
    tq.tq_decode_attention(lay, q, kp, vp, 1, n, dev(th.Pi), dev(th.Pi), dev(th.S), dev(c), dev(c), out, ws,
                           q_positions=qpos, rope_base=th.rope_base, scores_out=scores)
    torch.cuda.synchronize()
    hk, hv = P.host_planes(kp), P.host_planes(vp)
    ref = oa.attention(th.Q, P.key_planes(hk, 3), P.value_planes(hv, 3), th.Pi, th.Pi, th.S, c, c,
                       q_positions=th.q_pos, rope_base=th.rope_base)
    P.check_scores(scores.cpu().numpy()[0, 0], ref.scores, np.linalg.norm(th.Q, axis=1), hk["norm"], d)
    P.check_out(out[0, 0], ref.out)


def test_tiny_head_dequantize_parity(tiny):
    th, kp, vp = tiny
    d, n = th.d, th.K.shape[0]
    lay = tq.layout(d, 3, 3)
    c, _ = book(d, 3)
    outk = torch.empty((n, d), device="cuda")
    outv = torch.empty((n, d), device="cuda")
    tq.tq_dequantize(lay, True, kp, n, dev(th.Pi), dev(c), outk, S=dev(th.S))
    tq.tq_dequantize(lay, False, vp, n, dev(th.Pi), dev(c), outv)
    torch.cuda.synchronize()
    hk, hv = P.host_planes(kp), P.host_planes(vp)
    refk = oa.dequantize_keys(P.key_planes(hk, 3), th.Pi, th.S, c, d)
    refv = oa.dequantize_values(P.value_planes(hv, 3), th.Pi, c, d)
    scale = np.abs(refk).max()
    np.testing.assert_allclose(outk.cpu().numpy(), refk, atol=1e-5 * scale)
    np.testing.assert_allclose(outv.cpu().numpy(), refv, atol=1e-5 * np.abs(refv).max())


# ---------------------------------------------------------------------------
# Llama-shaped GQA slice: several tiles + ragged tails, 2/3/4 key bits.
# ---------------------------------------------------------------------------
def _llama_slice(seed, b, hkv, n, d=128):
    rg = np.random.default_rng(seed)
    K = rg.standard_normal((b, hkv, n, d))
    V = rg.standard_normal((b, hkv, n, d))
    for h in range(hkv):
        ch = rg.choice(d, 3, replace=False)
        K[:, h, :, ch] *= 10.0
        V[:, h, :, ch] *= 10.0
    Kb = synth.to_bf16(K.astype(np.float32))
    Vb = synth.to_bf16(V.astype(np.float32))
    return Kb, Vb


@pytest.mark.parametrize("kbits", [2, 3, 4])
def test_llama_slice_quantize_and_decode(kbits):
    b, hkv, hq, n, d = 2, 2, 8, 1000, 128
    Kb, Vb = _llama_slice(kbits, b, hkv, n, d)
    Pi = synth.random_rotation(d, 0)
    S = synth.gaussian_projection(d, 0)
    kp = quantize_gpu(Kb.reshape(-1, d).cuda(), d, kbits, True, Pi, S)
    vp = quantize_gpu(Vb.reshape(-1, d).cuda(), d, 3, False, Pi)
    K64 = Kb.float().numpy().reshape(-1, d).astype(np.float64)
    V64 = Vb.float().numpy().reshape(-1, d).astype(np.float64)
    hk, hv = P.host_planes(kp), P.host_planes(vp)
    P.compare_quantized(hk, quantize_ref(K64, d, kbits, True, Pi, S), d, kbits, True)
    P.compare_quantized(hv, quantize_ref(V64, d, 3, False, Pi), d, 3, False)

    lay = tq.layout(d, kbits, 3)
    cK, _ = book(d, kbits)
    cV, _ = book(d, 3)
    Q = synth.to_bf16(np.random.default_rng(7).standard_normal((b, hq, 1, d)).astype(np.float32))
    out = torch.empty((b, hq, 1, d), dtype=torch.bfloat16, device="cuda")
    scores = torch.empty((b, hq, 1, n), device="cuda")
    ws = tq.decode_workspace(lay, b, hq, hkv, 1, n)
    tq.tq_decode_attention(lay, Q.cuda(), kp, vp, hkv, n, dev(Pi), dev(Pi), dev(S), dev(cK), dev(cV), out, ws,
                           scores_out=scores)
    torch.cuda.synchronize()
    Qn = Q.float().numpy().astype(np.float64)
    G = hq // hkv
    for bi in range(b):
        for kv in range(hkv):
            rows = slice((bi * hkv + kv) * n, (bi * hkv + kv + 1) * n)
            kpl = oa.KeyPlanes(hk["idx"][rows], hk["sign"][rows], hk["norm"][rows], hk["rnorm"][rows], kbits)
            vpl = oa.ValuePlanes(hv["idx"][rows], hv["norm"][rows], 3)
            qs = Qn[bi, kv * G:(kv + 1) * G, 0]
            ref = oa.attention(qs, kpl, vpl, Pi, Pi, S, cK, cV)
            P.check_scores(scores[bi, kv * G:(kv + 1) * G, 0].cpu().numpy(), ref.scores,
                           np.linalg.norm(qs, axis=1), hk["norm"][rows], d)
            P.check_out(out[bi, kv * G:(kv + 1) * G, 0], ref.out)


# ---------------------------------------------------------------------------
# Edge cases.
# ---------------------------------------------------------------------------
def test_edge_zero_vectors_single_token_and_ragged_rows():
    d = 64
    Pi = synth.random_rotation(d, 1)
    S = synth.gaussian_projection(d, 1)
    rg = np.random.default_rng(11)
    X = rg.standard_normal((37, d)).astype(np.float32)     # ragged quantize tile (32 + 5)
    X[3] = 0.0
    X[36] = 0.0
    kp = quantize_gpu(dev(X), d, 3, True, Pi, S)
    vp = quantize_gpu(dev(X), d, 3, False, Pi)
    P.compare_quantized(P.host_planes(kp), quantize_ref(X, d, 3, True, Pi, S), d, 3, True)
    P.compare_quantized(P.host_planes(vp), quantize_ref(X, d, 3, False, Pi), d, 3, False)
    # n_ctx = 1: the output is the single dequantised value.
    lay = tq.layout(d, 3, 3)
    c, _ = book(d, 3)
    q = dev(rg.standard_normal((1, 1, 1, d)))
    out = torch.empty((1, 1, 1, d), device="cuda")
    ws = tq.decode_workspace(lay, 1, 1, 1, 1, 1)
    tq.tq_decode_attention(lay, q, kp.rows(0, 1), vp.rows(0, 1), 1, 1, dev(Pi), dev(Pi), dev(S), dev(c), dev(c),
                           out, ws)
    torch.cuda.synchronize()
    hv = P.host_planes(vp.rows(0, 1))
    P.check_out(out[0, 0], oa.dequantize_values(P.value_planes(hv, 3), Pi, c, d))


def test_edge_ctx_stride_and_zero_query():
    # Two streams stored with capacity 300 but only 257 valid tokens (garbage after).
    d, n, cap = 64, 257, 300
    Pi = synth.random_rotation(d, 2)
    S = synth.gaussian_projection(d, 2)
    rg = np.random.default_rng(12)
    X = rg.standard_normal((2 * cap, d)).astype(np.float32)
    kp = quantize_gpu(dev(X), d, 3, True, Pi, S)
    vp = quantize_gpu(dev(X[::-1].copy()), d, 3, False, Pi)
    lay = tq.layout(d, 3, 3)
    c, _ = book(d, 3)
    q = torch.zeros((1, 2, 1, d), device="cuda")         # zero query: uniform softmax
    q[0, 1] = dev(rg.standard_normal(d))
    out = torch.empty((1, 2, 1, d), device="cuda")
    ws = tq.decode_workspace(lay, 1, 2, 2, 1, n)
    tq.tq_decode_attention(lay, q, kp, vp, 2, n, dev(Pi), dev(Pi), dev(S), dev(c), dev(c), out, ws, ctx_stride=cap)
    torch.cuda.synchronize()
    hk, hv = P.host_planes(kp), P.host_planes(vp)
    qn = q.cpu().numpy().astype(np.float64)
    for h in range(2):
        rows = slice(h * cap, h * cap + n)
        kpl = oa.KeyPlanes(hk["idx"][rows], hk["sign"][rows], hk["norm"][rows], hk["rnorm"][rows], 3)
        vpl = oa.ValuePlanes(hv["idx"][rows], hv["norm"][rows], 3)
        ref = oa.attention(qn[0, h], kpl, vpl, Pi, Pi, S, c, c)
        P.check_out(out[0, h], ref.out)
    ref0 = oa.dequantize_values(oa.ValuePlanes(hv["idx"][:n], hv["norm"][:n], 3), Pi, c, d).mean(0)
    P.check_out(out[0, 0, 0], ref0)


def test_device_status_reports_bad_codebook_and_position():
    d = 64
    Pi = dev(synth.random_rotation(d, 0))
    x = dev(np.random.default_rng(1).standard_normal((8, d)))
    lay = tq.layout(d, 3, 3)
    planes = tq.alloc_planes(8, d, 3, False)
    c, t = book(d, 3)
    bad_t = t.copy()
    bad_t[2], bad_t[3] = bad_t[3], bad_t[2]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_quantize_kv(lay, False, x, planes, Pi, dev(c), dev(bad_t), d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & tq.TQ_DEV_BAD_CODEBOOK
    st.zero_()
    pos = torch.tensor([0, 1, -5, 3, 4, 5, 6, 7], dtype=torch.int32, device="cuda")
    tq.tq_quantize_kv(lay, False, x, planes, Pi, dev(c), dev(t), positions=pos, rope_base=1e4, d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & tq.TQ_DEV_BAD_POSITION


# ---------------------------------------------------------------------------
# Full-size Llama-shaped layer (B=8, 32/8 heads, d=128, 32768 tokens), sampled.
# ---------------------------------------------------------------------------
def test_full_llama_layer_sampled():
    shape = synth.LlamaDecodeShape()
    d, layer = shape.d, 5
    K = synth.llama_layer_kv(shape, 0, layer, "cuda", "K").reshape(-1, d)
    V = synth.llama_layer_kv(shape, 0, layer, "cuda", "V").reshape(-1, d)
    Q = synth.llama_queries(shape, 0, "cuda")[layer].reshape(shape.batch, shape.hq, 1, d).contiguous()
    Pi = synth.random_rotation(d, 0)
    S = synth.gaussian_projection(d, 0)
    kp = quantize_gpu(K, d, 3, True, Pi, S)
    vp = quantize_gpu(V, d, 3, False, Pi)
    n = K.shape[0]
    rg = np.random.default_rng(99)
    sample = np.sort(rg.choice(n, 20000, replace=False))
    si = torch.as_tensor(sample, device="cuda")
    Ks = K[si].float().cpu().numpy().astype(np.float64)
    Vs = V[si].float().cpu().numpy().astype(np.float64)

    def sub(p, key):
        h = {"idx": p.idx[si].cpu().numpy(), "norm": p.norm[si].cpu().numpy()}
        if key:
            h["sign"] = p.sign[si].cpu().numpy().view(np.uint32)
            h["rnorm"] = p.rnorm[si].cpu().numpy()
        return h

    P.compare_quantized(sub(kp, True), quantize_ref(Ks, d, 3, True, Pi, S), d, 3, True)
    P.compare_quantized(sub(vp, False), quantize_ref(Vs, d, 3, False, Pi), d, 3, False)

    lay = tq.layout(d, 3, 3)
    c, _ = book(d, 3)
    N = shape.n_ctx
    out = torch.empty((shape.batch, shape.hq, 1, d), dtype=torch.bfloat16, device="cuda")
    scores = torch.empty((shape.batch, shape.hq, 1, N), dtype=torch.float32, device="cuda")
    ws = tq.decode_workspace(lay, shape.batch, shape.hq, shape.hkv, 1, N)
    tq.tq_decode_attention(lay, Q, kp, vp, shape.hkv, N, dev(Pi), dev(Pi), dev(S), dev(c), dev(c), out, ws,
                           scores_out=scores)
    torch.cuda.synchronize()
    G = shape.hq // shape.hkv
    Qn = Q.float().cpu().numpy().astype(np.float64)
    hk_all, hv_all = P.host_planes(kp), P.host_planes(vp)
    sc_all = scores.cpu().numpy()
    worst_s, worst_o = 0.0, 0.0
    for bi in range(shape.batch):                      # every (batch, kv head) stream
        for kv in range(shape.hkv):
            rows = slice((bi * shape.hkv + kv) * N, (bi * shape.hkv + kv + 1) * N)
            hk = {k: v[rows] for k, v in hk_all.items()}
            hv = {k: v[rows] for k, v in hv_all.items()}
            qs = Qn[bi, kv * G:(kv + 1) * G, 0]
            ref = oa.attention(qs, P.key_planes(hk, 3), P.value_planes(hv, 3), Pi, Pi, S, c, c)
            worst_s = max(worst_s, P.check_scores(sc_all[bi, kv * G:(kv + 1) * G, 0], ref.scores,
                                                  np.linalg.norm(qs, axis=1), hk["norm"], d))
            worst_o = max(worst_o, P.check_out(out[bi, kv * G:(kv + 1) * G, 0], ref.out))
    print(f"full layer, 64 streams: worst score error / bound {worst_s:.3g}, worst |out - ref| {worst_o:.3g}")


# ---------------------------------------------------------------------------
# Both quantize kernels (tensor-core and CUDA-core) against the oracle.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_tensor_core_and_cuda_core_quantize_paths(d, bits, monkeypatch):
    rg = np.random.default_rng(100 * d + bits)
    n = 128 * 5 + 37                                   # ragged last tile
    X = rg.standard_normal((n, d))
    X[:, rg.choice(d, 3, replace=False)] *= 10.0
    X[5] = 0.0
    X[n - 1] = 0.0
    Xb = synth.to_bf16(X.astype(np.float32))
    X64 = Xb.float().numpy().astype(np.float64)
    Pi = synth.random_rotation(d, 3)
    S = synth.gaussian_projection(d, 3)
    for is_key in (True, False):
        ref = quantize_ref(X64, d, bits, is_key, Pi, S if is_key else None)
        monkeypatch.setenv("TQ_QUANTIZE_PATH", "tensor-core")
        p_tc = quantize_gpu(Xb.cuda(), d, bits, is_key, Pi, S if is_key else None)
        monkeypatch.setenv("TQ_QUANTIZE_PATH", "cuda-core")
        p_cc = quantize_gpu(Xb.cuda(), d, bits, is_key, Pi, S if is_key else None)
        monkeypatch.delenv("TQ_QUANTIZE_PATH")
        p_ex = quantize_gpu(Xb.cuda(), d, bits, is_key, Pi, S if is_key else None)   # small call: exact kernel
        for p in (p_tc, p_cc, p_ex):
            P.compare_quantized(P.host_planes(p), ref, d, bits, is_key)


# ---------------------------------------------------------------------------
# The tensor-core quantizer searches a 3-bit table by |y| when the table is
# exactly symmetric and by the general binary search otherwise: both against
# the oracle, keys and values, several tiles and a ragged tail.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("shift", [0.0, 0.013])
def test_tensor_core_quantize_symmetric_and_shifted_tables(shift):
    d, bits = 128, 3
    b = ocb.lloyd_max_beta(d, bits)
    c = np.asarray(b.centroids, dtype=np.float64)
    c = 0.5 * (c - c[::-1])                              # exactly antisymmetric levels
    c = c + shift / np.sqrt(d)                           # a shift breaks the symmetry
    c32 = c.astype(np.float32)
    t32 = (0.5 * (c[1:] + c[:-1])).astype(np.float32)
    if shift == 0.0:
        assert np.all(t32 == -t32[::-1]) and t32[3] == 0.0
    else:
        assert not np.all(t32 == -t32[::-1])
    rg = np.random.default_rng(7)
    n = 128 * 9 + 5
    X = rg.standard_normal((n, d))
    X[:, rg.choice(d, 3, replace=False)] *= 10.0
    X[3] = 0.0
    Xb = synth.to_bf16(X.astype(np.float32))
    X64 = Xb.float().numpy().astype(np.float64)
    Pi = synth.random_rotation(d, 5)
    S = synth.gaussian_projection(d, 5)
    lay = tq.layout(d, bits, bits)
    for is_key in (True, False):
        ref = oq.quantize(X64, Pi, c32.astype(np.float64), t32.astype(np.float64), bits, S=S if is_key else None)
        planes = tq.alloc_planes(n, d, bits, is_key)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        tq.tq_quantize_kv(lay, is_key, Xb.cuda(), planes, dev(Pi), dev(c32), dev(t32),
                          S=dev(S) if is_key else None, d_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        P.compare_quantized(P.host_planes(planes), ref, d, bits, is_key)


# ---------------------------------------------------------------------------
# Guard canaries: every output buffer sits between 4 KiB fences of a known byte;
# after quantize (ragged tail), decode and dequantize the fences must be intact.
# ---------------------------------------------------------------------------
_FENCE = 4096


def _fenced(shape, dtype):
    n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    buf = torch.full((2 * _FENCE + n,), 0xA5, dtype=torch.uint8, device="cuda")
    return buf, buf[_FENCE:_FENCE + n].view(dtype).view(*shape)


def _fences_intact(buf):
    return bool((buf[:_FENCE] == 0xA5).all()) and bool((buf[buf.numel() - _FENCE:] == 0xA5).all())


def test_output_fences_intact_after_quantize_decode_dequantize():
    d, bits, B, HKV, HQ, N = 128, 3, 2, 2, 8, 1000     # tensor-core paths, ragged tiles
    n = B * HKV * N
    c32, t32 = book(d, bits)
    Pi = synth.random_rotation(d, 11)
    S = synth.gaussian_projection(d, 11)
    rg = np.random.default_rng(11)
    X = synth.to_bf16(rg.standard_normal((2, n, d)).astype(np.float32)).cuda()
    lay = tq.layout(d, bits, bits)
    bufs = []

    def fenced_planes(is_key):
        fb = [_fenced((n, tq.tq_idx_row_bytes(d, bits)), torch.uint8), _fenced((n,), torch.float32)]
        if is_key:
            fb += [_fenced((n, tq.tq_sign_words(d)), torch.int32), _fenced((n,), torch.float32)]
        bufs.extend(b for b, _ in fb)
        v = [t for _, t in fb]
        return tq.Planes(idx=v[0], norm=v[1], sign=v[2] if is_key else None, rnorm=v[3] if is_key else None)

    kp, vp = fenced_planes(True), fenced_planes(False)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_quantize_kv(lay, True, X[0], kp, dev(Pi), dev(c32), dev(t32), S=dev(S), d_status=st)
    tq.tq_quantize_kv(lay, False, X[1], vp, dev(Pi), dev(c32), dev(t32), d_status=st)
    q = torch.randn(B, HQ, 1, d, device="cuda")
    ob, out = _fenced((B, HQ, 1, d), torch.float32)
    ws_bytes = (tq.tq_decode_workspace_bytes(lay, B, HQ, HKV, 1, N) + 255) // 256 * 256
    wb, ws = _fenced((ws_bytes,), torch.uint8)
    sb, scores = _fenced((B, HQ, 1, N), torch.float32)
    tq.tq_decode_attention(lay, q, kp, vp, HKV, N, dev(Pi), dev(Pi), dev(S), dev(c32), dev(c32), out, ws,
                           scores_out=scores, d_status=st)
    db, deq = _fenced((n, d), torch.float32)
    tq.tq_dequantize(lay, True, kp, n, dev(Pi), dev(c32), deq, S=dev(S))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    bufs += [ob, wb, sb, db]
    assert all(_fences_intact(b) for b in bufs)
    assert torch.isfinite(out).all() and torch.isfinite(deq).all()


# ---------------------------------------------------------------------------
# Per-head rotations (one Pi per `vpp` consecutive vectors): the tensor-core
# quantiser takes them at d = 64 when vpp is a multiple of its 128-vector
# tile (many heads per CTA, so the two Pi slots are reused), the CUDA-core
# kernel otherwise (vpp = 100). Ragged last head in every case.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("vpp,heads", [(128, 600), (384, 100), (100, 50)])
def test_per_head_rotation_quantize(bits, vpp, heads):
    d = 64
    n = heads * vpp - 37
    rg = np.random.default_rng(1000 * bits + vpp)
    X = rg.standard_normal((n, d))
    X[:, rg.choice(d, 4, replace=False)] *= 8.0
    X[7] = 0.0
    Xb = synth.to_bf16(X.astype(np.float32))
    X64 = Xb.float().numpy().astype(np.float64)
    Pis = np.stack([synth.random_rotation(d, 50 + h) for h in range(heads)])
    S = synth.gaussian_projection(d, 4)
    group = np.arange(n) // vpp
    for is_key in (True, False):
        planes = quantize_gpu(Xb.cuda(), d, bits, is_key, Pis.reshape(heads * d, d), S if is_key else None,
                              vpp=vpp, pi_stride=d * d)
        ref = quantize_ref(X64, d, bits, is_key, Pis, S if is_key else None, pi_group=group)
        P.compare_quantized(P.host_planes(planes), ref, d, bits, is_key)
