"""GPU parity on the ESM-2-shaped cache and the long-context bit sweep.

ESM-shaped (33 layers x 20 heads, d=64, 1024 tokens, bf16): every head has its
own rotation Pi_h = Pi_rand V_h^T fitted on 256 calibration tokens, keys and
values use their own empirical (dual) codebooks, the whole cache is quantised
and one bidirectional 1024-query attention pass runs per head. Long context
(131072 tokens, 8/32 heads, d=128): key bits 2/3/4 with QJL, sampled parity
and the score error of each bit-width against exact q.k/sqrt(d).
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import attention as oa
from oracle import calib as oc
from oracle import codebook as ocb
from oracle import quantize as oq

from . import parity as P

pytestmark = pytest.mark.gpu
tq = pytest.importorskip("kv_cache_vector_rope_b200")


def dev(x, dtype=torch.float32):
    return torch.as_tensor(np.ascontiguousarray(x), device="cuda").to(dtype)


def f32_book(book):
    c = book.centroids.astype(np.float32)
    t = (0.5 * (book.centroids[1:] + book.centroids[:-1])).astype(np.float32)
    return c, t


@pytest.fixture(scope="module")
def esm():
    data = synth.esm_cache(0)
    L, H, N, d = data.K.shape
    cK = data.calib_K.float().numpy().astype(np.float64)
    cV = data.calib_V.float().numpy().astype(np.float64)
    PiK = np.stack([oc.head_rotation(data.Pi, cK[l, h]) for l in range(L) for h in range(H)]).astype(np.float32)
    PiV = np.stack([oc.head_rotation(data.Pi, cV[l, h]) for l in range(L) for h in range(H)]).astype(np.float32)
    bk, bv = oc.dual_codebooks([cK[l, h] for l in range(L) for h in range(H)],
                               [cV[l, h] for l in range(L) for h in range(H)],
                               list(PiK.astype(np.float64)), list(PiV.astype(np.float64)), 3)
    return data, PiK, PiV, f32_book(bk), f32_book(bv)


def test_esm_shape_quantize_and_full_sequence_attention(esm):
    data, PiK, PiV, (cK, tK), (cV, tV) = esm
    L, H, N, d = data.K.shape
    n = L * H * N
    lay = tq.layout(d, 3, 3)
    Kd = data.K.reshape(n, d).cuda()
    Vd = data.V.reshape(n, d).cuda()
    kp = tq.alloc_planes(n, d, 3, True)
    vp = tq.alloc_planes(n, d, 3, False)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_quantize_kv(lay, True, Kd, kp, dev(PiK), dev(cK), dev(tK), S=dev(data.S), vectors_per_pi=N,
                      pi_stride=d * d, d_status=st)
    tq.tq_quantize_kv(lay, False, Vd, vp, dev(PiV), dev(cV), dev(tV), vectors_per_pi=N, pi_stride=d * d,
                      d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    # Sampled code parity over the whole cache (per-head rotations).
    rg = np.random.default_rng(5)
    sample = np.sort(rg.choice(n, 20000, replace=False))
    si = torch.as_tensor(sample, device="cuda")
    group = sample // N
    for which, x, p, Pi, c, t, key in (("K", Kd, kp, PiK, cK, tK, True), ("V", Vd, vp, PiV, cV, tV, False)):
        xs = x[si].float().cpu().numpy().astype(np.float64)
        ref = oq.quantize(xs, Pi, c.astype(np.float64), t.astype(np.float64), 3, S=data.S if key else None,
                          pi_group=group)
        h = {"idx": p.idx[si].cpu().numpy(), "norm": p.norm[si].cpu().numpy()}
        if key:
            h["sign"] = p.sign[si].cpu().numpy().view(np.uint32)
            h["rnorm"] = p.rnorm[si].cpu().numpy()
        P.compare_quantized(h, ref, d, 3, key)
    # One full bidirectional pass of layer 7: 1024 queries per head.
    l = 7
    q = data.Q[l].reshape(1, H, N, d).contiguous().cuda()
    out = torch.empty((1, H, N, d), dtype=torch.float32, device="cuda")
    scores = torch.empty((1, H, N, N), dtype=torch.float32, device="cuda")
    ws = tq.decode_workspace(lay, 1, H, H, N, N)
    rows = slice(l * H * N, (l + 1) * H * N)
    tq.tq_decode_attention(lay, q, kp.rows(rows.start, rows.stop), vp.rows(rows.start, rows.stop), H, N,
                           dev(PiK[l * H:(l + 1) * H]), dev(PiV[l * H:(l + 1) * H]), dev(data.S), dev(cK), dev(cV),
                           out, ws, pi_stride=d * d, scores_out=scores)
    torch.cuda.synchronize()
    hk = {"idx": kp.idx[rows].cpu().numpy(), "sign": kp.sign[rows].cpu().numpy().view(np.uint32),
          "norm": kp.norm[rows].cpu().numpy(), "rnorm": kp.rnorm[rows].cpu().numpy()}
    hv = {"idx": vp.idx[rows].cpu().numpy(), "norm": vp.norm[rows].cpu().numpy()}
    qn = data.Q[l].float().numpy().astype(np.float64)
    for h in (0, 11, 19):
        r = slice(h * N, (h + 1) * N)
        kpl = oa.KeyPlanes(hk["idx"][r], hk["sign"][r], hk["norm"][r], hk["rnorm"][r], 3)
        vpl = oa.ValuePlanes(hv["idx"][r], hv["norm"][r], 3)
        ref = oa.attention(qn[h], kpl, vpl, PiK[l * H + h], PiV[l * H + h], data.S, cK, cV)
        P.check_scores(scores[0, h].cpu().numpy(), ref.scores, np.linalg.norm(qn[h], axis=1), hk["norm"][r], d)
        P.check_out(out[0, h], ref.out)


@pytest.mark.parametrize("kbits", [2, 3, 4])
def test_long_context_bits_sampled(kbits):
    d, n = 128, 131072
    lc = synth.long_context(0, n=n, device="cuda")
    hkv, hq = lc.K.shape[1], lc.Q.shape[1]
    kb = ocb.lloyd_max_beta(d, kbits)
    vb = ocb.lloyd_max_beta(d, 3)
    cK, tK = f32_book(kb)
    cV, tV = f32_book(vb)
    lay = tq.layout(d, kbits, 3)
    K = lc.K.reshape(-1, d)
    V = lc.V.reshape(-1, d)
    kp = tq.alloc_planes(K.shape[0], d, kbits, True)
    vp = tq.alloc_planes(V.shape[0], d, 3, False)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_quantize_kv(lay, True, K, kp, dev(lc.Pi), dev(cK), dev(tK), S=dev(lc.S), d_status=st)
    tq.tq_quantize_kv(lay, False, V, vp, dev(lc.Pi), dev(cV), dev(tV), d_status=st)
    out = torch.empty((1, hq, 1, d), dtype=torch.bfloat16, device="cuda")
    scores = torch.empty((1, hq, 1, n), device="cuda")
    ws = tq.decode_workspace(lay, 1, hq, hkv, 1, n)
    q = lc.Q.reshape(1, hq, 1, d).contiguous()
    tq.tq_decode_attention(lay, q, kp, vp, hkv, n, dev(lc.Pi), dev(lc.Pi), dev(lc.S), dev(cK), dev(cV), out, ws,
                           scores_out=scores)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rg = np.random.default_rng(kbits)
    sample = np.sort(rg.choice(K.shape[0], 8000, replace=False))
    si = torch.as_tensor(sample, device="cuda")
    ref = oq.quantize(K[si].float().cpu().numpy().astype(np.float64), lc.Pi, cK.astype(np.float64),
                      tK.astype(np.float64), kbits, S=lc.S)
    P.compare_quantized({"idx": kp.idx[si].cpu().numpy(), "sign": kp.sign[si].cpu().numpy().view(np.uint32),
                         "norm": kp.norm[si].cpu().numpy(), "rnorm": kp.rnorm[si].cpu().numpy()}, ref, d, kbits, True)
    G = hq // hkv
    qn = lc.Q.float().cpu().numpy().astype(np.float64)[0]
    for kv in (0, 5):
        rows = slice(kv * n, (kv + 1) * n)
        hk = {"idx": kp.idx[rows].cpu().numpy(), "sign": kp.sign[rows].cpu().numpy().view(np.uint32),
              "norm": kp.norm[rows].cpu().numpy(), "rnorm": kp.rnorm[rows].cpu().numpy()}
        hv = {"idx": vp.idx[rows].cpu().numpy(), "norm": vp.norm[rows].cpu().numpy()}
        qs = qn[kv * G:(kv + 1) * G]
        ref = oa.attention(qs, P.key_planes(hk, kbits), P.value_planes(hv, 3), lc.Pi, lc.Pi, lc.S, cK, cV)
        P.check_scores(scores[0, kv * G:(kv + 1) * G, 0].cpu().numpy(), ref.scores, np.linalg.norm(qs, axis=1),
                       hk["norm"], d)
        P.check_out(out[0, kv * G:(kv + 1) * G, 0], ref.out)


def test_search_top10_full_corpus():
    from oracle import search as osr
    corpus = synth.search_corpus(0)
    X, Q, d = corpus.X, corpus.Q, corpus.d
    n_db, nq, k = X.shape[0], Q.shape[0], 10
    book = ocb.lloyd_max_beta(d, 3)
    c, t = f32_book(book)
    lay = tq.layout(d, 3, 3)
    planes = tq.alloc_planes(n_db, d, 3, True)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_quantize_kv(lay, True, dev(X), planes, dev(corpus.Pi), dev(c), dev(t), S=dev(corpus.S), d_status=st)
    top_i = torch.empty((nq, k), dtype=torch.int64, device="cuda")
    top_s = torch.empty((nq, k), dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.tq_search_workspace_bytes(lay, nq, n_db, k) + 256, dtype=torch.uint8, device="cuda")
    tq.tq_search_topk(lay, dev(Q), planes, n_db, dev(corpus.Pi), dev(corpus.S), dev(c), k, top_i, top_s, ws)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    gi, gs = top_i.cpu().numpy(), top_s.cpu().numpy()
    assert np.all(np.diff(gs, axis=1) <= 0)                         # sorted by decreasing score
    sub = np.arange(0, nq, 100)                                     # 100 queries
    hp = P.host_planes(planes)
    ref = np.empty((len(sub), n_db))
    for s0 in range(0, n_db, 100000):
        kpl = oa.KeyPlanes(hp["idx"][s0:s0 + 100000], hp["sign"][s0:s0 + 100000], hp["norm"][s0:s0 + 100000],
                           hp["rnorm"][s0:s0 + 100000], 3)
        ref[:, s0:s0 + 100000] = osr.estimated_scores(Q[sub].astype(np.float64), kpl, corpus.Pi, corpus.S, c)
    ref_top = osr.top_k(ref, k)
    for row, qi in enumerate(sub):
        typical = np.linalg.norm(Q[qi]) * np.abs(hp["norm"]).max() / math.sqrt(d)
        tol = P.SCORE_RTOL * typical
        np.testing.assert_allclose(gs[qi], ref[row, gi[qi]], atol=tol)
        cut = ref[row, ref_top[row, k - 1]]
        for i in set(gi[qi]) - set(ref_top[row]):
            assert ref[row, i] >= cut - tol
        for i in set(ref_top[row]) - set(gi[qi]):
            assert ref[row, i] <= cut + tol
    # Recall@10 against exact search is a property of the method on this data
    # (tight mixture clusters make the true top-10 nearly tied); the GPU must
    # reproduce the oracle's estimated-search recall.
    exact = osr.exact_top_k(Q[sub], X, k)
    recall = osr.recall_at_k(gi[sub], exact)
    recall_ref = osr.recall_at_k(ref_top, exact)
    assert abs(recall - recall_ref) <= 0.01, (recall, recall_ref)
    print(f"recall@10 (100 queries): gpu {recall:.3f}, oracle {recall_ref:.3f}")
