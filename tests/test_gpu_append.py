"""Incremental decode: quantise-and-append one token per stream, then decode.

A cache of capacity 600 per (batch, kv head) stream holds 517 prefilled tokens
(keys RoPE'd at positions 0..516). Three decode steps each append one new key
(RoPE at its position) and value per stream with tq_append_kv, then attend a
query at that position over the grown cache with tq_decode_attention
(ctx_stride 600). The appended rows must equal the oracle's quantisation of
the new vectors (bit-exact outside the guard band), rows outside the slot
must not change, and scores and outputs must match the oracle over the grown
cache. d = 128, GQA group 4, 3-bit values (the tensor-core decode) and a
group-8 case (the CUDA-core decode).
"""
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


def _dev(x, dt=torch.float32):
    return torch.as_tensor(np.ascontiguousarray(x), device="cuda").to(dt)


@pytest.mark.parametrize("G", [4, 8])
def test_append_three_tokens_then_decode(G):
    b, hkv, d, cap, n0, base = 2, 2, 128, 600, 517, 10000.0
    hq, streams = hkv * G, b * hkv
    rg = np.random.default_rng(40 + G)
    book = ocb.lloyd_max_beta(d, 3)
    c = book.centroids.astype(np.float32)
    t = (0.5 * (book.centroids[1:] + book.centroids[:-1])).astype(np.float32)
    Pi = synth.random_rotation(d, 7)
    S = synth.gaussian_projection(d, 7)
    lay = tq.layout(d, 3, 3)
    # Prefill: streams x cap rows, the first n0 of each stream valid.
    K0 = synth.to_bf16(rg.standard_normal((streams, cap, d)).astype(np.float32))
    V0 = synth.to_bf16(rg.standard_normal((streams, cap, d)).astype(np.float32))
    pos0 = np.tile(np.arange(cap, dtype=np.int32), streams)
    kp = tq.alloc_planes(streams * cap, d, 3, True)
    vp = tq.alloc_planes(streams * cap, d, 3, False)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_quantize_kv(lay, True, K0.reshape(-1, d).cuda(), kp, _dev(Pi), _dev(c), _dev(t), S=_dev(S),
                      positions=torch.as_tensor(pos0, device="cuda"), rope_base=base, d_status=st)
    tq.tq_quantize_kv(lay, False, V0.reshape(-1, d).cuda(), vp, _dev(Pi), _dev(c), _dev(t), d_status=st)
    ws = tq.decode_workspace(lay, b, hq, hkv, 1, cap)
    for step in range(3):
        slot = n0 + step
        kn = synth.to_bf16(rg.standard_normal((streams, d)).astype(np.float32))
        vn = synth.to_bf16(rg.standard_normal((streams, d)).astype(np.float32))
        pos = np.full(streams, slot, dtype=np.int32)
        before = P.host_planes(kp), P.host_planes(vp)
        tq.tq_append_kv(lay, True, kn.cuda(), kp, cap, slot, _dev(Pi), _dev(c), _dev(t), S=_dev(S),
                        positions=torch.as_tensor(pos, device="cuda"), rope_base=base, d_status=st)
        tq.tq_append_kv(lay, False, vn.cuda(), vp, cap, slot, _dev(Pi), _dev(c), _dev(t), d_status=st)
        q = synth.to_bf16(rg.standard_normal((b, hq, 1, d)).astype(np.float32))
        n = slot + 1
        out = torch.empty((b, hq, 1, d), dtype=torch.float32, device="cuda")
        scores = torch.empty((b, hq, 1, n), device="cuda")
        tq.tq_decode_attention(lay, q.cuda(), kp, vp, hkv, n, _dev(Pi), _dev(Pi), _dev(S), _dev(c), _dev(c), out, ws,
                               q_positions=torch.full((b, 1), slot, dtype=torch.int32, device="cuda"),
                               rope_base=base, ctx_stride=cap, scores_out=scores, d_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        hk, hv = P.host_planes(kp), P.host_planes(vp)
        rows = np.arange(streams) * cap + slot
        # The appended rows against the oracle; every other row unchanged.
        c64, t64 = c.astype(np.float64), t.astype(np.float64)
        refk = oq.quantize(kn.float().numpy().astype(np.float64), Pi, c64, t64, 3, S=S, positions=pos, rope_base=base)
        refv = oq.quantize(vn.float().numpy().astype(np.float64), Pi, c64, t64, 3)
        P.compare_quantized({k: v[rows] for k, v in hk.items()}, refk, d, 3, True)
        P.compare_quantized({k: v[rows] for k, v in hv.items()}, refv, d, 3, False)
        keep = np.ones(streams * cap, dtype=bool)
        keep[rows] = False
        for new, old in ((hk, before[0]), (hv, before[1])):
            for k in new:
                assert np.array_equal(new[k][keep], old[k][keep]), k
        # Decode over the grown cache.
        qn = q.float().numpy().astype(np.float64)
        for bi in range(b):
            for kv in range(hkv):
                s0 = (bi * hkv + kv) * cap
                r = slice(s0, s0 + n)
                kpl = P.key_planes({k: v[r] for k, v in hk.items()}, 3)
                vpl = P.value_planes({k: v[r] for k, v in hv.items()}, 3)
                qs = qn[bi, kv * G:(kv + 1) * G, 0]
                ref = oa.attention(qs, kpl, vpl, Pi, Pi, S, c, c, q_positions=np.full(G, slot), rope_base=base)
                P.check_scores(scores[bi, kv * G:(kv + 1) * G, 0].cpu().numpy(), ref.scores,
                               np.linalg.norm(qs, axis=1), hk["norm"][r], d)
                P.check_out(out[bi, kv * G:(kv + 1) * G, 0], ref.out)
