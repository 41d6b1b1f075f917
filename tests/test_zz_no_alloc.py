"""tq_decode_attention_noalloc against tq_decode_attention (GPU).

The no-allocation entry point serves callers that cannot allocate device
memory when they call (for instance a serving loop that must not stall on
cudaMalloc's device synchronisation, or a plugin whose host framework owns all
device memory). It runs the same kernels with the library's fixed device
scratch array instead of a caller workspace, so its output must match the
regular entry point's within the decode tolerance — on consecutive calls,
since the shared array keeps the previous call's contents.

This file is named to be collected last; it also passes alone in a fresh
process (the first call on the device sets the scratch address up).
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from oracle import codebook as ocb

from . import parity as P

pytestmark = pytest.mark.gpu
tq = pytest.importorskip("kv_cache_vector_rope_b200")


def _cache(b=2, hkv=2, n=1000, d=128, seed=17):
    rg = np.random.default_rng(seed)
    K = synth.to_bf16(rg.standard_normal((b * hkv * n, d)).astype(np.float32)).cuda()
    V = synth.to_bf16(rg.standard_normal((b * hkv * n, d)).astype(np.float32)).cuda()
    book = ocb.lloyd_max_beta(d, 3)
    c = torch.as_tensor(book.centroids.astype(np.float32), device="cuda")
    t = torch.as_tensor((0.5 * (book.centroids[1:] + book.centroids[:-1])).astype(np.float32), device="cuda")
    Pi = torch.as_tensor(synth.random_rotation(d, 9), device="cuda")
    S = torch.as_tensor(synth.gaussian_projection(d, 9), device="cuda")
    lay = tq.layout(d, 3, 3)
    kp = tq.alloc_planes(K.shape[0], d, 3, True)
    vp = tq.alloc_planes(V.shape[0], d, 3, False)
    tq.tq_quantize_kv(lay, True, K, kp, Pi, c, t, S=S)
    tq.tq_quantize_kv(lay, False, V, vp, Pi, c, t)
    return lay, kp, vp, Pi, S, c


def test_noalloc_entry_point_matches_workspace_entry_point_on_consecutive_calls():
    b, hkv, hq, n, d = 2, 2, 8, 1000, 128
    lay, kp, vp, Pi, S, c = _cache(b, hkv, n, d)
    rg = np.random.default_rng(3)
    ws = tq.decode_workspace(lay, b, hq, hkv, 1, n)
    for call in range(2):
        q = synth.to_bf16(rg.standard_normal((b, hq, 1, d)).astype(np.float32)).cuda()
        ref = torch.empty((b, hq, 1, d), device="cuda")
        got = torch.empty((b, hq, 1, d), device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        tq.tq_decode_attention(lay, q, kp, vp, hkv, n, Pi, Pi, S, c, c, ref, ws, d_status=st)
        tq.tq_decode_attention_noalloc(lay, q, kp, vp, hkv, n, Pi, Pi, S, c, c, got, d_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0, f"call {call}: device status {int(st.item())}"
        P.check_out(got, ref.cpu().numpy().astype(np.float64))


def test_noalloc_entry_point_rejects_shapes_beyond_its_scratch():
    # 8 x 32 query heads x 4096 queries each needs far more than the fixed array.
    lay = tq.layout(128, 3, 3)
    kp = tq._Planes(0x1000, 0x2000, 0x3000, 0x4000)
    vp = tq._Planes(0x5000, 0, 0x6000, 0)
    st = tq._lib.tq_decode_attention_noalloc(ctypes.byref(lay), 0x100, 1, 8, 32, 8, 4096, 4096, 0, None, 0.0,
                                             ctypes.byref(kp), ctypes.byref(vp), 0x7000, 0x8000, 0, 0x9000, 0xa000,
                                             0xb000, 0.1, 0xc000, 0, None, None, None)
    assert st == tq.TQ_ERR_UNSUPPORTED
    assert "scratch" in tq.tq_last_error_string()
