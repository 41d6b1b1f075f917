"""Search for batch serving: sharded corpora and query batches larger than one pass.

* A corpus searched in two row ranges (shards) and merged with
  tq_search_merge_topk (ids shifted by the shard offset) must give exactly the
  ids and scores of one search over the whole corpus, also when the merge
  writes over one of its inputs.
* A workspace that holds only a few queries' share makes tq_search_topk run
  many passes; the results must equal the one-pass results bit for bit.
* The one-pass results themselves match the oracle's estimated top-k.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import attention as oa
from oracle import codebook as ocb
from oracle import search as osr

from . import parity as P

pytestmark = pytest.mark.gpu
tq = pytest.importorskip("kv_cache_vector_rope_b200")


def _dev(x):
    return torch.as_tensor(np.ascontiguousarray(x), device="cuda", dtype=torch.float32)


@pytest.fixture(scope="module")
def corpus():
    d, n, nq = 128, 70001, 300
    rg = np.random.default_rng(31)
    X = rg.standard_normal((n, d)).astype(np.float32)
    Q = rg.standard_normal((nq, d)).astype(np.float32)
    book = ocb.lloyd_max_beta(d, 3)
    c = book.centroids.astype(np.float32)
    t = (0.5 * (book.centroids[1:] + book.centroids[:-1])).astype(np.float32)
    Pi, S = synth.random_rotation(d, 8), synth.gaussian_projection(d, 8)
    lay = tq.layout(d, 3, 3)
    planes = tq.alloc_planes(n, d, 3, True)
    tq.tq_quantize_kv(lay, True, _dev(X), planes, _dev(Pi), _dev(c), _dev(t), S=_dev(S))
    torch.cuda.synchronize()
    return dict(d=d, n=n, nq=nq, X=X, Q=Q, c=c, Pi=Pi, S=S, lay=lay, planes=planes)


def _search(cp, planes, n_db, k, ws_bytes=None):
    nq = cp["nq"]
    ti = torch.empty((nq, k), dtype=torch.int64, device="cuda")
    ts = torch.empty((nq, k), device="cuda")
    need = tq.tq_search_workspace_bytes(cp["lay"], nq, n_db, k)
    ws = torch.empty((ws_bytes or need) + 256, dtype=torch.uint8, device="cuda")
    tq.tq_search_topk(cp["lay"], _dev(cp["Q"]), planes, n_db, _dev(cp["Pi"]), _dev(cp["S"]), _dev(cp["c"]), k, ti,
                      ts, ws[:ws_bytes] if ws_bytes else ws)
    torch.cuda.synchronize()
    return ti, ts


@pytest.mark.parametrize("k", [1, 10, 32])
def test_two_shards_merged_equal_the_whole_corpus(corpus, k):
    cp = corpus
    n, cut = cp["n"], 31337
    whole_i, whole_s = _search(cp, cp["planes"], n, k)
    ai, as_ = _search(cp, cp["planes"].rows(0, cut), cut, k)
    bi, bs = _search(cp, cp["planes"].rows(cut, n), n - cut, k)
    mi = torch.empty_like(ai)
    ms = torch.empty_like(as_)
    tq.tq_search_merge_topk(ai, as_, 0, bi, bs, cut, mi, ms)
    torch.cuda.synchronize()
    assert torch.equal(mi, whole_i) and torch.equal(ms, whole_s)
    # in place, and with the shards in the other order
    tq.tq_search_merge_topk(bi, bs, cut, ai, as_, 0, bi, bs)
    torch.cuda.synchronize()
    assert torch.equal(bi, whole_i) and torch.equal(bs, whole_s)


def test_query_blocks_equal_one_pass_and_the_oracle(corpus):
    cp = corpus
    k = 10
    one_i, one_s = _search(cp, cp["planes"], cp["n"], k)
    small = tq.tq_search_workspace_bytes(cp["lay"], 7, cp["n"], k)     # seven queries per pass
    blk_i, blk_s = _search(cp, cp["planes"], cp["n"], k, ws_bytes=(small + 255) // 256 * 256)
    assert torch.equal(blk_i, one_i) and torch.equal(blk_s, one_s)
    hp = P.host_planes(cp["planes"])
    kp = oa.KeyPlanes(hp["idx"], hp["sign"], hp["norm"], hp["rnorm"], 3)
    sub = np.arange(0, cp["nq"], 30)
    ref = osr.estimated_scores(cp["Q"][sub].astype(np.float64), kp, cp["Pi"], cp["S"], cp["c"])
    gi, gs = one_i.cpu().numpy(), one_s.cpu().numpy()
    for row, qi in enumerate(sub):
        typical = np.linalg.norm(cp["Q"][qi]) * np.abs(hp["norm"]).max() / np.sqrt(cp["d"])
        np.testing.assert_allclose(gs[qi], ref[row, gi[qi]], atol=P.SCORE_RTOL * typical)
        cut = np.sort(ref[row])[::-1][k - 1]
        assert np.all(ref[row, gi[qi]] >= cut - P.SCORE_RTOL * typical)
