"""Inner-product search over compressed codes (oracle, fp64).

Test infrastructure only. Sources: sudonull.com "TurboQuant: compresión 6x de
LLM KV-cache" (QJL preserves the inner products needed for attention; the same
codes serve vector search) and news.hada.io's TurboQuant summary (vector
search: recall of the true top inner products among the approximate top-k).

The estimated score of a database vector x for a query q is the attention
score without the 1/sqrt(d) factor (which does not change the ranking):
  est(q, x) = ||x|| <Pi q, c[idx_x]> + sqrt(pi/2)/d ||r_x|| <S Pi q, 2 sign_x - 1>.
Ranking is by decreasing score; equal scores rank by increasing index.
"""
from __future__ import annotations

import numpy as np

from .attention import KeyPlanes, key_scores, rotate_query


def top_k(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest scores per row, ties by lower index."""
    order = np.lexsort((np.broadcast_to(np.arange(scores.shape[1]), scores.shape), -scores), axis=-1)
    return order[:, :k]


def estimated_scores(Q: np.ndarray, planes: KeyPlanes, Pi: np.ndarray, S: np.ndarray,
                     centroids: np.ndarray) -> np.ndarray:
    return key_scores(rotate_query(Q, Pi), planes, S, centroids, 1.0)


def exact_top_k(Q: np.ndarray, X: np.ndarray, k: int, block: int = 65536) -> np.ndarray:
    """Exact inner-product top-k by brute force in fp64."""
    Q = np.asarray(Q, dtype=np.float64)
    best_s = np.full((Q.shape[0], 0), -np.inf)
    best_i = np.zeros((Q.shape[0], 0), dtype=np.int64)
    for s0 in range(0, X.shape[0], block):
        blk = np.asarray(X[s0:s0 + block], dtype=np.float64)
        sc = Q @ blk.T
        idx = np.broadcast_to(np.arange(s0, s0 + blk.shape[0]), sc.shape)
        cs = np.concatenate([best_s, sc], axis=1)
        ci = np.concatenate([best_i, idx], axis=1)
        order = np.lexsort((ci, -cs), axis=-1)[:, :k]
        best_s = np.take_along_axis(cs, order, axis=1)
        best_i = np.take_along_axis(ci, order, axis=1)
    return best_i


def recall_at_k(approx: np.ndarray, exact: np.ndarray) -> float:
    k = exact.shape[1]
    hits = [len(set(a.tolist()) & set(e.tolist())) for a, e in zip(approx, exact)]
    return float(np.mean(hits)) / k
