"""Attention over the packed cache and dequantisation (oracle, fp64).

Test infrastructure only. Sources:
  * 7minutos.es "KV cache ... TurboQuant", Etapa 1: dequantisation looks each
    index up in the codebook and multiplies by the transpose of the rotation,
    K_hat = R^T c[idx]. Etapa 2: the stored sign bits are multiplied by S^T and
    scaled by sqrt(pi/2)/d and the stored residual norm, which makes the
    sign-based inner-product estimate unbiased; K_tilde = K_hat + K_tilde_QJL.
  * gist.science "TurboESM ..." section 2A: scores are computed after RoPE and
    the orthogonal Pi (Pi^T Pi = I preserves them); section 2E: the decode
    kernel fuses unpacking, the QJL correction, the inverse rotation Pi^T and
    online-softmax attention.

Readings (pages silent): scale 1/sqrt(d); no mask (the decode query attends
the whole cache; the ESM-shaped pass is bidirectional); query head h reads
KV head h // (Hq/Hkv); V is accumulated in rotated coordinates and turned back
by Pi_V^T once, which equals dequantising every value first.

Score of key j for a query q (both already RoPE'd):
  q_rot = Pi_K q,  s = S q_rot,
  score_j = scale * ( ||k_j|| <q_rot, c_K[idx_j]>
                      + sqrt(pi/2)/d * ||r_j|| <s, 2*sign_j - 1> ).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

from .quantize import rope, unpack_codes, unpack_signs


@dataclasses.dataclass
class KeyPlanes:
    idx: np.ndarray     # [N, d*b/8] uint8
    sign: np.ndarray    # [N, ceil(d/32)] uint32
    norm: np.ndarray    # [N] float32
    rnorm: np.ndarray   # [N] float32
    bits: int


@dataclasses.dataclass
class ValuePlanes:
    idx: np.ndarray     # [N, d*b/8] uint8
    norm: np.ndarray    # [N] float32
    bits: int


def qjl_scale(d: int) -> float:
    return math.sqrt(math.pi / 2.0) / d


def rotate_query(q: np.ndarray, Pi: np.ndarray, positions=None, rope_base: float = 0.0) -> np.ndarray:
    q = np.asarray(q, dtype=np.float64)
    if rope_base > 0.0 and positions is not None:
        q = rope(q, positions, rope_base)
    return q @ np.asarray(Pi, dtype=np.float64).T


def key_scores(q_rot: np.ndarray, kp: KeyPlanes, S: np.ndarray, centroids: np.ndarray,
               scale: float) -> np.ndarray:
    """[nq, N] scores of rotated queries against packed keys."""
    q_rot = np.atleast_2d(np.asarray(q_rot, dtype=np.float64))
    d = q_rot.shape[1]
    codes = unpack_codes(kp.idx, kp.bits, d)
    c = np.asarray(centroids, dtype=np.float64)[codes]               # [N, d]
    pm = np.where(unpack_signs(kp.sign, d), 1.0, -1.0)               # [N, d]
    s = q_rot @ np.asarray(S, dtype=np.float64).T                    # [nq, d]
    mse_term = (q_rot @ c.T) * kp.norm.astype(np.float64)[None, :]
    qjl_term = qjl_scale(d) * (s @ pm.T) * kp.rnorm.astype(np.float64)[None, :]
    return scale * (mse_term + qjl_term)


def value_rows_rotated(vp: ValuePlanes, centroids: np.ndarray, d: int) -> np.ndarray:
    """[N, d] ||v|| c_V[idx] in rotated coordinates."""
    codes = unpack_codes(vp.idx, vp.bits, d)
    return np.asarray(centroids, dtype=np.float64)[codes] * vp.norm.astype(np.float64)[:, None]


def softmax(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(z - z.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


@dataclasses.dataclass
class AttentionResult:
    out: np.ndarray      # [nq, d] in the original V coordinates
    scores: np.ndarray   # [nq, N]
    probs: np.ndarray    # [nq, N]


def attention(q: np.ndarray, kp: KeyPlanes, vp: ValuePlanes, PiK: np.ndarray, PiV: np.ndarray,
              S: np.ndarray, cK: np.ndarray, cV: np.ndarray, scale: float | None = None,
              q_positions=None, rope_base: float = 0.0) -> AttentionResult:
    """Exact softmax attention of queries q ([nq, d], pre-RoPE) over one head's cache."""
    q = np.atleast_2d(q)
    d = q.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    q_rot = rotate_query(q, PiK, q_positions, rope_base)
    sc = key_scores(q_rot, kp, S, cK, scale)
    p = softmax(sc)
    o_rot = p @ value_rows_rotated(vp, cV, d)
    out = o_rot @ np.asarray(PiV, dtype=np.float64)       # Pi_V^T o_rot, row form
    return AttentionResult(out=out, scores=sc, probs=p)


def dequantize_keys(kp: KeyPlanes, Pi: np.ndarray, S: np.ndarray, centroids: np.ndarray,
                    d: int) -> np.ndarray:
    """K_tilde = Pi^T ( ||k|| c[idx] + sqrt(pi/2)/d ||r|| S^T (2 sign - 1) ), rows [N, d]."""
    codes = unpack_codes(kp.idx, kp.bits, d)
    k_hat_rot = np.asarray(centroids, dtype=np.float64)[codes] * kp.norm.astype(np.float64)[:, None]
    pm = np.where(unpack_signs(kp.sign, d), 1.0, -1.0)
    corr_rot = qjl_scale(d) * kp.rnorm.astype(np.float64)[:, None] * (pm @ np.asarray(S, dtype=np.float64))
    return (k_hat_rot + corr_rot) @ np.asarray(Pi, dtype=np.float64)


def dequantize_values(vp: ValuePlanes, Pi: np.ndarray, centroids: np.ndarray, d: int) -> np.ndarray:
    """V_hat = Pi^T ||v|| c[idx], rows [N, d]."""
    return value_rows_rotated(vp, centroids, d) @ np.asarray(Pi, dtype=np.float64)


def plain_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float | None = None) -> np.ndarray:
    """Unquantised softmax attention, fp64 (for the invariance and quality checks)."""
    q = np.atleast_2d(np.asarray(q, dtype=np.float64))
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[1])
    return softmax(scale * q @ K.T) @ V
