"""RoPE -> rotation -> norm + Lloyd-Max codes -> QJL signs (oracle, fp64).

Test infrastructure only. Sources:
  * gist.science "TurboESM ..." section 2A (RoPE-invariant orthogonal
    transform): RoPE is applied first, then the orthogonal Pi; scores are
    preserved because Pi^T Pi = I.
  * 7minutos.es "KV cache ... TurboQuant", Etapa 1: y = R x with a random
    orthogonal R; each coordinate is replaced by the index of its Lloyd-Max
    level (b bits per coordinate); the cache keeps the indices.
    Etapa 2: the residual of stage 1 is multiplied by a random Gaussian
    projection S (d x d); only the signs of the result are kept, together with
    the L2 norm of the residual as one scalar per vector.
  * The extra scalar per vector (the norm) is what lets a codebook that
    depends only on (d, b) be used: coordinates are quantised on the unit
    sphere.

Readings taken where the pages are silent (each listed in the design notes):
  * RoPE pairs channel i with channel i + d/2 ("rotate-half") and turns the
    pair by pos * base^(-2i/d).
  * The norm ||x|| is stored as float32; the unit vector y/||x|| is quantised.
  * Bucketize is strict: code_i = #{j : u_i > t_j}; a tie goes to the lower
    code. A zero vector has u = 0.
  * The residual lives in rotated coordinates, r = y - ||x|| c[code], and S
    acts there (S_page = S Pi is Gaussian too, so the estimator is unchanged).
    Sign bit i is 1 iff (S r)_i >= 0.
  * Packing: a group of 8 consecutive coordinates occupies b bytes; read as a
    little-endian integer it holds code[8g + j] at bits [b*j, b*j + b).
    Sign bit i sits at bit (i mod 32) of 32-bit word floor(i / 32); pad bits
    are 0.
"""
from __future__ import annotations

import dataclasses

import numpy as np


def rope(x: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """Rotate-half RoPE in fp64: pair (i, i + d/2) turned by pos * base^(-2i/d)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = d // 2
    i = np.arange(h, dtype=np.float64)
    theta = np.asarray(pos, dtype=np.float64)[..., None] * base ** (-2.0 * i / d)
    c, s = np.cos(theta), np.sin(theta)
    a, b = x[..., :h], x[..., h:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def bucketize(u: np.ndarray, boundaries: np.ndarray) -> np.ndarray:
    """code = number of boundaries strictly below u."""
    t = np.asarray(boundaries, dtype=np.float64)
    return (u[..., None] > t).sum(axis=-1).astype(np.int64)


def nearest_centroid(u: np.ndarray, centroids: np.ndarray) -> np.ndarray:
    """Brute force over all centroids; lowest index on an exact tie."""
    c = np.asarray(centroids, dtype=np.float64)
    return np.argmin(np.abs(u[..., None] - c), axis=-1)


def row_bytes(d: int, bits: int) -> int:
    assert d % 8 == 0
    return d * bits // 8


def sign_words(d: int) -> int:
    return (d + 31) // 32


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """[n, d] codes -> [n, d*bits/8] bytes, 8 codes per `bits` bytes, little-endian."""
    codes = np.asarray(codes, dtype=np.int64)
    n, d = codes.shape
    out = np.zeros((n, row_bytes(d, bits)), dtype=np.uint8)
    for g in range(d // 8):
        word = np.zeros(n, dtype=np.int64)
        for j in range(8):
            word |= codes[:, 8 * g + j] << (bits * j)
        for byte in range(bits):
            out[:, g * bits + byte] = (word >> (8 * byte)) & 0xFF
    return out


def unpack_codes(plane: np.ndarray, bits: int, d: int) -> np.ndarray:
    plane = np.asarray(plane, dtype=np.int64)
    n = plane.shape[0]
    out = np.zeros((n, d), dtype=np.int64)
    mask = (1 << bits) - 1
    for g in range(d // 8):
        word = np.zeros(n, dtype=np.int64)
        for byte in range(bits):
            word |= plane[:, g * bits + byte] << (8 * byte)
        for j in range(8):
            out[:, 8 * g + j] = (word >> (bits * j)) & mask
    return out


def pack_signs(bits_set: np.ndarray) -> np.ndarray:
    """[n, d] booleans -> [n, ceil(d/32)] uint32, bit i at (word i//32, bit i%32)."""
    b = np.asarray(bits_set, dtype=bool)
    n, d = b.shape
    out = np.zeros((n, sign_words(d)), dtype=np.uint64)
    for i in range(d):
        out[:, i // 32] |= b[:, i].astype(np.uint64) << np.uint64(i % 32)
    return out.astype(np.uint32)


def unpack_signs(plane: np.ndarray, d: int) -> np.ndarray:
    plane = np.asarray(plane, dtype=np.uint64)
    out = np.zeros((plane.shape[0], d), dtype=bool)
    for i in range(d):
        out[:, i] = ((plane[:, i // 32] >> np.uint64(i % 32)) & np.uint64(1)) == 1
    return out


@dataclasses.dataclass
class Quantized:
    codes: np.ndarray        # [n, d] int64
    idx_plane: np.ndarray    # [n, d*b/8] uint8
    norm: np.ndarray         # [n] float32 (rounded from fp64)
    norm64: np.ndarray       # [n] float64
    u: np.ndarray            # [n, d] float64: y / ||x||
    code_margin: np.ndarray  # [n, d] float64: min_j |u_i - t_j|
    y: np.ndarray            # [n, d] float64 rotated vector
    # keys only
    signs: np.ndarray | None = None       # [n, d] bool
    sign_plane: np.ndarray | None = None  # [n, ceil(d/32)] uint32
    rnorm: np.ndarray | None = None       # [n] float32
    rnorm64: np.ndarray | None = None
    p: np.ndarray | None = None           # [n, d] float64 projection S r
    r: np.ndarray | None = None           # [n, d] float64 residual (rotated)


def quantize(x: np.ndarray, Pi: np.ndarray, centroids: np.ndarray, boundaries: np.ndarray,
             bits: int, S: np.ndarray | None = None, positions: np.ndarray | None = None,
             rope_base: float = 0.0, pi_group: np.ndarray | None = None) -> Quantized:
    """Quantise rows of x ([n, d]).

    Pi is [d, d] (shared) or [G, d, d] with ``pi_group[n]`` choosing each row's
    matrix. S (keys only) is [d, d]. centroids/boundaries are the codebook as
    stored (float32 values, used exactly)."""
    x = np.asarray(x, dtype=np.float64)
    n, d = x.shape
    if rope_base > 0.0 and positions is not None:
        x = rope(x, positions, rope_base)
    Pi = np.asarray(Pi, dtype=np.float64)
    if Pi.ndim == 2:
        y = x @ Pi.T
    else:
        y = np.einsum("nij,nj->ni", Pi[np.asarray(pi_group)], x)
    norm = np.sqrt(np.sum(x * x, axis=1))
    safe = np.where(norm > 0.0, norm, 1.0)
    u = np.where(norm[:, None] > 0.0, y / safe[:, None], 0.0)
    t = np.asarray(boundaries, dtype=np.float64)
    c = np.asarray(centroids, dtype=np.float64)
    codes = bucketize(u, t)
    margin = np.min(np.abs(u[..., None] - t), axis=-1)
    q = Quantized(codes=codes, idx_plane=pack_codes(codes, bits), norm=norm.astype(np.float32),
                  norm64=norm, u=u, code_margin=margin, y=y)
    if S is not None:
        r = y - norm[:, None] * c[codes]
        rn = np.sqrt(np.sum(r * r, axis=1))
        p = r @ np.asarray(S, dtype=np.float64).T
        signs = p >= 0.0
        q.signs, q.sign_plane = signs, pack_signs(signs)
        q.rnorm, q.rnorm64, q.p, q.r = rn.astype(np.float32), rn, p, r
    return q
