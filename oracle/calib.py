"""Per-head SVD calibration of the rotation (oracle, fp64).

Test infrastructure only. Source: gist.science "TurboESM ..." section 2B
(head-wise SVD calibration): instead of one global or random matrix, a Pi is
computed for every layer and attention head by SVD of real activations, which
equalises the variance across directions before quantisation.

Reading (pages silent on the composition): with X the uncentred C x d matrix
of one head's calibration vectors and X = U Sigma V^T its SVD, the head's
rotation is Pi_h = Pi_rand V^T — first turn into the singular basis, then apply
the seeded random rotation. Singular vectors are ordered by decreasing
singular value and each is signed so that its largest-magnitude entry is
positive (an SVD fixes them only up to sign).

The dual lookup tables (section 2C) are empirical Lloyd codebooks fitted to
the rotated, normalised calibration coordinates of K and of V separately,
pooled over all layers and heads.
"""
from __future__ import annotations

import numpy as np

from .codebook import lloyd_empirical


def right_singular_basis(X: np.ndarray) -> np.ndarray:
    """V (d x d, columns = right singular vectors) with the sign convention above."""
    X = np.asarray(X, dtype=np.float64)
    _, _, vt = np.linalg.svd(X, full_matrices=True)
    V = vt.T.copy()
    for j in range(V.shape[1]):
        k = int(np.argmax(np.abs(V[:, j])))
        if V[k, j] < 0:
            V[:, j] = -V[:, j]
    return V


def head_rotation(Pi_rand: np.ndarray, X: np.ndarray) -> np.ndarray:
    """Pi_h = Pi_rand V^T (fp64)."""
    return np.asarray(Pi_rand, dtype=np.float64) @ right_singular_basis(X).T


def rotated_unit_coordinates(X: np.ndarray, Pi: np.ndarray) -> np.ndarray:
    """Coordinates of Pi x / ||x|| for every row x (zero rows are skipped)."""
    X = np.asarray(X, dtype=np.float64)
    n = np.linalg.norm(X, axis=1)
    keep = n > 0
    return ((X[keep] @ np.asarray(Pi, dtype=np.float64).T) / n[keep, None]).ravel()


def dual_codebooks(calib_K, calib_V, rotations_K, rotations_V, bits: int):
    """Empirical Lloyd codebooks for K and for V, each pooled over all heads.

    calib_*: iterables of C x d arrays, one per (layer, head); rotations_*: the
    matching d x d rotations."""
    uk = np.concatenate([rotated_unit_coordinates(X, P) for X, P in zip(calib_K, rotations_K)])
    uv = np.concatenate([rotated_unit_coordinates(X, P) for X, P in zip(calib_V, rotations_V)])
    return lloyd_empirical(uk, bits), lloyd_empirical(uv, bits)
