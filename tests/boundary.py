"""Inputs built to land on or beside the quantiser's decision points.

Test infrastructure (CPU, fp64). A bf16 row x is moved, one bf16 step of one
coordinate at a time, until a chosen quantity reaches its target:

  * code rows: u_i = (Pi x)_i / ||x|| at t_j + delta * sigma_d, with t_j a
    decision boundary of the codebook and sigma_d = 1/sqrt(d);
  * sign rows (keys): p_i = (S r)_i at delta * ||r||, r = Pi x - ||x|| c[codes];
  * wide rows: one channel scaled x1e4 (extreme dynamic range).

Rows carry a few coordinates of tiny magnitude (1e-2 down to 1e-12) whose bf16
steps are fine enough to reach a target to fp64 resolution. Every quantity is
re-evaluated exactly (fp64) after each move, so a row's true distance from
its decision point is known; the tests read it back from the oracle.
"""
from __future__ import annotations

import numpy as np
import torch

_TINY = (1e-2, 1e-4, 1e-6, 1e-8, 1e-10, 1e-12)


def to_bf16(x) -> np.ndarray:
    """Round to the nearest bf16 (ties to even), returned as float64."""
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


def _candidates(x: np.ndarray, steps: int = 8) -> np.ndarray:
    """[d, 2*steps] bf16 values reached from each coordinate by +-1..steps bf16 spacings."""
    mag = np.maximum(np.abs(x), 1e-30)
    ulp = np.exp2(np.floor(np.log2(mag)) - 7)
    s = np.concatenate([-np.arange(steps, 0, -1), np.arange(1, steps + 1)]).astype(np.float64)
    return to_bf16(x[:, None] + ulp[:, None] * s[None, :])


def _seed_row(rg, d, scale=1.0):
    x = rg.standard_normal(d) * scale
    tiny = rg.choice(d, len(_TINY), replace=False)
    x[tiny] = np.asarray(_TINY) * np.where(rg.random(len(_TINY)) < 0.5, -1.0, 1.0)
    return to_bf16(x)


def _descend(x, value_of_move, current, iters=600):
    """Greedy: apply the single-coordinate bf16 move that most reduces |f - target|."""
    for _ in range(iters):
        cand = _candidates(x)
        f = value_of_move(x, cand)                # [d, m] |f - target| after each move
        k, m = np.unravel_index(np.argmin(f), f.shape)
        if not f[k, m] < current:
            break
        x = x.copy()
        x[k] = cand[k, m]
        current = f[k, m]
    return x, current


def _tol(delta):
    return max(1e-3 * abs(delta), 1e-11)


def code_row(rg, Pi, boundary, delta_sigma, i, iters=600, attempts=6):
    """A bf16 row whose u_i sits at boundary + delta_sigma / sqrt(d)."""
    d = Pi.shape[0]
    sigma = 1.0 / np.sqrt(d)
    target = boundary + delta_sigma * sigma

    def f_move(x, cand):
        y = Pi[i] @ x
        n2 = np.sum(x * x)
        dlt = cand - x[:, None]
        y2 = y + Pi[i][:, None] * dlt
        n2b = n2 + 2 * x[:, None] * dlt + dlt * dlt
        return np.abs(y2 / np.sqrt(n2b) - target)

    best = None
    for _ in range(attempts):
        x = _seed_row(rg, d)
        k0 = int(np.argmax(np.abs(Pi[i])))
        for _ in range(8):                        # coarse: solve for the largest weight
            n = np.sqrt(np.sum(x * x))
            x[k0] = to_bf16(x[k0] + (target * n - Pi[i] @ x) / Pi[i, k0])
        cur = abs((Pi[i] @ x) / np.sqrt(np.sum(x * x)) - target)
        x, cur = _descend(x, f_move, cur, iters)
        if best is None or cur < best[1]:
            best = (x, cur)
        if cur <= _tol(delta_sigma) * sigma:
            break
    return best[0].astype(np.float32)


def sign_row(rg, Pi, S, centroids, boundaries, delta, i, iters=600, attempts=12):
    """A bf16 row whose projected residual (S r)_i sits at delta * ||r||.

    The residual r = Pi x - ||x|| c[codes] depends on the codes, so every
    candidate move is first ranked with the codes held fixed, then checked
    exactly; a move that changes a code is taken only if it still improves the
    exact distance."""
    d = Pi.shape[0]
    c = np.asarray(centroids, dtype=np.float64)
    t = np.asarray(boundaries, dtype=np.float64)
    w = S[i] @ Pi                                 # p_i = w.x - ||x|| (S_i . c[codes])

    def exact(x):
        n = np.sqrt(np.sum(x * x))
        y = Pi @ x
        codes = np.searchsorted(t, y / n, side="right")
        r = y - n * c[codes]
        rn = np.sqrt(np.sum(r * r))
        return abs(S[i] @ r - delta * rn) / max(rn, 1e-300), codes

    best = None
    for _ in range(attempts):
        x = _seed_row(rg, d)
        cur, codes = exact(x)
        for _ in range(iters):
            n = np.sqrt(np.sum(x * x))
            y = Pi @ x
            r = y - n * c[codes]
            rn = np.sqrt(np.sum(r * r))
            a = S[i] @ c[codes]
            cand = _candidates(x)
            dlt = cand - x[:, None]
            n2b = np.sum(x * x) + 2 * x[:, None] * dlt + dlt * dlt
            f = np.abs((w @ x) + w[:, None] * dlt - np.sqrt(n2b) * a - delta * rn) / rn
            moved = False
            for flat in np.argsort(f, axis=None)[:64]:
                k, m = np.unravel_index(flat, f.shape)
                if not f[k, m] < cur:
                    break
                x2 = x.copy()
                x2[k] = cand[k, m]
                e2, c2 = exact(x2)
                if e2 < cur:
                    x, cur, codes, moved = x2, e2, c2, True
                    break
            if not moved:
                break
        if best is None or cur < best[1]:
            best = (x, cur)
        if cur <= _tol(delta):
            break
    return best[0].astype(np.float32)


def wide_rows(rg, d, n, factor=1e4):
    """bf16 N(0,1) rows with one random channel of magnitude >= factor / 2."""
    X = rg.standard_normal((n, d))
    ch = rg.integers(0, d, n)
    z = X[np.arange(n), ch]
    X[np.arange(n), ch] = factor * np.sign(z) * np.maximum(np.abs(z), 0.5)
    return to_bf16(X).astype(np.float32)


DELTAS = (0.0, 1e-9, -1e-9, 1e-7, -1e-7, 1e-6, -1e-6, 2e-6, -2e-6)


def build(d, bits, Pi, S, centroids, boundaries, seed=0, sign_coords=4, wide=64):
    """Code rows for every boundary and delta, sign rows (keys), wide rows.

    Returns (X [n, d] float32 bf16-exact, kind [n] str, delta [n] float,
    coord [n] int: the targeted coordinate, target [n] float: the boundary
    value for code rows)."""
    rg = np.random.default_rng(seed)
    rows, kind, dl, co, tg = [], [], [], [], []
    for tb in np.asarray(boundaries, dtype=np.float64):
        for ds in DELTAS:
            i = int(rg.integers(0, d))
            rows.append(code_row(rg, Pi, tb, ds, i))
            kind.append("code")
            dl.append(ds)
            co.append(i)
            tg.append(tb)
    if S is not None:
        for ds in DELTAS:
            for _ in range(sign_coords):
                i = int(rg.integers(0, d))
                rows.append(sign_row(rg, Pi, S, centroids, boundaries, ds, i))
                kind.append("sign")
                dl.append(ds)
                co.append(i)
                tg.append(np.nan)
    W = wide_rows(rg, d, wide)
    rows.extend(W)
    kind.extend(["wide"] * wide)
    dl.extend([np.nan] * wide)
    co.extend([-1] * wide)
    tg.extend([np.nan] * wide)
    return (np.stack(rows).astype(np.float32), np.asarray(kind), np.asarray(dl), np.asarray(co),
            np.asarray(tg))
