"""Seeded synthetic inputs for the compressed-KV hot path.

This module draws random data only: Gaussian keys, values and queries with
outlier channels, the random orthogonal rotation Pi, the Gaussian QJL
projection S, calibration tokens and a Gaussian-mixture search corpus. It
holds none of the method's arithmetic (no rotation, quantisation, scoring or
softmax), so both the CUDA library's tests/benchmarks and the CPU oracle can
take their inputs from here without sharing any of the computation.

Streams are keyed by ``(seed, tag, ...)``:

====  ======================================
tag   stream
====  ======================================
0     Pi (random orthogonal rotation)
1     S (Gaussian QJL projection)
2     K
3     V
4     Q
5     calibration tokens
6     outlier-channel choice
7     mixture components / assignments
====  ======================================

CPU-sized workloads use NumPy ``default_rng(SeedSequence([seed, tag, ...]))``.
The 32-layer Llama-shaped decode workload (34 GB of bf16 K/V) is drawn on the
device with a ``torch.Generator`` seeded from the same SeedSequence; tests that
check it copy the sampled rows of those inputs to the host.

Workload shapes follow the five configurations the method is evaluated on:
a tiny single head (d=64, RoPE), an ESM-2-650M-shaped cache (33x20 heads,
d=64, 1024 tokens), a Llama-3.1-8B-shaped decode (32 layers, 32/8 heads,
d=128, 32768 tokens, batch 8), a 131072-token long-context sweep and a
1M x d=200 vector-search corpus.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

TAG_PI, TAG_S, TAG_K, TAG_V, TAG_Q, TAG_CALIB, TAG_OUTLIER, TAG_MIX = range(8)


def rng(seed: int, tag: int, *extra: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, tag, *extra]))


def torch_seed(seed: int, tag: int, *extra: int) -> int:
    return int(np.random.SeedSequence([seed, tag, *extra]).generate_state(1, dtype=np.uint64)[0] >> 1)


def random_rotation(d: int, seed: int = 0, *extra: int) -> np.ndarray:
    """A Haar-distributed d x d orthogonal matrix, stored as float32.

    Drawn as the Q factor of a standard-normal matrix with the signs of R's
    diagonal folded in (the usual way to make the QR draw Haar-uniform).
    """
    g = rng(seed, TAG_PI, d, *extra).standard_normal((d, d))
    q, r = np.linalg.qr(g)
    q = q * np.sign(np.diag(r))[None, :]
    return np.ascontiguousarray(q.astype(np.float32))


def gaussian_projection(d: int, seed: int = 0, rows: int | None = None) -> np.ndarray:
    """The QJL projection S: rows x d i.i.d. N(0,1), float32."""
    m = d if rows is None else rows
    return np.ascontiguousarray(rng(seed, TAG_S, d, m).standard_normal((m, d)).astype(np.float32))


def to_bf16(x) -> torch.Tensor:
    """Round a float array to bfloat16 (round-to-nearest-even), on its device."""
    t = x if isinstance(x, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16)


# --------------------------------------------------------------------------
# Workload 1: tiny single head with RoPE.
# --------------------------------------------------------------------------
@dataclasses.dataclass
class TinyHead:
    K: np.ndarray          # [N, d] float32, pre-RoPE
    V: np.ndarray          # [N, d] float32
    Q: np.ndarray          # [nq, d] float32, pre-RoPE
    Pi: np.ndarray         # [d, d] float32
    S: np.ndarray          # [d, d] float32
    k_pos: np.ndarray      # [N] int32
    q_pos: np.ndarray      # [nq] int32
    rope_base: float
    d: int


def tiny_head(seed: int = 0, d: int = 64, n: int = 256, nq: int = 4,
              spikes=(3, 17, 40), spike_scale: float = 20.0) -> TinyHead:
    """d=64, N=256 keys/values, 4 queries, fp32 N(0,1); channels 3, 17, 40 of
    K and V scaled x20 (outlier spikes); RoPE base 10000; keys at positions
    0..N-1, the queries at position N."""
    K = rng(seed, TAG_K).standard_normal((n, d))
    V = rng(seed, TAG_V).standard_normal((n, d))
    Q = rng(seed, TAG_Q).standard_normal((nq, d))
    for c in spikes:
        K[:, c] *= spike_scale
        V[:, c] *= spike_scale
    return TinyHead(K=K.astype(np.float32), V=V.astype(np.float32), Q=Q.astype(np.float32),
                    Pi=random_rotation(d, seed), S=gaussian_projection(d, seed),
                    k_pos=np.arange(n, dtype=np.int32), q_pos=np.full(nq, n, dtype=np.int32),
                    rope_base=10000.0, d=d)


# --------------------------------------------------------------------------
# Heavy-tailed outlier channels (lognormal magnitude, random sign).
# --------------------------------------------------------------------------
def _lognormal_channels(g: np.random.Generator, x: np.ndarray, chans: np.ndarray) -> None:
    shape = x.shape[:-1] + (len(chans),)
    mag = g.lognormal(mean=2.0, sigma=1.0, size=shape)
    sgn = np.where(g.random(shape) < 0.5, -1.0, 1.0)
    x[..., chans] = mag * sgn


# --------------------------------------------------------------------------
# Workload 2: ESM-2-650M-shaped cache.
# --------------------------------------------------------------------------
@dataclasses.dataclass
class EsmCache:
    K: torch.Tensor        # [L, H, N, d] bf16 (post-RoPE)
    V: torch.Tensor        # [L, H, N, d] bf16
    Q: torch.Tensor        # [L, H, NQ, d] bf16
    calib_K: torch.Tensor  # [L, H, C, d] bf16
    calib_V: torch.Tensor  # [L, H, C, d] bf16
    Pi: np.ndarray         # [d, d] float32 (random part of each head's rotation)
    S: np.ndarray          # [d, d] float32
    outlier_channels: np.ndarray  # [L, H, 4] int
    d: int


def esm_cache(seed: int = 0, layers: int = 33, heads: int = 20, d: int = 64, n: int = 1024,
              nq: int = 1024, calib: int = 256, n_outlier: int = 4) -> EsmCache:
    """33 layers x 20 heads x d=64, 1024 tokens, batch 1, bf16 K/V after RoPE.

    Every entry is N(0,1) except 4 of the 64 channels of each (layer, head),
    chosen without replacement, whose entries are lognormal(mu=2, sigma=1)
    with a random sign. 256 calibration tokens per (layer, head) are a
    separate draw from the same law (same outlier channels)."""
    chans = np.stack([np.stack([rng(seed, TAG_OUTLIER, l, h).choice(d, n_outlier, replace=False)
                                for h in range(heads)]) for l in range(layers)])
    out = {}
    for name, tag, rows in (("K", TAG_K, n), ("V", TAG_V, n), ("cK", TAG_CALIB, calib), ("cV", TAG_CALIB, calib)):
        arr = np.empty((layers, heads, rows, d), dtype=np.float32)
        for l in range(layers):
            for h in range(heads):
                sub = 0 if name in ("K", "V", "cK") else 1
                g = rng(seed, tag, l, h, sub)
                x = g.standard_normal((rows, d))
                _lognormal_channels(g, x, chans[l, h])
                arr[l, h] = x
        out[name] = to_bf16(arr)
    Q = to_bf16(rng(seed, TAG_Q).standard_normal((layers, heads, nq, d)).astype(np.float32))
    return EsmCache(K=out["K"], V=out["V"], Q=Q, calib_K=out["cK"], calib_V=out["cV"],
                    Pi=random_rotation(d, seed), S=gaussian_projection(d, seed),
                    outlier_channels=chans, d=d)


# --------------------------------------------------------------------------
# Workload 3: Llama-3.1-8B-shaped decode (device-side generation).
# --------------------------------------------------------------------------
@dataclasses.dataclass
class LlamaDecodeShape:
    layers: int = 32
    batch: int = 8
    hq: int = 32
    hkv: int = 8
    d: int = 128
    n_ctx: int = 32768
    outlier_frac: float = 0.02
    outlier_scale: float = 10.0

    @property
    def n_outlier(self) -> int:
        return int(round(self.outlier_frac * self.d))


def llama_outlier_channels(shape: LlamaDecodeShape, seed: int, layer: int) -> np.ndarray:
    """[hkv, n_outlier] channel ids scaled x10 in this layer (K and V alike)."""
    return np.stack([rng(seed, TAG_OUTLIER, layer, h).choice(shape.d, shape.n_outlier, replace=False)
                     for h in range(shape.hkv)])


def llama_layer_kv(shape: LlamaDecodeShape, seed: int, layer: int, device, which: str) -> torch.Tensor:
    """One layer's K ("K") or V ("V") as [batch, hkv, n_ctx, d] bf16 on `device`.

    N(0,1) entries; the layer's outlier channels (2% of d, per kv-head) are
    scaled x10. Drawn with a torch.Generator on `device`."""
    tag = TAG_K if which == "K" else TAG_V
    g = torch.Generator(device=device)
    g.manual_seed(torch_seed(seed, tag, layer))
    x = torch.randn((shape.batch, shape.hkv, shape.n_ctx, shape.d), generator=g, device=device,
                    dtype=torch.float32)
    chans = torch.as_tensor(llama_outlier_channels(shape, seed, layer), device=device)
    scale = torch.ones((shape.hkv, shape.d), device=device)
    scale.scatter_(1, chans, shape.outlier_scale)
    x.mul_(scale[None, :, None, :])
    return x.to(torch.bfloat16)


def llama_queries(shape: LlamaDecodeShape, seed: int, device) -> torch.Tensor:
    """[layers, batch, hq, d] bf16 N(0,1) decode queries."""
    g = torch.Generator(device=device)
    g.manual_seed(torch_seed(seed, TAG_Q))
    return torch.randn((shape.layers, shape.batch, shape.hq, shape.d), generator=g, device=device,
                       dtype=torch.float32).to(torch.bfloat16)


# --------------------------------------------------------------------------
# Workload 4: long-context sweep.
# --------------------------------------------------------------------------
@dataclasses.dataclass
class LongContext:
    K: torch.Tensor   # [1, hkv, N, d] bf16
    V: torch.Tensor
    Q: torch.Tensor   # [1, hq, d] bf16
    Pi: np.ndarray
    S: np.ndarray
    outlier_channels: np.ndarray  # [hkv, n_outlier]
    d: int


def long_context(seed: int = 0, n: int = 131072, hkv: int = 8, hq: int = 32, d: int = 128,
                 n_outlier: int = 8, device="cpu") -> LongContext:
    """1 layer, batch 1, 8 KV / 32 query heads, d=128, bf16 Gaussian K/V with
    heavy-tailed outlier channels as in the ESM-shaped cache (the same 1/16
    fraction of channels: 8 of 128, lognormal(2,1) with random sign)."""
    chans = np.stack([rng(seed, TAG_OUTLIER, 0, h).choice(d, n_outlier, replace=False) for h in range(hkv)])
    tensors = []
    for tag in (TAG_K, TAG_V):
        arr = np.empty((1, hkv, n, d), dtype=np.float32)
        for h in range(hkv):
            g = rng(seed, tag, 0, h)
            x = g.standard_normal((n, d))
            _lognormal_channels(g, x, chans[h])
            arr[0, h] = x
        tensors.append(to_bf16(arr).to(device))
    Q = to_bf16(rng(seed, TAG_Q).standard_normal((1, hq, d)).astype(np.float32)).to(device)
    return LongContext(K=tensors[0], V=tensors[1], Q=Q, Pi=random_rotation(d, seed),
                       S=gaussian_projection(d, seed), outlier_channels=chans, d=d)


# --------------------------------------------------------------------------
# Workload 5: vector search corpus (stand-in for GloVe d=200).
# --------------------------------------------------------------------------
@dataclasses.dataclass
class SearchCorpus:
    X: np.ndarray   # [n_db, d] float32, unit norm
    Q: np.ndarray   # [n_q, d] float32, unit norm
    Pi: np.ndarray
    S: np.ndarray
    d: int


def search_corpus(seed: int = 0, n_db: int = 1_000_000, n_q: int = 10_000, d: int = 200,
                  components: int = 100, spread: float = 0.5) -> SearchCorpus:
    """A 100-component equal-weight Gaussian mixture in d=200: component means
    ~ N(0, I), points = mean + 0.5 N(0, I), then L2-normalised. Queries are
    drawn the same way from the same components."""
    g = rng(seed, TAG_MIX)
    mu = g.standard_normal((components, d))

    def draw(count: int, sub: int) -> np.ndarray:
        gg = rng(seed, TAG_MIX, sub)
        out = np.empty((count, d), dtype=np.float32)
        step = 1 << 18
        for s in range(0, count, step):
            m = min(step, count - s)
            comp = gg.integers(0, components, m)
            x = mu[comp] + spread * gg.standard_normal((m, d))
            x /= np.linalg.norm(x, axis=1, keepdims=True)
            out[s:s + m] = x
        return out

    return SearchCorpus(X=draw(n_db, 1), Q=draw(n_q, 2), Pi=random_rotation(d, seed),
                        S=gaussian_projection(d, seed), d=d)
