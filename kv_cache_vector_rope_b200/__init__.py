"""B200-native compressed KV cache: TurboQuant-style 3-bit + QJL keys/values
and attention computed directly over the packed cache.

This package is a thin ctypes binding over ``libtq.so`` (C ABI declared in
``include/tq.h``). Every function here only marshals arguments — tensor
pointers, sizes, the current CUDA stream — and calls the library of the same
name; all arithmetic runs in the library's CUDA kernels (or, for
``tq_make_codebook``, its host C++ code). There is no Python or CPU fallback:
if the library is missing, importing the binding raises.

PyTorch is used for device memory and streams only.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtq.so")

TQ_OK, TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_CUDA, TQ_ERR_WORKSPACE = range(5)
TQ_F32, TQ_BF16 = 0, 1
TQ_DEV_BAD_CODEBOOK, TQ_DEV_BAD_POSITION, TQ_DEV_TIMEOUT = 0x1, 0x2, 0x4

_STATUS = {1: "TQ_ERR_INVALID_ARG", 2: "TQ_ERR_UNSUPPORTED", 3: "TQ_ERR_CUDA", 4: "TQ_ERR_WORKSPACE"}


class TQError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


class Layout(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("key_bits", ctypes.c_int32), ("value_bits", ctypes.c_int32)]


class _Planes(ctypes.Structure):
    _fields_ = [("idx", ctypes.c_void_p), ("sign", ctypes.c_void_p), ("norm", ctypes.c_void_p),
                ("rnorm", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I32, _I64, _F32, _SZ = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t

_SIGNATURES = {
    "tq_idx_row_bytes": (_I64, [_I32, _I32]),
    "tq_sign_words": (_I64, [_I32]),
    "tq_packed_bytes": (_I64, [ctypes.POINTER(Layout), _I64, _I32]),
    "tq_make_codebook": (ctypes.c_int, [_I32, _I32, _I32, _P, _I64, _P, _P, _P]),
    "tq_quantize_kv": (ctypes.c_int, [ctypes.POINTER(Layout), _I32, _P, ctypes.c_int, _I64, _I64, _P, _F32,
                                      _P, _I64, _I64, _P, _P, _P, ctypes.POINTER(_Planes), _P, _P]),
    "tq_decode_attention": (ctypes.c_int, [ctypes.POINTER(Layout), _P, ctypes.c_int, _I32, _I32, _I32, _I32, _I64,
                                           _I64, _P, _F32, ctypes.POINTER(_Planes), ctypes.POINTER(_Planes),
                                           _P, _P, _I64, _P, _P, _P, _F32, _P, ctypes.c_int, _P, _P, _SZ, _P, _P]),
    "tq_append_kv": (ctypes.c_int, [ctypes.POINTER(Layout), _I32, _P, ctypes.c_int, _I64, _I64, _P, _F32, _P, _P, _P, _P,
                                    ctypes.POINTER(_Planes), _I64, _I64, _P, _P]),
    "tq_decode_workspace_bytes": (_SZ, [ctypes.POINTER(Layout), _I32, _I32, _I32, _I32, _I64]),
    "tq_decode_attention_noalloc": (ctypes.c_int, [ctypes.POINTER(Layout), _P, ctypes.c_int, _I32, _I32, _I32, _I32,
                                                   _I64, _I64, _P, _F32, ctypes.POINTER(_Planes),
                                                   ctypes.POINTER(_Planes), _P, _P, _I64, _P, _P, _P, _F32, _P,
                                                   ctypes.c_int, _P, _P, _P]),
    "tq_dequantize": (ctypes.c_int, [ctypes.POINTER(Layout), _I32, _I64, ctypes.POINTER(_Planes), _P, _I64, _I64,
                                     _P, _P, _P, ctypes.c_int, _I64, _P]),
    "tq_dequantize_sign_mean": (ctypes.c_int, [ctypes.POINTER(Layout), _I32, _I64, ctypes.POINTER(_Planes), _P, _I64,
                                               _I64, _P, _F32, _P, ctypes.c_int, _I64, _P]),
    "tq_residual_mean": (ctypes.c_int, [_P, _I64, _P, _P, _I32, ctypes.POINTER(ctypes.c_double)]),
    "tq_search_topk": (ctypes.c_int, [ctypes.POINTER(Layout), _P, ctypes.c_int, _I32, ctypes.POINTER(_Planes), _I64,
                                      _P, _P, _P, _I32, _P, _P, _P, _SZ, _P]),
    "tq_search_merge_topk": (ctypes.c_int, [_I32, _I32, _P, _P, _I64, _P, _P, _I64, _P, _P, _P]),
    "tq_search_workspace_bytes": (_SZ, [ctypes.POINTER(Layout), _I32, _I64, _I32]),
    "tq_fit_rotation": (ctypes.c_int, [_I32, _P, _I64, _P, _P]),
    "tq_rotate_normalize": (ctypes.c_int, [_I32, _P, _I64, _P, _P, ctypes.POINTER(_I64)]),
    "tq_last_error_string": (ctypes.c_char_p, []),
    "tq_version": (ctypes.c_char_p, []),
    "tq_kernel_launches": (ctypes.c_uint64, []),
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libtq.so is not built ({LIB_PATH}); run `python kv_cache_vector_rope_b200/build.py` "
                          "(the CUDA library is the only implementation; there is no fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def exported_symbols() -> list[str]:
    return list(_SIGNATURES)


def _check(status: int) -> None:
    if status != TQ_OK:
        raise TQError(status, _lib.tq_last_error_string().decode())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        return t.data_ptr()
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return int(t)


def _dev(t: torch.Tensor, name: str) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    return t.data_ptr()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return TQ_F32
    if t.dtype == torch.bfloat16:
        return TQ_BF16
    raise ValueError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def layout(d: int, key_bits: int = 3, value_bits: int = 3) -> Layout:
    return Layout(d, key_bits, value_bits)


@dataclasses.dataclass
class Planes:
    """Packed planes of n vectors (torch tensors on one device)."""
    idx: torch.Tensor            # uint8 [n, d*bits/8]
    norm: torch.Tensor           # float32 [n]
    sign: torch.Tensor | None = None    # int32 [n, ceil(d/32)] (uint32 bit patterns)
    rnorm: torch.Tensor | None = None   # float32 [n]

    def c(self) -> _Planes:
        return _Planes(_ptr(self.idx), _ptr(self.sign), _ptr(self.norm), _ptr(self.rnorm))

    def rows(self, start: int, stop: int) -> "Planes":
        return Planes(self.idx[start:stop], self.norm[start:stop],
                      None if self.sign is None else self.sign[start:stop],
                      None if self.rnorm is None else self.rnorm[start:stop])

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.idx, self.norm, self.sign, self.rnorm)
                   if t is not None)


def tq_idx_row_bytes(d: int, bits: int) -> int:
    return int(_lib.tq_idx_row_bytes(d, bits))


def tq_sign_words(d: int) -> int:
    return int(_lib.tq_sign_words(d))


def tq_packed_bytes(lay: Layout, n_vectors: int, is_key: bool) -> int:
    return int(_lib.tq_packed_bytes(ctypes.byref(lay), n_vectors, int(is_key)))


def alloc_planes(n: int, d: int, bits: int, is_key: bool, device="cuda") -> Planes:
    """Allocates the planes of n vectors (allocation is PyTorch's)."""
    return Planes(idx=torch.empty((n, tq_idx_row_bytes(d, bits)), dtype=torch.uint8, device=device),
                  norm=torch.empty((n,), dtype=torch.float32, device=device),
                  sign=torch.empty((n, tq_sign_words(d)), dtype=torch.int32, device=device) if is_key else None,
                  rnorm=torch.empty((n,), dtype=torch.float32, device=device) if is_key else None)


def tq_make_codebook(d: int, bits: int, mode: int = 0, samples=None):
    """Lloyd-Max codebook (host). Returns (centroids, boundaries, mse) as float32 arrays and a float."""
    n = 1 << bits
    c = np.zeros(n, dtype=np.float32)
    t = np.zeros(max(n - 1, 1), dtype=np.float32)
    mse = ctypes.c_double(0.0)
    smp = None
    ns = 0
    if samples is not None:
        smp = np.ascontiguousarray(np.asarray(samples, dtype=np.float32).ravel())
        ns = smp.size
    _check(_lib.tq_make_codebook(d, bits, mode, _ptr(smp), ns, c.ctypes.data, t.ctypes.data, ctypes.byref(mse)))
    return c, t[:n - 1], float(mse.value)


def tq_quantize_kv(lay: Layout, is_key: bool, x: torch.Tensor, out: Planes, Pi: torch.Tensor,
                   centroids: torch.Tensor, boundaries: torch.Tensor, S: torch.Tensor | None = None,
                   positions: torch.Tensor | None = None, rope_base: float = 0.0,
                   vectors_per_pi: int = 1, pi_stride: int = 0, d_status: torch.Tensor | None = None,
                   stream=None) -> None:
    """Quantises the rows of x ([n, d], unit stride along d) into `out`."""
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be [n, d] with unit stride along d")
    _check(_lib.tq_quantize_kv(ctypes.byref(lay), int(is_key), _dev(x, "x"), _dtype_code(x), x.shape[0],
                               x.stride(0), _ptr(positions), float(rope_base), _dev(Pi, "Pi"), vectors_per_pi,
                               pi_stride, _ptr(S), _dev(centroids, "centroids"), _dev(boundaries, "boundaries"),
                               ctypes.byref(out.c()), _ptr(d_status), _stream(stream)))


def tq_append_kv(lay: Layout, is_key: bool, x: torch.Tensor, cache: Planes, ctx_stride: int, slot: int,
                 Pi: torch.Tensor, centroids: torch.Tensor, boundaries: torch.Tensor, S: torch.Tensor | None = None,
                 positions: torch.Tensor | None = None, rope_base: float = 0.0, d_status: torch.Tensor | None = None,
                 stream=None) -> None:
    """Quantises row s of x ([n_streams, d]) into cache row s * ctx_stride + slot."""
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be [n_streams, d] with unit stride along d")
    _check(_lib.tq_append_kv(ctypes.byref(lay), int(is_key), _dev(x, "x"), _dtype_code(x), x.shape[0], x.stride(0),
                             _ptr(positions), float(rope_base), _dev(Pi, "Pi"), _ptr(S), _dev(centroids, "centroids"),
                             _dev(boundaries, "boundaries"), ctypes.byref(cache.c()), ctx_stride, slot,
                             _ptr(d_status), _stream(stream)))


def tq_decode_workspace_bytes(lay: Layout, batch: int, hq: int, hkv: int, nq: int, n_ctx: int) -> int:
    return int(_lib.tq_decode_workspace_bytes(ctypes.byref(lay), batch, hq, hkv, nq, n_ctx))


def decode_workspace(lay: Layout, batch: int, hq: int, hkv: int, nq: int, n_ctx: int, device="cuda") -> torch.Tensor:
    n = tq_decode_workspace_bytes(lay, batch, hq, hkv, nq, n_ctx)
    return torch.empty((max(n, 256) + 255) // 256 * 256, dtype=torch.uint8, device=device)


def tq_decode_attention(lay: Layout, q: torch.Tensor, k: Planes, v: Planes, hkv: int, n_ctx: int,
                        PiK: torch.Tensor, PiV: torch.Tensor, S: torch.Tensor, cK: torch.Tensor, cV: torch.Tensor,
                        out: torch.Tensor, workspace: torch.Tensor, scale: float | None = None,
                        q_positions: torch.Tensor | None = None, rope_base: float = 0.0, pi_stride: int = 0,
                        ctx_stride: int = 0, scores_out: torch.Tensor | None = None,
                        d_status: torch.Tensor | None = None, stream=None) -> None:
    """Attention of q ([batch, hq, nq, d], contiguous) over packed K/V planes of [batch, hkv, ctx] rows."""
    if q.dim() != 4 or not q.is_contiguous():
        raise ValueError("q must be a contiguous [batch, hq, nq, d] tensor")
    if not out.is_contiguous():
        raise ValueError("out must be contiguous [batch, hq, nq, d]")
    batch, hq, nq, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    _check(_lib.tq_decode_attention(
        ctypes.byref(lay), _dev(q, "q"), _dtype_code(q), batch, hq, hkv, nq, n_ctx, ctx_stride,
        _ptr(q_positions), float(rope_base), ctypes.byref(k.c()), ctypes.byref(v.c()),
        _dev(PiK, "PiK"), _dev(PiV, "PiV"), pi_stride, _dev(S, "S"), _dev(cK, "cK"), _dev(cV, "cV"),
        float(scale), _dev(out, "out"), _dtype_code(out), _ptr(scores_out), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _ptr(d_status), _stream(stream)))


def tq_decode_attention_noalloc(lay: Layout, q: torch.Tensor, k: Planes, v: Planes, hkv: int, n_ctx: int,
                                PiK: torch.Tensor, PiV: torch.Tensor, S: torch.Tensor, cK: torch.Tensor,
                                cV: torch.Tensor, out: torch.Tensor, scale: float | None = None,
                                q_positions: torch.Tensor | None = None, rope_base: float = 0.0, pi_stride: int = 0,
                                ctx_stride: int = 0, scores_out: torch.Tensor | None = None,
                                d_status: torch.Tensor | None = None, stream=None) -> None:
    """tq_decode_attention with the library's fixed device scratch instead of a workspace.

    For callers that cannot allocate device memory at call time. Calls that
    overlap on the GPU share the scratch and must be serialised by the caller."""
    if q.dim() != 4 or not q.is_contiguous() or not out.is_contiguous():
        raise ValueError("q and out must be contiguous [batch, hq, nq, d] tensors")
    batch, hq, nq, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    _check(_lib.tq_decode_attention_noalloc(
        ctypes.byref(lay), _dev(q, "q"), _dtype_code(q), batch, hq, hkv, nq, n_ctx, ctx_stride,
        _ptr(q_positions), float(rope_base), ctypes.byref(k.c()), ctypes.byref(v.c()),
        _dev(PiK, "PiK"), _dev(PiV, "PiV"), pi_stride, _dev(S, "S"), _dev(cK, "cK"), _dev(cV, "cV"),
        float(scale), _dev(out, "out"), _dtype_code(out), _ptr(scores_out), _ptr(d_status), _stream(stream)))


def tq_dequantize(lay: Layout, is_key: bool, planes: Planes, n_vectors: int, Pi: torch.Tensor,
                  centroids: torch.Tensor, out: torch.Tensor, S: torch.Tensor | None = None,
                  vectors_per_pi: int = 1, pi_stride: int = 0, stream=None) -> None:
    if out.dim() != 2 or out.stride(1) != 1:
        raise ValueError("out must be [n, d] with unit stride along d")
    _check(_lib.tq_dequantize(ctypes.byref(lay), int(is_key), n_vectors, ctypes.byref(planes.c()),
                              _dev(Pi, "Pi"), vectors_per_pi, pi_stride, _ptr(S), _dev(centroids, "centroids"),
                              _dev(out, "out"), _dtype_code(out), out.stride(0), _stream(stream)))


def tq_dequantize_sign_mean(lay: Layout, is_key: bool, planes: Planes, n_vectors: int, Pi: torch.Tensor,
                            centroids: torch.Tensor, e_bar: float, out: torch.Tensor, vectors_per_pi: int = 1,
                            pi_stride: int = 0, stream=None) -> None:
    """x_tilde = Pi^T ||x|| (c[code] + e_bar (2 sign - 1)) for rows 0..n_vectors-1."""
    if out.dim() != 2 or out.stride(1) != 1:
        raise ValueError("out must be [n, d] with unit stride along d")
    _check(_lib.tq_dequantize_sign_mean(ctypes.byref(lay), int(is_key), n_vectors, ctypes.byref(planes.c()),
                                        _dev(Pi, "Pi"), vectors_per_pi, pi_stride, _dev(centroids, "centroids"),
                                        float(e_bar), _dev(out, "out"), _dtype_code(out), out.stride(0),
                                        _stream(stream)))


def tq_residual_mean(samples, centroids, boundaries, bits: int) -> float:
    """Mean |u - c[code(u)]| over host samples u (the e_bar of tq_dequantize_sign_mean)."""
    u = np.ascontiguousarray(np.asarray(samples, dtype=np.float32).ravel())
    c = np.ascontiguousarray(np.asarray(centroids, dtype=np.float32))
    t = np.ascontiguousarray(np.asarray(boundaries, dtype=np.float32))
    e = ctypes.c_double(0.0)
    _check(_lib.tq_residual_mean(u.ctypes.data, u.size, c.ctypes.data, t.ctypes.data, bits, ctypes.byref(e)))
    return float(e.value)


def tq_search_workspace_bytes(lay: Layout, n_queries: int, n_db: int, k: int) -> int:
    return int(_lib.tq_search_workspace_bytes(ctypes.byref(lay), n_queries, n_db, k))


def tq_search_topk(lay: Layout, q: torch.Tensor, db: Planes, n_db: int, Pi: torch.Tensor, S: torch.Tensor,
                   centroids: torch.Tensor, k: int, top_idx: torch.Tensor, top_scores: torch.Tensor,
                   workspace: torch.Tensor, stream=None) -> None:
    """k best corpus rows per query ([n_queries, d], contiguous) by estimated inner product."""
    if q.dim() != 2 or not q.is_contiguous():
        raise ValueError("q must be a contiguous [n_queries, d] tensor")
    _check(_lib.tq_search_topk(ctypes.byref(lay), _dev(q, "q"), _dtype_code(q), q.shape[0], ctypes.byref(db.c()),
                               n_db, _dev(Pi, "Pi"), _dev(S, "S"), _dev(centroids, "centroids"), k,
                               _dev(top_idx, "top_idx"), _dev(top_scores, "top_scores"), _dev(workspace, "workspace"),
                               workspace.numel() * workspace.element_size(), _stream(stream)))


def tq_search_merge_topk(idx_a: torch.Tensor, scores_a: torch.Tensor, offset_a: int, idx_b: torch.Tensor,
                         scores_b: torch.Tensor, offset_b: int, idx_out: torch.Tensor, scores_out: torch.Tensor,
                         stream=None) -> None:
    """Merges two [n_queries, k] top-k lists (ids shifted by their shard offsets) into idx_out / scores_out."""
    nq, k = idx_a.shape
    _check(_lib.tq_search_merge_topk(nq, k, _dev(idx_a, "idx_a"), _dev(scores_a, "scores_a"), offset_a,
                                     _dev(idx_b, "idx_b"), _dev(scores_b, "scores_b"), offset_b,
                                     _dev(idx_out, "idx_out"), _dev(scores_out, "scores_out"), _stream(stream)))


def tq_fit_rotation(X, Pi_rand) -> np.ndarray:
    """Per-head rotation Pi_rand V^T from calibration rows X ([n, d], host)."""
    X = np.ascontiguousarray(np.asarray(X, dtype=np.float32))
    P = np.ascontiguousarray(np.asarray(Pi_rand, dtype=np.float32))
    n, d = X.shape
    out = np.zeros((d, d), dtype=np.float32)
    _check(_lib.tq_fit_rotation(d, X.ctypes.data, n, P.ctypes.data, out.ctypes.data))
    return out


def tq_rotate_normalize(X, Pi) -> np.ndarray:
    """Coordinates of Pi x / ||x|| for the non-zero rows of X (host)."""
    X = np.ascontiguousarray(np.asarray(X, dtype=np.float32))
    P = np.ascontiguousarray(np.asarray(Pi, dtype=np.float32))
    n, d = X.shape
    out = np.zeros((n, d), dtype=np.float32)
    m = ctypes.c_int64(0)
    _check(_lib.tq_rotate_normalize(d, X.ctypes.data, n, P.ctypes.data, out.ctypes.data, ctypes.byref(m)))
    return out[:m.value]


def tq_last_error_string() -> str:
    return _lib.tq_last_error_string().decode()


def tq_version() -> str:
    return _lib.tq_version().decode()


def tq_kernel_launches() -> int:
    """Kernels the library has launched (or captured) since it was loaded."""
    return int(_lib.tq_kernel_launches())
