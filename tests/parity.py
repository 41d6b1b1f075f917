"""Comparison rules between the CUDA library and the oracle.

Tolerances (stated once, used by every GPU test):

CODE_BAND   A code may differ from the oracle's only if the oracle's u_i lies
            within 1e-6 * sigma_d of a boundary (sigma_d = 1/sqrt(d), the
            coordinate scale); such coordinates are "excused".
SIGN_BAND   A sign may differ only if |(S r)_i| <= 1e-6 ||r||, or if a code of
            the same vector was excused (its residual then differs).
EXCUSED_CAP Excused differences must stay below 1e-5 of all coordinates.
NORM_RTOL   ||x||: 1e-6 relative (fp64 accumulation, one fp32 rounding; RoPE'd
            inputs add one fp32 rounding per element).
RNORM_RTOL  ||r||: 2e-5 relative — the fp32 rotation errs by at most ~3e-7 ||x||
            per coordinate, and ||r|| is ~0.1-0.2 ||x|| at 2-4 bits.
SCORE rule  |s_gpu - s_ref| <= 1e-4 * max(|s_ref|, ||q|| ||k|| / d), with the
            oracle scoring the GPU's own planes (identical codes).
OUT rule    max |out_gpu - out_ref| <= 2e-3, plus half the bf16 spacing at the
            larger of |out_gpu|, |out_ref| for bf16 outputs (rounding to bf16 is
            part of producing a bf16 output); oracle again on the GPU's planes.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from oracle import attention as oa
from oracle import quantize as oq

CODE_BAND = 1e-6
SIGN_BAND = 1e-6
EXCUSED_CAP = 1e-5
NORM_RTOL = 1e-6
RNORM_RTOL = 2e-5
SCORE_RTOL = 1e-4
OUT_ATOL = 2e-3


def host_planes(p) -> dict:
    out = {"idx": p.idx.cpu().numpy(), "norm": p.norm.cpu().numpy()}
    if p.sign is not None:
        out["sign"] = p.sign.cpu().numpy().view(np.uint32)
        out["rnorm"] = p.rnorm.cpu().numpy()
    return out


def compare_quantized(gpu: dict, ref: oq.Quantized, d: int, bits: int, is_key: bool) -> dict:
    """Applies the band rules; raises AssertionError on any unexcused difference."""
    n = ref.codes.shape[0]
    codes = oq.unpack_codes(gpu["idx"], bits, d)
    sigma = 1.0 / math.sqrt(d)
    diff = codes != ref.codes
    excused_code = diff & (ref.code_margin <= CODE_BAND * sigma)
    bad_code = diff & ~excused_code
    assert not bad_code.any(), f"{int(bad_code.sum())} codes differ outside the band, e.g. {np.argwhere(bad_code)[:5]}"
    vec_excused = excused_code.any(axis=1)
    stats = {"coords": int(codes.size), "excused_codes": int(excused_code.sum())}
    nrm_err = np.abs(gpu["norm"].astype(np.float64) - ref.norm64) / np.maximum(ref.norm64, 1e-30)
    assert np.all((nrm_err <= NORM_RTOL) | (ref.norm64 == 0)), f"norm rel err {nrm_err.max()}"
    assert np.all(gpu["norm"][ref.norm64 == 0] == 0)
    if is_key:
        signs = oq.unpack_signs(gpu["sign"], d)
        sd = signs != ref.signs
        near = np.abs(ref.p) <= SIGN_BAND * ref.rnorm64[:, None]
        excused_sign = sd & (near | vec_excused[:, None])
        bad_sign = sd & ~excused_sign
        assert not bad_sign.any(), f"{int(bad_sign.sum())} signs differ outside the band, e.g. {np.argwhere(bad_sign)[:5]}"
        # pad bits of the last word are zero
        if d % 32:
            assert np.all((gpu["sign"][:, -1] >> np.uint32(d % 32)) == 0)
        rn_err = np.abs(gpu["rnorm"].astype(np.float64) - ref.rnorm64) / np.maximum(ref.rnorm64, 1e-30)
        ok = (rn_err <= RNORM_RTOL) | vec_excused | (ref.rnorm64 == 0)
        assert np.all(ok), f"rnorm rel err {rn_err[~ok].max()}"
        stats["excused_signs"] = int(excused_sign.sum())
        stats["rnorm_max_rel"] = float(rn_err[~vec_excused].max()) if (~vec_excused).any() else 0.0
    total = stats["excused_codes"] + stats.get("excused_signs", 0)
    assert total <= EXCUSED_CAP * codes.size + 0, f"excused {total} of {codes.size}"
    stats["norm_max_rel"] = float(nrm_err.max())
    return stats


def key_planes(h: dict, bits: int) -> oa.KeyPlanes:
    return oa.KeyPlanes(h["idx"], h["sign"], h["norm"], h["rnorm"], bits)


def value_planes(h: dict, bits: int) -> oa.ValuePlanes:
    return oa.ValuePlanes(h["idx"], h["norm"], bits)


# Worst ratios against the literal tolerances (score: 1e-4 * |s_ref| alone, over
# the scores with |s_ref| >= the typical scale, where a relative bound means
# something; fp32 outputs: 2e-3 max-abs; bf16 outputs: the error over 2e-3 plus
# half the bf16 spacing, the rounding a bf16 output cannot avoid).
# Collected by every check and printed at the end of the session.
LITERAL = {"score_rel": 0.0, "score_rel_all": 0.0, "out_abs_f32": 0.0, "out_bf16_vs_rounding": 0.0, "checks": 0}


def check_scores(gpu_scores: np.ndarray, ref_scores: np.ndarray, q_norm: np.ndarray, k_norm: np.ndarray, d: int):
    """The SCORE rule on [nq, N] score matrices; returns the worst ratio to the bound."""
    typical = q_norm[:, None] * k_norm[None, :].astype(np.float64) / d
    bound = SCORE_RTOL * np.maximum(np.abs(ref_scores), typical)
    err = np.abs(gpu_scores.astype(np.float64) - ref_scores)
    worst = float((err / np.maximum(bound, 1e-300)).max())
    rel = err / np.maximum(SCORE_RTOL * np.abs(ref_scores), 1e-300)
    big = np.abs(ref_scores) >= typical
    if big.any():
        LITERAL["score_rel"] = max(LITERAL["score_rel"], float(rel[big].max()))
    LITERAL["score_rel_all"] = max(LITERAL["score_rel_all"], float(rel.max()))
    LITERAL["checks"] += 1
    assert np.all(err <= bound), f"score error {err.max()} exceeds bound (worst ratio {worst})"
    return worst


def check_out(gpu_out: torch.Tensor, ref: np.ndarray) -> float:
    g = gpu_out.float().cpu().numpy().astype(np.float64)
    tol = OUT_ATOL
    if gpu_out.dtype == torch.bfloat16:
        # bf16 keeps 8 significant bits: spacing 2^(floor(log2|x|) - 7). Use the
        # larger magnitude of the pair, since rounding may cross a power of two.
        m = np.maximum(np.abs(ref), np.abs(g))
        spacing = np.exp2(np.floor(np.log2(np.maximum(m, 1e-30))) - 7)
        tol = OUT_ATOL + 0.5 * spacing
    err = np.abs(g - ref)
    if gpu_out.dtype == torch.bfloat16:
        LITERAL["out_bf16_vs_rounding"] = max(LITERAL["out_bf16_vs_rounding"], float((err / tol).max()))
    else:
        LITERAL["out_abs_f32"] = max(LITERAL["out_abs_f32"], float(err.max()) / OUT_ATOL)
    LITERAL["checks"] += 1
    assert np.all(err <= tol), f"output max abs error {err.max()}"
    return float(err.max())


def device_codebook(book_c: np.ndarray, book_t: np.ndarray, device="cuda"):
    return (torch.as_tensor(np.asarray(book_c, dtype=np.float32), device=device),
            torch.as_tensor(np.asarray(book_t, dtype=np.float32), device=device))
