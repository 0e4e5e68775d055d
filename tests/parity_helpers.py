"""Comparison rules between the CUDA path and the CPU oracle.

Tolerances (the method fixes no precision; these readings are the parity bar):
* packed codes: bit-exact except coordinates whose oracle value y lies within
  1e-5 (unit-direction units) of a threshold; mismatch rate <= 1e-4.
* QJL sign bits: bit-exact except projections with |(S r)_m| < 1e-5, and
  except vectors that already have an in-window code mismatch (their residual
  differs by a centroid gap).
* fp16 norms: equal, or one fp16 ulp apart (rounding of a value computed in a
  different order); the count is reported.
* attention: per (sequence, query head) ||o_gpu - o_ref||_inf <= 1e-3 ||o_ref||_inf
  and |lse_gpu - lse_ref| <= 1e-3 max(1, max_j |s_j|).
"""
from __future__ import annotations

import numpy as np

from oracle import turboquant_oracle as o

CODE_WINDOW = 1e-5
MAX_MISMATCH_RATE = 1e-4
ATTN_RTOL = 1e-3


def f16_bits_to_f64(bits) -> np.ndarray:
    return np.asarray(bits).astype(np.uint16).view(np.float16).astype(np.float64)


def code_window_mask(y, thresholds) -> np.ndarray:
    """True where y is within CODE_WINDOW of some threshold."""
    t = np.asarray(thresholds, dtype=np.float64)
    return np.min(np.abs(np.asarray(y)[..., None] - t), axis=-1) < CODE_WINDOW


def compare_codes(gpu_packed, ref: o.Quantized, bits: int, thresholds, d: int = 128) -> dict:
    gpu_codes = o.unpack_codes(gpu_packed, bits, d)
    mism = gpu_codes != ref.codes
    inwin = code_window_mask(ref.y, thresholds)
    bad = mism & ~inwin
    return {"n": int(mism.size), "mismatch": int(mism.sum()), "outside_window": int(bad.sum()),
            "rate": float(mism.sum()) / max(1, mism.size), "vec_mismatch": mism.any(axis=1)}


def compare_fp16(gpu_bits, ref_values) -> dict:
    g = f16_bits_to_f64(gpu_bits)
    r = np.asarray(ref_values, dtype=np.float64)
    gb = np.asarray(gpu_bits).astype(np.uint16).astype(np.int64)
    rb = r.astype(np.float16).view(np.uint16).astype(np.int64)
    ulp = np.abs(gb - rb)
    return {"equal": int((g == r).sum()), "one_ulp": int((ulp == 1).sum()), "worse": int((ulp > 1).sum())}


def compare_signs(gpu_packed, ref: o.Quantized, skip_vectors=None) -> dict:
    gpu = o.unpack_signs(gpu_packed, ref.qjl_signs.shape[1])
    mism = gpu != ref.qjl_signs
    ok = np.abs(ref.qjl_proj) < CODE_WINDOW
    if skip_vectors is not None:
        ok = ok | np.asarray(skip_vectors)[:, None]
    return {"mismatch": int(mism.sum()), "outside_window": int((mism & ~ok).sum()),
            "n": int(mism.size)}


def attention_ok(o_gpu, o_ref, lse_gpu=None, lse_ref=None, max_abs_score=None) -> tuple[bool, float]:
    """Returns (all within tolerance, worst relative error)."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    den = np.maximum(np.abs(o_ref).max(axis=-1), 1e-30)
    rel = np.abs(o_gpu - o_ref).max(axis=-1) / den
    worst = float(rel.max()) if rel.size else 0.0
    ok = bool(np.all(rel <= ATTN_RTOL))
    if lse_gpu is not None:
        scale = np.maximum(1.0, np.asarray(max_abs_score, dtype=np.float64))
        lrel = np.abs(np.asarray(lse_gpu, dtype=np.float64) - np.asarray(lse_ref)) / scale
        ok = ok and bool(np.all(lrel <= ATTN_RTOL))
        worst = max(worst, float(lrel.max()) if lrel.size else 0.0)
    return ok, worst
