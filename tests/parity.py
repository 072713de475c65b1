"""Acceptance rules for the CUDA path against the CPU oracle (test infrastructure).

Tolerances (the SignRot build's stated acceptance bar):
  * fp32 rotation: per-token relative L2 error <= 2e-3 and max absolute error <= 1e-2;
  * per-token scale within 1e-5 relative; zero-point exact, except at a rounding tie of
    -lo/scale, where it may differ by exactly 1;
  * INT4 codes bit-exact except at rounding ties: a code may differ by 1 only where the
    oracle's pre-round value y/scale + zero lies within TIE_EPS of a half-integer, and such
    codes may be at most 1e-4 of all elements (rounded up to a whole element);
  * calibration index k, its signed value x_k and the sign vector s exactly.

A token whose zero-point took the other side of a tie is compared against the oracle's codes
recomputed with that zero (both are correct roundings of the same tie).
"""
from __future__ import annotations

import math

import numpy as np

from oracle import signrot_oracle as o

ROT_REL_L2 = 2e-3
ROT_MAX_ABS = 1e-2
SCALE_REL = 1e-5
TIE_EPS = 1e-3
TIE_FRAC = 1e-4


def _half_dist(v: np.ndarray) -> np.ndarray:
    return np.abs(v - np.floor(v) - 0.5)


def check_rotation(y_gpu: np.ndarray, y_ref: np.ndarray) -> dict:
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    num = np.linalg.norm(y_gpu - y_ref, axis=1)
    den = np.maximum(np.linalg.norm(y_ref, axis=1), 1e-30)
    rel = num / den
    mx = float(np.abs(y_gpu - y_ref).max()) if y_ref.size else 0.0
    assert (rel <= ROT_REL_L2).all(), f"per-token rel L2 {rel.max():.3e} > {ROT_REL_L2}"
    assert mx <= ROT_MAX_ABS, f"max abs error {mx:.3e} > {ROT_MAX_ABS}"
    return {"rel_l2_max": float(rel.max()) if rel.size else 0.0, "max_abs": mx}


def check_quant(q_gpu: np.ndarray, scale_gpu: np.ndarray, zero_gpu: np.ndarray, y_ref: np.ndarray,
                clip: float = 1.0) -> dict:
    T, n = y_ref.shape
    codes_ref, scale_ref, zero_ref = o.quantize_asym(y_ref, clip=clip)
    vpre, zpre = o.asym_preround(y_ref, clip=clip)
    codes_gpu = o.unpack_nibbles(np.asarray(q_gpu, dtype=np.uint8).reshape(T, n // 2))
    scale_gpu = np.asarray(scale_gpu, dtype=np.float32)
    zero_gpu = np.asarray(zero_gpu, dtype=np.float32)

    srel = np.abs(scale_gpu.astype(np.float64) - scale_ref) / np.abs(scale_ref)
    assert (srel <= SCALE_REL).all(), f"scale rel err {srel.max():.3e} > {SCALE_REL}"

    zdiff = zero_gpu.astype(np.float64) - zero_ref
    ztie = _half_dist(zpre.astype(np.float64)) < TIE_EPS
    bad = ~((zdiff == 0) | ((np.abs(zdiff) == 1) & ztie))
    assert not bad.any(), f"zero mismatch on tokens {np.flatnonzero(bad)[:8]}: {zero_gpu[bad][:4]} vs {zero_ref[bad][:4]}"
    shifted = np.flatnonzero(zdiff != 0)
    if shifted.size:  # the other side of a zero-point tie: redo the codes with the GPU's zero
        y32 = y_ref.astype(np.float32)
        for t in shifted:
            v = np.rint(y32[t] / scale_ref[t]) + zero_gpu[t]
            codes_ref[t] = np.clip(v, 0, 15).astype(np.uint8)
            vpre[t] = y32[t] / scale_ref[t] + zero_gpu[t]

    diff = codes_gpu.astype(np.int32) - codes_ref.astype(np.int32)
    mism = diff != 0
    tie = _half_dist(vpre.astype(np.float64)) < TIE_EPS
    hard = mism & ~((np.abs(diff) == 1) & tie)
    assert not hard.any(), (f"{int(hard.sum())} code mismatches away from ties, first at "
                            f"{np.argwhere(hard)[:4].tolist()}")
    allowed = math.ceil(TIE_FRAC * T * n)
    assert int(mism.sum()) <= allowed, f"{int(mism.sum())} tie mismatches > {allowed}"
    return {"code_mismatches": int(mism.sum()), "zero_ties": int(shifted.size),
            "scale_rel_max": float(srel.max()) if srel.size else 0.0}
