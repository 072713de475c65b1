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

Conditioning. The quantizer's inputs are differences of fp32 values: hi - lo, and y / scale with
|y| / scale up to |zero|. Where a row's spread is tiny next to its magnitude (a massive outlier on
a very short row, e.g. n = 2), fp32 rounding of y alone moves the pre-round values by more than
the tie window. Given the input rows (x64), the checker bounds that rounding per token,
    delta_t = (log2(M) + F - 1 + 2) * 2^-24 * ||x_t||_1 / sqrt(n) + max_j |y_tj| * 2^-24
(each output is a sum with at most log2(M) + F - 1 additions on any path, every partial sum is
bounded by ||x_t||_1, plus the 1/sqrt(n) product and the final rounding), and calls a token
ill-conditioned only when that bound alone, in code units (delta_t / scale_t), exceeds TIE_EPS.
Every other token is held to the bar above unwidened: windows of TIE_EPS, scale within 1e-5, and
its code mismatches counted toward TIE_FRAC. An ill-conditioned token's windows are widened by
its bound instead, and every one of its codes must dequantize to within half a step (+ delta_t)
of the exact rotation; the number of such tokens is reported.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

from oracle import signrot_oracle as o

ROT_REL_L2 = 2e-3
ROT_MAX_ABS = 1e-2
SCALE_REL = 1e-5
TIE_EPS = 1e-3
TIE_FRAC = 1e-4
ILL_MAX_N = 1024
U32 = 2.0 ** -24


def _half_dist(v: np.ndarray) -> np.ndarray:
    return np.abs(v - np.floor(v) - 0.5)


def fp32_rotation_bound(x64: np.ndarray, acc_eps: float = U32) -> np.ndarray:
    """Per-token bound on |y_fp32 - y_exact| for the rotation accumulated with unit roundoff
    acc_eps (2^-24: fp32 sums; 2^-53: the fp64 sums of the generic kernel) and rounded once to
    fp32 at the end (the max |y| * 2^-24 term check_quant adds)."""
    T, n = x64.shape
    F, M = o.factor_n(n)
    S = int(round(math.log2(M))) + (F - 1) + 2
    return S * acc_eps * np.abs(x64).sum(axis=1) / math.sqrt(n)


def oracle_sign(x64: np.ndarray, d: np.ndarray) -> np.ndarray:
    """The sign vector the oracle derives on its own from calibration rows x64: the reference of
    every parity test takes s from here, never from the CUDA path."""
    k, xk = o.calibrate(x64)
    return o.build_sign(x64.shape[1], k, xk, d)


def check_rotation(y_gpu: np.ndarray, y_ref: np.ndarray) -> dict:
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    num = np.linalg.norm(y_gpu - y_ref, axis=1)
    den = np.maximum(np.linalg.norm(y_ref, axis=1), 1e-30)
    rel = num / den
    mx = float(np.abs(y_gpu - y_ref).max()) if y_ref.size else 0.0
    assert (rel <= ROT_REL_L2).all(), f"per-token rel L2 {rel.max():.3e} > {ROT_REL_L2}"
    assert mx <= ROT_MAX_ABS, f"max abs error {mx:.3e} > {ROT_MAX_ABS}"
    return {"rel_l2_max": float(rel.max()) if rel.size else 0.0, "max_abs": mx}


def decode_codes(q: np.ndarray, T: int, n: int, bits: int = 4, sym: bool = False) -> np.ndarray:
    """Unpack the library's code layout to one int32 code per element: bits 4 -> two per byte
    (element 2i in the low nibble; two's complement nibbles on the symmetric grid), bits 8 -> one
    per byte (int8 on the symmetric grid)."""
    q = np.asarray(q)
    if bits == 8:
        flat = q.reshape(T, n)
        return flat.view(np.int8).astype(np.int32) if sym else flat.view(np.uint8).astype(np.int32)
    nib = o.unpack_nibbles(q.view(np.uint8).reshape(T, n // 2)).astype(np.int32)
    return ((nib ^ 8) - 8) if sym else nib


def check_quant(q_gpu: np.ndarray, scale_gpu: np.ndarray, zero_gpu: np.ndarray | None, y_ref: np.ndarray,
                clip: float = 1.0, x64: np.ndarray | None = None, bits: int = 4, sym: bool = False,
                allow_ill: bool | None = None, acc_eps: float = U32) -> dict:
    """Codes, scale and zero-point against the oracle's grid: asymmetric (codes 0 .. 2^bits - 1,
    fp32 zero-point) or, with sym, symmetric (codes -L .. L, L = 2^(bits-1) - 1, no zero-point).

    Without x64 every token is held to the bar as stated; with the input rows, tokens whose fp32
    rotation bound alone exceeds the tie window are checked as ill-conditioned (module doc).
    allow_ill (default: only for n < ILL_MAX_N, or an 8-bit grid) says whether such tokens may occur
    at all: 4-bit rows of ILL_MAX_N channels or more never leave the stated bar. acc_eps is the unit roundoff of the
    kernel's accumulation (fp32 unless the shape runs on the fp64-accumulating generic kernel)."""
    T, n = y_ref.shape
    y32 = y_ref.astype(np.float32)
    if sym:
        L = 2 ** (bits - 1) - 1
        codes_ref, scale_ref = o.quantize_sym(y_ref, bits=bits)
        codes_ref = codes_ref.astype(np.int32)
        zero_ref = np.zeros(T, dtype=np.float32)
        with np.errstate(divide="ignore", invalid="ignore"):
            vpre = y32 / scale_ref[:, None]
        zpre = np.zeros(T, dtype=np.float32)
        code_min, code_max = -L, L
        lo_c = -np.abs(y32).max(axis=1).astype(np.float64)
        hi_c = -lo_c
        zero_gpu = np.zeros(T, dtype=np.float32)
    else:
        codes_ref, scale_ref, zero_ref = o.quantize_asym(y_ref, bits=bits, clip=clip)
        codes_ref = codes_ref.astype(np.int32)
        vpre, zpre = o.asym_preround(y_ref, bits=bits, clip=clip)
        code_min, code_max = 0, 2 ** bits - 1
        lo_c = y32.min(axis=1).astype(np.float64) * clip
        hi_c = y32.max(axis=1).astype(np.float64) * clip
        zero_gpu = np.asarray(zero_gpu, dtype=np.float32)
    codes_gpu = decode_codes(q_gpu, T, n, bits, sym)
    scale_gpu = np.asarray(scale_gpu, dtype=np.float32)
    rng = np.maximum(hi_c - lo_c, 1e-30)
    amax = np.abs(y_ref).max(axis=1)

    if x64 is None:
        delta = np.zeros(T)
    else:
        delta = fp32_rotation_bound(x64, acc_eps) + amax * U32
    cond = delta / scale_ref  # the fp32 rotation bound in code units
    ill = cond > TIE_EPS
    well = ~ill
    if allow_ill is None:  # an 8-bit grid's codes are 17x finer: its long rows are not all well-conditioned
        allow_ill = n < ILL_MAX_N or bits > 4
    assert allow_ill or not ill.any(), (f"{int(ill.sum())} ill-conditioned tokens at n = {n}, "
                                        f"worst bound {float(cond.max()):.2e} code units")
    # well-conditioned tokens: the stated bar; ill-conditioned ones: widened by their bound
    srel_tol = np.where(ill, SCALE_REL + 2.0 * clip * delta / rng, SCALE_REL)
    w_code = np.where(ill, np.maximum(TIE_EPS, cond + (amax / scale_ref) * srel_tol * (1 + 1e-3)), TIE_EPS)
    w_zero = np.where(ill, np.maximum(TIE_EPS, clip * cond + (np.abs(lo_c) / scale_ref) * srel_tol * (1 + 1e-3)),
                      TIE_EPS)

    srel = np.abs(scale_gpu.astype(np.float64) - scale_ref) / np.abs(scale_ref)
    assert (srel <= srel_tol).all(), f"scale rel err {srel.max():.3e} > {srel_tol[np.argmax(srel - srel_tol)]:.3e}"

    zdiff = zero_gpu.astype(np.float64) - zero_ref
    zpre64 = zpre.astype(np.float64)
    zero_ok = (zdiff == 0) | ((np.abs(zdiff) == 1) & (np.abs(zero_gpu - zpre64) <= 0.5 + w_zero))
    zero_ok |= ill & (np.abs(zero_gpu - zpre64) <= 0.5 + w_zero)
    bad = ~zero_ok
    assert not bad.any(), (f"zero mismatch on tokens {np.flatnonzero(bad)[:8]}: "
                           f"{zero_gpu[bad][:4]} vs {zero_ref[bad][:4]}")
    shifted = np.flatnonzero(zdiff != 0)
    for t in shifted:  # the other side of a zero-point tie: redo the codes with the GPU's zero
        v = np.rint(y32[t] / scale_ref[t]) + zero_gpu[t]
        codes_ref[t] = np.clip(v, code_min, code_max).astype(np.int32)
        vpre[t] = y32[t] / scale_ref[t] + zero_gpu[t]

    diff = codes_gpu - codes_ref
    mism = diff != 0
    window = w_code[:, None]
    tie = _half_dist(vpre.astype(np.float64)) < window
    allowed_step = np.where(ill, 1 + np.floor(w_code), 1)[:, None]
    hard = mism & ~((np.abs(diff) <= allowed_step) & tie)
    wide = (ill & (w_code > 0.5))[:, None]  # rounding noise spans whole codes: decided by the dequantized value
    hard = hard & ~wide
    assert not hard.any(), (f"{int(hard.sum())} code mismatches away from ties, first at "
                            f"{np.argwhere(hard)[:4].tolist()}")
    n_well = int(mism[well].sum())
    allowed = math.ceil(TIE_FRAC * max(int(well.sum()), 1) * n)
    assert n_well <= allowed, f"{n_well} tie mismatches on well-conditioned tokens > {allowed}"
    if ill.any():
        deq = (codes_gpu.astype(np.float64) - zero_gpu[:, None]) * scale_gpu[:, None].astype(np.float64)
        lo_g = (code_min - zero_gpu.astype(np.float64)) * scale_gpu
        hi_g = (code_max - zero_gpu.astype(np.float64)) * scale_gpu
        yc = np.clip(y_ref, lo_g[:, None], hi_g[:, None])
        err = np.abs(deq - yc)[ill]
        lim = (scale_gpu[:, None] * 0.5 * (1 + 1e-5) + delta[:, None] + 1e-30)[ill]
        assert (err <= lim).all(), f"dequantized error {float((err - lim).max()):.3e} above half a step"
    return {"code_mismatches": int(mism.sum()), "mismatch_frac": float(mism.mean()) if mism.size else 0.0,
            "well_mismatches": n_well, "well_elements": int(well.sum()) * n,
            "zero_ties": int(shifted.size), "scale_rel_max": float(srel.max()) if srel.size else 0.0,
            "ill_conditioned_tokens": int(ill.sum())}


def record(name: str, stats: dict) -> None:
    """Append a test's parity statistics to $SIGNROT_PARITY_STATS (JSON lines), if set."""
    path = os.environ.get("SIGNROT_PARITY_STATS")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": name, **stats}) + "\n")
