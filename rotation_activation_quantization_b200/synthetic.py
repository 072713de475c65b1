"""Seeded synthetic activations shaped like a LLaMA down-projection input.

This module holds random draws and storage-format conversion only (draw in float64, round
to fp32, then to bf16 by round-to-nearest-even). None of the rotation, sign-adjustment or
quantization arithmetic lives here, so the CPU oracle and the CUDA path can both consume the
same bytes without sharing any of the method's code.

Value models (SignRot explainer, learnaivisually.com, "Here is how it breaks" and "SignRot asks
one crowd to walk across the hall": one massive-outlier channel that stays the same channel
across tokens, on top of ordinary channels):

  * ``gauss``   -- ordinary channels i.i.d. N(0, sigma^2)
  * ``laplace`` -- ordinary channels i.i.d. Laplace(0, sigma), plus ``secondaries`` distinct
    channels carrying +/-U[sec_lo, sec_hi] on every token

and in both a fixed, seed-chosen channel ``k0`` that carries +/-U[lo, hi] (sign drawn per
token) on a fraction ``outlier_frac`` of the tokens.

Every stream is seeded from ``[seed, stream, chunk]`` so a block of 256 tokens can be drawn on
its own: token t's values depend only on (workload, t // 256), never on how many tokens were
drawn before it.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np

CHUNK = 256  # tokens per independently seeded block

# seed streams
_S_CHANNELS, _S_D, _S_TOKENS, _S_CALIB = 0, 1, 2, 3


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    n: int
    T: int
    dtype: str  # "bf16" or "f32" (storage type of the activations)
    base: str  # "gauss" or "laplace"
    sigma: float
    outlier_lo: float
    outlier_hi: float
    outlier_frac: float
    secondaries: int = 0
    sec_lo: float = 0.0
    sec_hi: float = 0.0
    calib_T: int = 0  # 0: calibrate on the workload's own tokens
    seed: int = 0

    @property
    def in_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    def with_T(self, T: int) -> "Workload":
        return replace(self, T=int(T))


def _wl(index, **kw) -> Workload:
    return Workload(index=index, seed=1000 + index, **kw)


WORKLOADS = {
    1: _wl(1, name="n1024_T64_f32_gauss", n=1024, T=64, dtype="f32", base="gauss", sigma=0.3,
           outlier_lo=1000.0, outlier_hi=2000.0, outlier_frac=1.0, calib_T=0),
    2: _wl(2, name="n4096_T2048_bf16_gauss", n=4096, T=2048, dtype="bf16", base="gauss",
           sigma=0.3, outlier_lo=500.0, outlier_hi=2000.0, outlier_frac=0.9, calib_T=512),
    3: _wl(3, name="llama3_8b_down_proj_n14336_T8192_bf16", n=14336, T=8192, dtype="bf16",
           base="laplace", sigma=0.2, outlier_lo=800.0, outlier_hi=2000.0, outlier_frac=0.95,
           secondaries=8, sec_lo=20.0, sec_hi=60.0, calib_T=2048),
    4: _wl(4, name="llama3_70b_down_proj_n28672_T16384_bf16", n=28672, T=16384, dtype="bf16",
           base="laplace", sigma=0.2, outlier_lo=1000.0, outlier_hi=3000.0, outlier_frac=0.95,
           secondaries=8, sec_lo=20.0, sec_hi=60.0, calib_T=4096),
    5: _wl(5, name="llama3_8b_down_proj_n14336_sweep_bf16", n=14336, T=32768, dtype="bf16",
           base="laplace", sigma=0.2, outlier_lo=800.0, outlier_hi=2000.0, outlier_frac=0.95,
           secondaries=8, sec_lo=20.0, sec_hi=60.0, calib_T=128 * 2048),
    # LLaMA-2-7B's down projection (n = 11008 = 344 * 32, H_344 kron H_32): the explainer's token
    # of paragraph "Here is how it breaks" (outlier 1510) sits inside the outlier range
    6: _wl(6, name="llama2_7b_down_proj_n11008_T8192_bf16", n=11008, T=8192, dtype="bf16",
           base="laplace", sigma=0.2, outlier_lo=1000.0, outlier_hi=2000.0, outlier_frac=0.95,
           secondaries=8, sec_lo=20.0, sec_hi=60.0, calib_T=2048),
}

SWEEP_T = (1, 8, 64, 256, 1024, 4096, 32768)


def workload(index: int) -> Workload:
    return WORKLOADS[int(index)]


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(k) for k in key]))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest, ties to even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = ((u >> 16) & 1) + 0x7FFF
    return ((u + bias) >> 16).astype(np.uint16)


def channels(w: Workload) -> tuple[int, np.ndarray]:
    """(k0, secondary channel indices): distinct, seed-chosen."""
    perm = _rng(w.seed, _S_CHANNELS).permutation(w.n)
    return int(perm[0]), np.sort(perm[1:1 + w.secondaries]).astype(np.int64)


def draw_d(w: Workload) -> np.ndarray:
    """The random diagonal D as int8 +/-1 of length n."""
    u = _rng(w.seed, _S_D).random(w.n)
    return np.where(u < 0.5, -1, 1).astype(np.int8)


def _draw_block(w: Workload, stream: int, chunk: int, rows: int) -> np.ndarray:
    rng = _rng(w.seed, stream, chunk)
    if w.base == "gauss":
        v = rng.normal(0.0, w.sigma, size=(rows, w.n))
    elif w.base == "laplace":
        v = rng.laplace(0.0, w.sigma, size=(rows, w.n))
    else:
        raise ValueError(w.base)
    k0, sec = channels(w)
    present = rng.random(rows) < w.outlier_frac
    mag = rng.uniform(w.outlier_lo, w.outlier_hi, size=rows)
    sgn = np.where(rng.random(rows) < 0.5, -1.0, 1.0)
    v[present, k0] = (sgn * mag)[present]
    if w.secondaries:
        smag = rng.uniform(w.sec_lo, w.sec_hi, size=(rows, w.secondaries))
        ssgn = np.where(rng.random((rows, w.secondaries)) < 0.5, -1.0, 1.0)
        v[:, sec] = ssgn * smag
    return v


def _encode(w: Workload, v: np.ndarray) -> np.ndarray:
    a32 = v.astype(np.float32)
    return f32_to_bf16_bits(a32) if w.dtype == "bf16" else a32


def _draw(w: Workload, stream: int, t0: int, t1: int) -> np.ndarray:
    dt = np.uint16 if w.dtype == "bf16" else np.float32
    out = np.empty((max(t1 - t0, 0), w.n), dtype=dt)
    t = t0
    while t < t1:
        c = t // CHUNK
        blk = _encode(w, _draw_block(w, stream, c, CHUNK))
        lo = t - c * CHUNK
        hi = min(CHUNK, t1 - c * CHUNK)
        out[t - t0:t - t0 + (hi - lo)] = blk[lo:hi]
        t += hi - lo
    return out


def draw_tokens(w: Workload, t0: int = 0, t1: int | None = None) -> np.ndarray:
    """Activation rows [t0, t1): uint16 bf16 bit patterns, or float32, shape [t1-t0, n]."""
    return _draw(w, _S_TOKENS, t0, w.T if t1 is None else t1)


def draw_calibration(w: Workload, t0: int = 0, t1: int | None = None) -> np.ndarray:
    """Calibration rows; a workload with calib_T == 0 calibrates on its own tokens."""
    if w.calib_T == 0:
        return draw_tokens(w, t0, t1)
    return _draw(w, _S_CALIB, t0, w.calib_T if t1 is None else t1)


def calibration_size(w: Workload) -> int:
    return w.calib_T if w.calib_T else w.T


def random_rows(n: int, T: int, dtype: str = "bf16", seed: int = 0, outlier: float = 1500.0,
                k: int | None = None, sigma: float = 0.3, base: str = "laplace",
                outlier_sign: str = "random") -> tuple[np.ndarray, np.ndarray, int]:
    """Small seeded rows for parity sweeps: ordinary channels plus one massive-outlier channel.

    Returns (x encoded as bf16 bits or fp32, D as int8 +/-1, outlier channel k)."""
    rng = _rng(7919, seed, n, T)
    k = int(rng.integers(n)) if k is None else int(k)
    if base == "laplace":
        v = rng.laplace(0.0, sigma, size=(T, n))
    else:
        v = rng.normal(0.0, sigma, size=(T, n))
    if outlier:
        if outlier_sign == "random":
            sgn = np.where(rng.random(T) < 0.5, -1.0, 1.0)
        else:
            sgn = np.full(T, 1.0 if outlier_sign == "+" else -1.0)
        v[:, k] = sgn * rng.uniform(0.5 * outlier, outlier, size=T)
    d = np.where(rng.random(n) < 0.5, -1, 1).astype(np.int8)
    a32 = v.astype(np.float32)
    return (f32_to_bf16_bits(a32) if dtype == "bf16" else a32), d, k
