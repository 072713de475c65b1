"""CPU oracle for SignRot's online down-projection activation path.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline leg may import this module. The product path (the CUDA library and its Python
binding) never calls it, and it shares no code, header, table or helper with that path.

What it computes, per token row x in R^n (the down-projection input of a LLaMA MLP):

    y = diag(s) . H . diag(D) . x / sqrt(n)          (float64, dense H, naive O(n^2))
    lo, hi = min y, max y;  scale = (hi - lo) / 15;  zero = rne(-lo / scale)
    q_j = clamp(rne(y_j / scale) + zero, 0, 15)      (packed two codes per byte)

Sources (page title, then the paragraph or table on it):

* "SignRot: LLM Quantization with Massive Outlier-Aware Sign-Adjusted Rotation" (arXiv
  2611.16502 abstract): randomized Hadamard transform applied online at the down-projection
  input by the fast Walsh-Hadamard transform; a sign adjustment vector that unifies the signs of
  the massive-outlier channel's Hadamard row, found in one calibration forward pass; asymmetric
  activation quantization whose zero-point absorbs the shift.
* "SignRot for 4-bit LLM quantization -- Sign-adjusted Hadamard rotation" (learnaivisually.com
  explainer):
    - "Picture the photographer": 16 levels spaced evenly from the smallest to the largest value
      of one token (so the range is the token's own [min, max], zero not forced in);
    - "The standard fix is rotation": Hadamard entries are +/-1/sqrt(n);
    - "Here is how it breaks": an outlier M gives every output a share +/-M/sqrt(n);
    - "SignRot asks one crowd to walk across the hall": the channel with the largest absolute
      calibration activation; each output j is multiplied by the sign of the outlier's entry,
      so the outlier adds the same +M/sqrt(n) everywhere; a diagonal sign matrix is its own
      inverse;
    - "The flip alone does nothing for a symmetric quantizer": asymmetric zero-point; the
      symmetric comparison grid;
    - "Worked example": steps are range/15 (asymmetric) and max|y|/7 (symmetric), no clipping.

Conventions the pages leave open, and the reading taken here:

* H = H_F kron H_M with n = F*M, F in {1, 28}, M = 2^m; channel j = a*M + b; H_M is Sylvester's
  (H_M[b, e] = (-1)^popcount(b & e)); H_28 is Paley's construction I over GF(27) =
  GF(3)[alpha]/(alpha^3 + 2 alpha + 1), field element index e = c0 + 3 c1 + 9 c2, Jacobsthal
  matrix Q[e, f] = chi(e - f), H_28 = I + [[0, 1^T], [-1, Q]] (index 0 is the point at
  infinity, index 1 + e the field element e). For the explainer's n = 11008 = 344 * 32 no page
  names the matrix; F = 344 is read as the same construction over GF(343) =
  GF(7)[alpha]/(alpha^3 + alpha + 1), element index e = c0 + 7 c1 + 49 c2.
* Column convention y = H x (y_j = sum_i H[j, i] x_i); D acts before H, s after it.
* s_j = +1 if H[j, k] * D_k * x_k >= 0 else -1, with x_k the signed calibration value of
  channel k at the first token attaining max_t |x_{t,k}|; k is the lowest channel index
  attaining the maximum.
* The quantizer takes its decisions (min, max, scale, zero, rounding of each code) in IEEE fp32,
  the precision of the GPU kernel: y is rounded once from float64 to fp32 first. Rounding is to
  nearest, ties to even. A row with hi == lo gets scale = 1 and zero = rne(-lo). A clip ratio c
  scales lo and hi (c = 1 is the only ratio the workloads use).
* Codes are unsigned 0..15; element 2i goes to the low nibble of byte i, 2i+1 to the high one.

Every function here is pinned by the CPU tests (tests/test_oracle_pins.py; the consumer side in
tests/test_oracle_consumer.py) against closed forms, invariants, brute force on tiny inputs, or
numbers printed on the pages.
"""
from __future__ import annotations

import math
from functools import lru_cache

import numpy as np

# ----------------------------------------------------------------------------------------------
# inputs: exact conversion of the stored activations to float64
# ----------------------------------------------------------------------------------------------


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly (bf16 is the top half of an fp32)."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


def to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return bf16_bits_to_f64(x)
    if dtype == "f32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    raise ValueError(dtype)


# ----------------------------------------------------------------------------------------------
# GF(p^3) arithmetic (p odd), elements as base-p digit vectors (c0, c1, c2) of c0 + c1 a + c2 a^2
# ----------------------------------------------------------------------------------------------


class GF3:
    """The field GF(p^3) built as GF(p)[a]/(a^3 + m2 a^2 + m1 a + m0) for an irreducible cubic."""

    def __init__(self, p: int, modulus: tuple[int, int, int]):
        self.p = p
        self.q = p ** 3
        self.m = tuple(int(c) % p for c in modulus)  # (m0, m1, m2)
        if any(self._poly_at(r) == 0 for r in range(p)):
            raise ValueError("modulus has a root in GF(p); not irreducible")

    def _poly_at(self, r: int) -> int:
        m0, m1, m2 = self.m
        return (r ** 3 + m2 * r * r + m1 * r + m0) % self.p

    def digits(self, e: int) -> list[int]:
        p = self.p
        return [e % p, (e // p) % p, (e // (p * p)) % p]

    def index(self, c) -> int:
        p = self.p
        return int(c[0] % p + p * (c[1] % p) + p * p * (c[2] % p))

    def sub(self, u: int, v: int) -> int:
        cu, cv = self.digits(u), self.digits(v)
        return self.index([cu[i] - cv[i] for i in range(3)])

    def mul(self, u: int, v: int) -> int:
        p = self.p
        cu, cv = self.digits(u), self.digits(v)
        prod = [0] * 5
        for i in range(3):
            for j in range(3):
                prod[i + j] += cu[i] * cv[j]
        # reduce from the top degree: a^d = a^(d-3) * a^3 and a^3 = -(m2 a^2 + m1 a + m0)
        for d in (4, 3):
            c = prod[d] % p
            prod[d] = 0
            for i, mi in enumerate(self.m):
                prod[d - 3 + i] -= c * mi
        return self.index(prod[:3])

    def nonzero_squares(self) -> set[int]:
        return {self.mul(y, y) for y in range(1, self.q)}

    def quadratic_character(self) -> np.ndarray:
        """chi(x) = 0 for x = 0, +1 for a nonzero square, -1 otherwise."""
        sq = self.nonzero_squares()
        return np.array([0] + [1 if e in sq else -1 for e in range(1, self.q)], dtype=np.int64)


GF27 = GF3(3, (1, 2, 0))  # a^3 + 2a + 1
GF343 = GF3(7, (1, 1, 0))  # a^3 + a + 1: H_344 for the n = 11008 example


def paley_skew_hadamard(field: GF3) -> np.ndarray:
    """Paley construction I for q = 3 (mod 4): an order q+1 skew Hadamard matrix, int8."""
    q = field.q
    if q % 4 != 3:
        raise ValueError("Paley construction I needs q = 3 (mod 4)")
    chi = field.quadratic_character()
    Q = np.empty((q, q), dtype=np.int64)
    for e in range(q):
        for f in range(q):
            Q[e, f] = chi[field.sub(e, f)]
    S = np.zeros((q + 1, q + 1), dtype=np.int64)
    S[0, 1:] = 1
    S[1:, 0] = -1
    S[1:, 1:] = Q
    return (np.eye(q + 1, dtype=np.int64) + S).astype(np.int8)


@lru_cache(maxsize=None)
def paley_h28() -> np.ndarray:
    h = paley_skew_hadamard(GF27)
    h.setflags(write=False)
    return h


@lru_cache(maxsize=None)
def paley_h344() -> np.ndarray:
    """Order-344 Paley matrix over GF(343) = GF(7)[a]/(a^3 + a + 1), same numbering and border as
    H_28: the explainer's n = 11008 (LLaMA2-7B intermediate size) token as 344 * 32."""
    h = paley_skew_hadamard(GF343)
    h.setflags(write=False)
    return h


_PALEY = {28: paley_h28, 344: paley_h344}


# ----------------------------------------------------------------------------------------------
# Hadamard matrices
# ----------------------------------------------------------------------------------------------


def sylvester(M: int) -> np.ndarray:
    """H_M[b, e] = (-1)^popcount(b & e), int8, M a power of two."""
    if M < 1 or M & (M - 1):
        raise ValueError("M must be a power of two")
    b = np.arange(M, dtype=np.int64)
    parity = np.zeros((M, M), dtype=np.int64)
    be = b[:, None] & b[None, :]
    while be.any():
        parity ^= be & 1
        be >>= 1
    return (1 - 2 * parity).astype(np.int8)


def factor_n(n: int) -> tuple[int, int]:
    """n = F * M with F in {1, 28} (344 for the oracle-only n = 11008 example) and M a power of
    two (M = 1 allowed for F > 1)."""
    for F in (1, 28, 344):
        if n % F == 0:
            M = n // F
            if M >= 1 and M & (M - 1) == 0 and (F > 1 or M >= 2):
                return F, M
    raise ValueError(f"unsupported n = {n}")


@lru_cache(maxsize=2)
def hadamard(n: int) -> np.ndarray:
    """Dense H_n = H_F kron H_M as int8 [n, n] (unnormalised, entries +/-1)."""
    F, M = factor_n(n)
    HM = sylvester(M)
    H = HM if F == 1 else np.kron(_PALEY[F](), HM).astype(np.int8)
    H.setflags(write=False)
    return H


# ----------------------------------------------------------------------------------------------
# the rotation, y = diag(s) H diag(D) x / sqrt(n)
# ----------------------------------------------------------------------------------------------


def rotate(x: np.ndarray, d: np.ndarray, s: np.ndarray | None = None) -> np.ndarray:
    """Float64 rotation of every row of x [T, n]: naive dense matrix-vector products.

    y_j = s_j * (sum_i H[j, i] * D_i * x_i) / sqrt(n). The products over the output index j are
    formed a block of rows of H at a time only to bound memory; each y_j is the plain sum.
    """
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    T, n = x.shape
    H = hadamard(n)
    xd = x * np.asarray(d, dtype=np.float64)[None, :]
    w = np.empty((T, n), dtype=np.float64)
    rows = max(1, (64 << 20) // (8 * n))
    for j0 in range(0, n, rows):
        j1 = min(n, j0 + rows)
        w[:, j0:j1] = xd @ H[j0:j1].astype(np.float64).T
    if s is not None:
        w *= np.asarray(s, dtype=np.float64)[None, :]
    return w / math.sqrt(n)


def rotate_fast(x: np.ndarray, d: np.ndarray, s: np.ndarray | None = None) -> np.ndarray:
    """The O(n log n) form: H_F across the stride-M axis, then an iterative FWHT over b.

    Not the authority (``rotate`` is); kept to cross-check the factorisation on small n.
    """
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    T, n = x.shape
    F, M = factor_n(n)
    z = (x * np.asarray(d, dtype=np.float64)[None, :]).reshape(T, F, M)
    if F > 1:
        z = np.einsum("ac,tcb->tab", _PALEY[F]().astype(np.float64), z)
    z = z.copy()
    h = 1
    while h < M:
        z = z.reshape(T, F, M // (2 * h), 2, h)
        u = z[:, :, :, 0, :].copy()
        v = z[:, :, :, 1, :].copy()
        z[:, :, :, 0, :] = u + v
        z[:, :, :, 1, :] = u - v
        h *= 2
    w = z.reshape(T, n)
    if s is not None:
        w = w * np.asarray(s, dtype=np.float64)[None, :]
    return w / math.sqrt(n)


# ----------------------------------------------------------------------------------------------
# calibration and the sign-adjustment vector
# ----------------------------------------------------------------------------------------------


def calibrate(x: np.ndarray) -> tuple[int, float]:
    """Outlier channel k (largest max_t |x_{t,i}|, lowest i on ties) and its signed value x_k
    at the first token attaining that maximum."""
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    A = np.abs(x).max(axis=0)
    k = int(np.flatnonzero(A == A.max())[0])
    t_star = int(np.flatnonzero(np.abs(x[:, k]) == A[k])[0])
    return k, float(x[t_star, k])


def build_sign(n: int, k: int, xk: float, d: np.ndarray) -> np.ndarray:
    """s_j = +1 if H[j, k] * D_k * x_k >= 0 else -1 (int8)."""
    col = hadamard(n)[:, k].astype(np.float64)
    v = col * float(d[k]) * float(xk)
    return np.where(v >= 0, 1, -1).astype(np.int8)


# ----------------------------------------------------------------------------------------------
# per-token quantizers (decisions in fp32)
# ----------------------------------------------------------------------------------------------


def quantize_asym(y: np.ndarray, bits: int = 4, clip: float = 1.0):
    """Asymmetric per-token quantizer. Returns (codes uint8 [T, n], scale f32 [T], zero f32 [T]).

    lo, hi = c*min y, c*max y; scale = (hi - lo) / (2^bits - 1); zero = rne(-lo / scale);
    code = clamp(rne(y / scale) + zero, 0, 2^bits - 1). All in fp32 after one rounding of y.
    """
    y32 = np.atleast_2d(np.asarray(y, dtype=np.float64)).astype(np.float32)
    qmax = np.float32(2 ** bits - 1)
    c = np.float32(clip)
    lo = y32.min(axis=1) * c
    hi = y32.max(axis=1) * c
    degenerate = hi == lo
    with np.errstate(divide="ignore", invalid="ignore"):
        scale = np.where(degenerate, np.float32(1.0), (hi - lo) / qmax).astype(np.float32)
        zero = np.rint(-lo / scale).astype(np.float32)
        v = np.rint(y32 / scale[:, None]) + zero[:, None]
    codes = np.clip(v, np.float32(0), qmax).astype(np.uint8)
    return codes, scale, zero


def asym_preround(y: np.ndarray, bits: int = 4, clip: float = 1.0) -> tuple[np.ndarray, np.ndarray]:
    """The values the two roundings of ``quantize_asym`` act on: (y/scale + zero, -lo/scale).

    Used by the parity tests to recognise rounding ties (a value within a hair of k + 1/2)."""
    y32 = np.atleast_2d(np.asarray(y, dtype=np.float64)).astype(np.float32)
    qmax = np.float32(2 ** bits - 1)
    c = np.float32(clip)
    lo = y32.min(axis=1) * c
    hi = y32.max(axis=1) * c
    with np.errstate(divide="ignore", invalid="ignore"):
        scale = np.where(hi == lo, np.float32(1.0), (hi - lo) / qmax).astype(np.float32)
        zpre = (-lo / scale).astype(np.float32)
        vpre = (y32 / scale[:, None]) + np.rint(zpre)[:, None]
    return vpre, zpre


def quantize_sym(y: np.ndarray, bits: int = 4):
    """Symmetric per-token comparison grid: levels -(2^(b-1)-1) .. +(2^(b-1)-1), step max|y|/L."""
    y32 = np.atleast_2d(np.asarray(y, dtype=np.float64)).astype(np.float32)
    L = np.float32(2 ** (bits - 1) - 1)
    amax = np.abs(y32).max(axis=1)
    scale = np.where(amax == 0, np.float32(1.0), amax / L).astype(np.float32)
    codes = np.clip(np.rint(y32 / scale[:, None]), -L, L).astype(np.int8)
    return codes, scale


def dequantize_asym(codes: np.ndarray, scale: np.ndarray, zero: np.ndarray) -> np.ndarray:
    return (codes.astype(np.float64) - zero.astype(np.float64)[:, None]) * scale.astype(np.float64)[:, None]


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """[T, n] codes 0..15 -> [T, n/2] bytes; element 2i low nibble, 2i+1 high nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], 2 * p.shape[1]), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def rotate_quant(x: np.ndarray, d: np.ndarray, s: np.ndarray | None, bits: int = 4, clip: float = 1.0):
    """The whole online path for rows x [T, n] (float64): (packed codes, scale, zero)."""
    codes, scale, zero = quantize_asym(rotate(x, d, s), bits=bits, clip=clip)
    return pack_nibbles(codes), scale, zero


# ----------------------------------------------------------------------------------------------
# consumer side: the down projection that reads the codes. Explainer, "SignRot asks one crowd to
# walk across the hall": the sign matrix is its own inverse and its flip is folded into the
# weights offline; "The flip alone does nothing for a symmetric quantizer": the zero-point's
# correction in the matrix multiply is the zero-point times a precomputed column sum of the
# weights. The weights' own quantizer (the pages use GPTQ) is out of scope; a per-output-channel
# symmetric round-to-nearest grid stands in for it.
# ----------------------------------------------------------------------------------------------


def fold_weights(w: np.ndarray, d: np.ndarray, s: np.ndarray | None = None) -> np.ndarray:
    """W' = W R^T for the down projection out = W x (w is [d_out, n]), R = diag(s) H diag(D) / sqrt(n).

    Then W' (R x) = W R^T R x = W x, R being orthogonal. Row o of W' is R applied to row o of W
    (W' = W R^T  <=>  W'^T = R W^T), so the fold is the activation rotation of W's rows.
    """
    return rotate(w, d, s)


def quantize_weights_sym(w: np.ndarray, bits: int = 4):
    """Per-output-channel symmetric grid for W' rows: (codes int8 [d_out, n], scale f32 [d_out])."""
    return quantize_sym(w, bits=bits)


def w4a4_matmul(codes: np.ndarray, scale: np.ndarray, zero: np.ndarray | None, wcodes: np.ndarray,
                wscale: np.ndarray) -> np.ndarray:
    """out[t, o] = scale_t * wscale_o * (sum_j codes[t, j] * wcodes[o, j] - zero_t * c_o),
    c_o = sum_j wcodes[o, j] (the precomputed column sum); zero = None for a symmetric grid.

    The integer sums are exact in float64 (|sum| < 2^53); the epilogue is float64.
    """
    q = np.atleast_2d(np.asarray(codes)).astype(np.float64)
    wq = np.atleast_2d(np.asarray(wcodes)).astype(np.float64)
    acc = q @ wq.T
    if zero is not None:
        c = wq.sum(axis=1)
        acc = acc - np.asarray(zero, dtype=np.float64)[:, None] * c[None, :]
    return acc * np.asarray(scale, dtype=np.float64)[:, None] * np.asarray(wscale, dtype=np.float64)[None, :]
