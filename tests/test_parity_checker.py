"""The GPU parity checker (tests/parity.py) on the CPU: the oracle's own codes in the library's
layout pass for every grid, and a code planted off a rounding tie, or a wrong scale, fails."""
import numpy as np
import pytest

from oracle import signrot_oracle as o

from parity import check_quant


def encode(codes: np.ndarray, bits: int, sym: bool) -> np.ndarray:
    c = np.asarray(codes, dtype=np.int32)
    if bits == 8:
        return c.astype(np.int8) if sym else c.astype(np.uint8)
    return o.pack_nibbles((c & 15).astype(np.uint8))


def rows(T=6, n=256, seed=3):
    rng = np.random.default_rng(seed)
    y = rng.laplace(0, 0.3, size=(T, n))
    y[:, 5] += 4.0
    return y


@pytest.mark.parametrize("bits,sym", [(4, False), (8, False), (4, True), (8, True)])
def test_oracle_codes_pass(bits, sym):
    y = rows()
    if sym:
        codes, scale = o.quantize_sym(y, bits=bits)
        zero = None
    else:
        codes, scale, zero = o.quantize_asym(y, bits=bits)
    st = check_quant(encode(codes, bits, sym), scale, zero, y, bits=bits, sym=sym)
    assert st["code_mismatches"] == 0


@pytest.mark.parametrize("bits,sym", [(4, False), (8, False), (4, True), (8, True)])
def test_planted_code_fails(bits, sym):
    y = rows()
    if sym:
        codes, scale = o.quantize_sym(y, bits=bits)
        zero = None
        vpre = y.astype(np.float32) / scale[:, None]
        lo_code = -(2 ** (bits - 1) - 1)
    else:
        codes, scale, zero = o.quantize_asym(y, bits=bits)
        vpre, _ = o.asym_preround(y, bits=bits)
        lo_code = 0
    codes = codes.astype(np.int32)
    far = np.abs(vpre - np.floor(vpre) - 0.5) > 0.1  # clearly not a tie
    far &= codes > lo_code
    t, j = np.argwhere(far)[0]
    codes[t, j] -= 1
    with pytest.raises(AssertionError):
        check_quant(encode(codes, bits, sym), scale, zero, y, bits=bits, sym=sym)


def test_wrong_symmetric_scale_fails():
    y = rows()
    codes, scale = o.quantize_sym(y, bits=4)
    bad = scale.copy()
    bad[2] *= 1.0001
    with pytest.raises(AssertionError):
        check_quant(encode(codes, 4, True), bad, None, y, bits=4, sym=True)
