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


def _outlier_rows(n=4096, T=64):
    from rotation_activation_quantization_b200 import synthetic as syn

    x, d, _ = syn.random_rows(n, T, "bf16", seed=17, outlier=1500.0)
    x64 = o.to_f64(x, "bf16")
    k, xk = o.calibrate(x64)
    y = o.rotate_fast(x64, d, o.build_sign(n, k, xk, d))
    return x64, y


def _flip_ties(codes, vpre, count):
    """Move `count` codes that sit at a rounding tie to the other neighbour of the tie."""
    c = codes.astype(np.int32).copy()
    frac = vpre - np.floor(vpre)
    ties = np.argwhere((np.abs(frac - 0.5) < 1e-3) & (c > 0) & (c < 15))
    assert len(ties) >= count
    for t, j in ties[:count]:
        fl = int(np.floor(vpre[t, j]))
        c[t, j] = fl + 1 if c[t, j] == fl else fl
    return c


def test_tie_cap_holds_on_rows_with_a_massive_outlier():
    """Rows whose rotation carries a massive outlier's shift are held to the 1e-4 tie cap, with the
    input rows given: a few tie flips pass, one more than the cap fails."""
    x64, y = _outlier_rows()
    codes, scale, zero = o.quantize_asym(y)
    vpre, _ = o.asym_preround(y)
    cap = int(np.ceil(1e-4 * y.size))
    ok = _flip_ties(codes, vpre, cap)
    st = check_quant(encode(ok, 4, False), scale, zero, y, x64=x64)
    assert st["ill_conditioned_tokens"] == 0 and st["well_mismatches"] == cap
    bad = _flip_ties(codes, vpre, cap + 1)
    with pytest.raises(AssertionError):
        check_quant(encode(bad, 4, False), scale, zero, y, x64=x64)


def test_scale_bar_is_not_widened_on_long_outlier_rows():
    x64, y = _outlier_rows()
    codes, scale, zero = o.quantize_asym(y)
    bad = scale.copy()
    bad[5] *= 1 + 3e-5
    with pytest.raises(AssertionError):
        check_quant(encode(codes, 4, False), bad, zero, y, x64=x64)


def test_an_extreme_one_ulp_off_fails_on_outlier_dominated_rows():
    """Rows like BASELINE config C1 (n = 1024 fp32, a massive outlier on every token): after the
    sign adjustment every output sits near |x_k| / sqrt(n) with a spread of about one, so
    |y| / scale is ~700. A grid built from a maximum one fp32 ulp above the true one passes the
    1e-5 scale bar, yet it moves every code by ~3e-3 of a step, and the checker rejects the codes.
    This is why the one-warp kernel for these rows sums in fp64."""
    rng = np.random.default_rng(11)
    n, T, k = 1024, 16, 300
    x = rng.normal(0.0, 0.3, size=(T, n)).astype(np.float32)
    x[:, k] = (np.where(rng.random(T) < 0.5, -1.0, 1.0) * rng.uniform(1000.0, 2000.0, size=T)).astype(np.float32)
    d = np.where(rng.random(n) < 0.5, -1, 1).astype(np.int8)
    x64 = x.astype(np.float64)
    kk, xk = o.calibrate(x64)
    y = o.rotate_fast(x64, d, o.build_sign(n, kk, xk, d))
    y32 = y.astype(np.float32)
    lo = y32.min(axis=1)
    hi = np.nextafter(y32.max(axis=1), np.float32(np.inf))
    scale = ((hi - lo) / np.float32(15)).astype(np.float32)
    zero = np.rint(-lo / scale).astype(np.float32)
    codes = np.clip(np.rint(y32 / scale[:, None]) + zero[:, None], 0, 15).astype(np.uint8)
    _, scale_ref, _ = o.quantize_asym(y)
    assert (np.abs(scale.astype(np.float64) / scale_ref - 1) <= 1e-5).all()
    assert float(np.median(np.abs(y32).max(axis=1) / scale_ref)) > 300
    with pytest.raises(AssertionError):
        check_quant(encode(codes, 4, False), scale, zero, y, x64=x64)
