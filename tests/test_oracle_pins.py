"""Pins for the CPU oracle: closed forms, invariants, brute force on tiny inputs, and the numbers
the SignRot explainer prints. None of these compares the oracle with itself."""
import json
import math
import os

import numpy as np
import pytest

from oracle import signrot_oracle as o
from rotation_activation_quantization_b200 import synthetic as syn

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "explainer_numbers.json")))

SMALL_N = [2, 4, 8, 16, 32, 64, 28, 56]


# ------------------------------------------------------------------------------------ GF(27)


def test_gf27_modulus_and_field_axioms():
    F = o.GF27
    a = 3  # the element alpha = (0, 1, 0)
    a3 = F.mul(F.mul(a, a), a)
    # alpha^3 + 2 alpha + 1 = 0  <=>  alpha^3 = alpha + 2
    assert F.digits(a3) == [2, 1, 0]
    one = 1
    for u in range(1, 27):
        assert sum(F.mul(u, v) == one for v in range(1, 27)) == 1  # a unique inverse
    # multiplication is commutative and distributes over subtraction
    rng = np.random.default_rng(0)
    for u, v, w in rng.integers(0, 27, size=(200, 3)):
        assert F.mul(u, v) == F.mul(v, u)
        assert F.mul(u, F.sub(v, w)) == F.sub(F.mul(u, v), F.mul(u, w))
    # the multiplicative group is cyclic of order 26
    orders = []
    for g in range(1, 27):
        x, k = g, 1
        while x != one:
            x, k = F.mul(x, g), k + 1
        orders.append(k)
    assert max(orders) == 26 and all(26 % k == 0 for k in orders)


def test_gf27_quadratic_character():
    chi = o.GF27.quadratic_character()
    assert (chi[1:] == 1).sum() == 13 and (chi[1:] == -1).sum() == 13 and chi[0] == 0
    minus_one = o.GF27.sub(0, 1)
    assert chi[minus_one] == -1  # q = 3 (mod 4): -1 is not a square, so Q is skew
    # chi is multiplicative
    for u in range(1, 27):
        for v in range(1, 27):
            assert chi[o.GF27.mul(u, v)] == chi[u] * chi[v]


# ---------------------------------------------------------------------------------- Hadamard


@pytest.mark.parametrize("order,build", [(28, o.paley_h28), (344, o.paley_h344)])
def test_paley_is_skew_hadamard(order, build):
    H = build().astype(np.int64)
    assert H.shape == (order, order)
    assert set(np.unique(H)) == {-1, 1}
    assert (H @ H.T == order * np.eye(order, dtype=np.int64)).all()
    assert (H + H.T == 2 * np.eye(order, dtype=np.int64)).all()


def test_paley_h28_convention_rows():
    """The fixed orientation: row 0 all +1, column 0 = (1, -1, ..., -1), unit diagonal."""
    H = o.paley_h28().astype(np.int64)
    assert (H[0] == 1).all()
    assert H[0, 0] == 1 and (H[1:, 0] == -1).all()
    assert (np.diag(H) == 1).all()


def _sylvester_by_doubling(M):
    H = np.array([[1]], dtype=np.int64)
    while H.shape[0] < M:
        H = np.block([[H, H], [H, -H]])
    return H


@pytest.mark.parametrize("M", [1, 2, 4, 8, 64, 512])
def test_sylvester_matches_doubling_definition(M):
    H = o.sylvester(M).astype(np.int64)
    assert (H == _sylvester_by_doubling(M)).all()
    assert (H == H.T).all()
    assert (H @ H == M * np.eye(M, dtype=np.int64)).all()


@pytest.mark.parametrize("n", [2, 64, 1024, 28, 56, 28 * 32, 28 * 64])
def test_kronecker_hadamard_orthogonal_and_blocks(n):
    H = o.hadamard(n).astype(np.int64)
    assert (H @ H.T == n * np.eye(n, dtype=np.int64)).all()
    F, M = o.factor_n(n)
    HM = _sylvester_by_doubling(M)
    HF = o.paley_h28().astype(np.int64) if F == 28 else np.ones((1, 1), dtype=np.int64)
    for a in range(F):
        for c in range(F):
            assert (H[a * M:(a + 1) * M, c * M:(c + 1) * M] == HF[a, c] * HM).all()


def test_factor_n_rejects_unsupported():
    for n in (3, 12, 14, 27, 29, 1000, 11008 * 3):
        with pytest.raises(ValueError):
            o.factor_n(n)
    assert o.factor_n(14336) == (28, 512)
    assert o.factor_n(28672) == (28, 1024)
    assert o.factor_n(4096) == (1, 4096)
    assert o.factor_n(28) == (28, 1)


# ---------------------------------------------------------------------------------- rotation


def _brute_rotate(x, d, s):
    """y_j = s_j * sum_i H[j,i] D_i x_i / sqrt(n), entries of H formed one by one."""
    n = x.shape[0]
    F, M = o.factor_n(n)
    H28 = o.paley_h28()
    y = []
    for j in range(n):
        a, b = divmod(j, M)
        acc = 0.0
        for i in range(n):
            c, e = divmod(i, M)
            hf = int(H28[a, c]) if F == 28 else 1
            h = hf * (-1) ** bin(b & e).count("1")
            acc += h * d[i] * x[i]
        y.append(s[j] * acc)
    return np.array(y) / math.sqrt(n)


@pytest.mark.parametrize("n", SMALL_N)
def test_rotate_brute_force_tiny(n):
    rng = np.random.default_rng(n)
    d = np.where(rng.random(n) < 0.5, -1, 1)
    s = np.where(rng.random(n) < 0.5, -1, 1)
    x = rng.normal(size=(3, n))
    y = o.rotate(x, d, s)
    for t in range(3):
        np.testing.assert_allclose(y[t], _brute_rotate(x[t], d, s), rtol=0, atol=1e-12)


@pytest.mark.parametrize("n", SMALL_N)
def test_fast_form_matches_dense_exactly(n):
    """All one-hot inputs and 100 integer rows: both forms must agree exactly in f64."""
    rng = np.random.default_rng(100 + n)
    d = np.where(rng.random(n) < 0.5, -1, 1)
    x = np.vstack([np.eye(n) * 3.0, rng.integers(-1000, 1000, size=(100, n)).astype(float)])
    a = o.rotate(x, d)
    b = o.rotate_fast(x, d)
    assert (a == b).all()  # both divide the same exact integer sums by the same sqrt(n)
    w = a * math.sqrt(n)
    assert np.abs(w - np.rint(w)).max() < 1e-9


@pytest.mark.parametrize("n", [64, 1024, 28 * 16, 28 * 64])
def test_rotation_preserves_norm(n):
    rng = np.random.default_rng(7 + n)
    d = np.where(rng.random(n) < 0.5, -1, 1)
    s = np.where(rng.random(n) < 0.5, -1, 1)
    x = rng.laplace(0, 0.2, size=(4, n))
    x[:, 3] = 1500.0
    y = o.rotate(x, d, s)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)


@pytest.mark.parametrize("n", [28, 56, 1024, 28 * 32, 4096, 14336])
@pytest.mark.parametrize("M", [1510.0, -1510.0])
def test_one_hot_collapses_to_plus_M_over_sqrt_n(n, M):
    """A one-hot M e_k, calibrated on itself: every sign-adjusted output is exactly |M|/sqrt(n)."""
    k = (n * 5) // 7
    rng = np.random.default_rng(n)
    d = np.where(rng.random(n) < 0.5, -1, 1).astype(np.int8)
    x = np.zeros((1, n))
    x[0, k] = M
    kk, xk = o.calibrate(x)
    assert (kk, xk) == (k, M)
    s = o.build_sign(n, kk, xk, d)
    y = o.rotate(x, d, s)[0]
    expect = abs(M) / math.sqrt(n)
    assert np.max(np.abs(y - expect)) <= 2 * np.spacing(expect)
    # without s the outputs split into two crowds at +/- |M|/sqrt(n)
    y0 = o.rotate(x, d)[0]
    assert np.allclose(np.abs(y0), expect, rtol=1e-15)
    assert (y0 > 0).any() and (y0 < 0).any()


def test_explainer_outlier_shift_n11008():
    """'Here is how it breaks': n = 11008, M = 1510 gives a shift of about 14.39 on every output
    (H_344 kron H_32, oracle-only), and with s every output sits at that one value."""
    g = GOLDEN["outlier_shift"]
    n, M = g["n"], float(g["M"])
    assert o.factor_n(n) == (344, 32)
    d = np.ones(n, dtype=np.int8)
    d[::3] = -1
    x = np.zeros((1, n))
    x[0, 4321] = M
    k, xk = o.calibrate(x)
    s = o.build_sign(n, k, xk, d)
    y = o.rotate(x, d, s)[0]
    assert np.allclose(y, y[0], rtol=1e-14)
    assert round(float(y[0]), g["shift_decimals"]) == g["shift"]
    y0 = o.rotate(x, d)[0]
    assert round(float(np.abs(y0).min()), 2) == g["shift"]
    assert (y0 < 0).sum() == n // 2


# --------------------------------------------------------------------- calibration and s


def test_calibrate_brute_force_with_ties():
    x = np.zeros((5, 6))
    x[1, 2] = -7.0
    x[3, 4] = 7.0  # ties channel 2 in |x|: the lower channel (2) wins
    x[4, 2] = 7.0  # ties within channel 2: the first token (t=1, value -7) supplies x_k
    x[0, 5] = 6.5
    assert o.calibrate(x) == (2, -7.0)
    x[2, 0] = -7.25
    assert o.calibrate(x) == (0, -7.25)


def test_calibrate_brute_force_random_tiny():
    rng = np.random.default_rng(3)
    for _ in range(50):
        x = rng.integers(-4, 5, size=(4, 5)).astype(float)
        best = None
        for i in range(5):
            for t in range(4):
                key = (abs(x[t, i]), -i, -t)
                if best is None or key > best[0]:
                    best = (key, i, x[t, i])
        assert o.calibrate(x) == (best[1], best[2])


@pytest.mark.parametrize("index", [1, 2, 3, 4, 6])
def test_calibration_finds_planted_channel(index):
    w = syn.workload(index)
    xc = o.to_f64(syn.draw_calibration(w, 0, min(256, syn.calibration_size(w))), w.dtype)
    k, xk = o.calibrate(xc)
    k0, _ = syn.channels(w)
    assert k == k0 and abs(xk) >= w.outlier_lo
    A = np.abs(xc).max(axis=0)
    assert np.sort(A)[-2] <= 100.0  # everything else is far below the massive outlier


@pytest.mark.parametrize("n", [8, 28, 56, 64])
def test_build_sign_brute_force(n):
    rng = np.random.default_rng(n)
    d = np.where(rng.random(n) < 0.5, -1, 1).astype(np.int8)
    for k in range(n):
        for xk in (3.0, -3.0, 0.0):
            s = o.build_sign(n, k, xk, d)
            e = np.zeros(n)
            e[k] = 1.0
            col = _brute_rotate(e, np.ones(n), np.ones(n)) * math.sqrt(n)  # column k of H
            expect = np.where(col * d[k] * xk >= 0, 1, -1)
            assert (s == expect).all()


# --------------------------------------------------------------------------------- quantizer


def _explainer_token(n=11008, seed=0):
    """A synthetic token whose sign-adjusted values span exactly [13.13, 15.63]."""
    g = GOLDEN["outlier_shift"]
    rng = np.random.default_rng(seed)
    y = rng.uniform(g["rotated_magnitude_lo"], g["rotated_magnitude_hi"], size=n)
    y[0], y[1] = g["rotated_magnitude_lo"], g["rotated_magnitude_hi"]
    return y


def test_worked_example_steps():
    """'Worked example': symmetric step 15.63/7 ~ 2.23, asymmetric without the flip 31.26/15 ~
    2.08, with flip + zero-point 2.50/15 ~ 0.167 (worst error ~ 0.083), about 13x finer."""
    g = GOLDEN["worked_example"]
    y = _explainer_token()
    rng = np.random.default_rng(1)
    y_split = y * np.where(rng.random(y.size) < 0.5, -1.0, 1.0)  # before s: two crowds
    y_split[0], y_split[1] = -15.63, 15.63

    codes, scale, zero = o.quantize_asym(y[None, :])
    assert round(float(scale[0]), 3) == g["asym_flip_step"]
    err = np.abs(o.dequantize_asym(codes, scale, zero)[0] - y.astype(np.float32))
    assert round(float(err.max()), 3) == g["asym_flip_worst_error"]

    _, scale_nf, _ = o.quantize_asym(y_split[None, :])
    assert round(float(scale_nf[0]), 2) == g["asym_noflip_step"]

    sc, ss = o.quantize_sym(y_split[None, :])
    assert round(float(ss[0]), 2) == g["sym_step"]
    assert round(float(ss[0]) / 2, 2) == g["sym_worst_error"]
    used = np.unique(sc[0])
    assert sorted(set(np.abs(used).tolist())) == [6, 7]
    level_values = sorted({round(float(abs(c) * ss[0]), 2) for c in used})
    assert level_values == g["sym_occupied_level_values"]
    assert g["sym_levels"] - len(used) == g["sym_empty_levels"]
    assert round(float(ss[0] / scale[0])) == g["step_ratio_approx"]


def test_symmetric_grid_ignores_the_flip():
    """'The flip alone does nothing for a symmetric quantizer': same scale with and without s."""
    n = 28 * 64
    rng = np.random.default_rng(5)
    d = np.where(rng.random(n) < 0.5, -1, 1).astype(np.int8)
    x = rng.laplace(0, 0.2, size=(6, n))
    x[:, 77] = rng.uniform(800, 2000, size=6)
    k, xk = o.calibrate(x)
    s = o.build_sign(n, k, xk, d)
    _, s1 = o.quantize_sym(o.rotate(x, d, s))
    _, s0 = o.quantize_sym(o.rotate(x, d))
    assert (s1 == s0).all()
    _, a1, _ = o.quantize_asym(o.rotate(x, d, s))
    _, a0, _ = o.quantize_asym(o.rotate(x, d))
    assert (a1 < a0 / 4).all()  # the asymmetric grid shrinks once the crowd is unimodal


def test_quantizer_invariants_random():
    rng = np.random.default_rng(11)
    y = rng.normal(3.0, 2.0, size=(200, 333))
    codes, scale, zero = o.quantize_asym(y)
    y32 = y.astype(np.float32)
    vpre, zpre = o.asym_preround(y)
    assert (codes <= 15).all()
    # codes are the clamped rounding of the pre-round values
    assert (np.clip(np.rint(vpre), 0, 15) == codes).all()
    assert (np.rint(zpre) == zero).all()
    # the min maps to 0 and the max to 15, away from rounding ties
    lo_i, hi_i = y32.argmin(axis=1), y32.argmax(axis=1)
    rows = np.arange(200)
    assert (codes[rows, lo_i] == 0).all()
    clean = np.abs(vpre[rows, hi_i] - np.floor(vpre[rows, hi_i]) - 0.5) > 1e-3
    assert (codes[rows, hi_i][clean] == 15).all()
    err = np.abs(o.dequantize_asym(codes, scale, zero) - y32)
    assert (err <= scale[:, None].astype(np.float64) * (0.5 + 1e-5)).all()
    np.testing.assert_allclose(scale, (y32.max(1) - y32.min(1)) / 15, rtol=1e-6)


def test_quantizer_ties_to_even_and_degenerate():
    codes, scale, zero = o.quantize_asym(np.array([[0.0, 1.5, 2.5, 3.5, 15.0]]))
    assert scale[0] == 1.0 and zero[0] == 0.0
    assert codes[0].tolist() == [0, 2, 2, 4, 15]
    codes, scale, zero = o.quantize_asym(np.full((1, 8), 62.5))
    assert scale[0] == 1.0 and zero[0] == -62.0 and (codes == 0).all()
    codes, scale, zero = o.quantize_asym(np.zeros((1, 8)))
    assert scale[0] == 1.0 and zero[0] == 0.0 and (codes == 0).all()


def test_clip_ratio_scales_range():
    y = np.array([[-2.0, 0.0, 1.0, 4.0]])
    _, scale, zero = o.quantize_asym(y, clip=0.5)
    assert scale[0] == np.float32(3.0 / 15) and zero[0] == np.rint(np.float32(1.0) / np.float32(0.2))


def test_pack_nibble_order():
    c = np.array([[1, 2, 15, 0, 7, 8]], dtype=np.uint8)
    p = o.pack_nibbles(c)
    assert p.tolist() == [[0x21, 0x0F, 0x87]]
    assert (o.unpack_nibbles(p) == c).all()


# ------------------------------------------------------ bimodal -> unimodal, split threshold


def _central_bins(y, bins=16):
    h, _ = np.histogram(y, bins=bins, range=(y.min(), y.max()))
    return h[bins // 4: 3 * bins // 4], h


@pytest.mark.parametrize("n", [1024, 28 * 64])
def test_bimodal_collapses_after_sign_adjustment(n):
    """'Here is how it breaks' / 'SignRot asks one crowd to walk across the hall': with a
    dominant outlier the rotated token has empty central bins; after s it is one crowd."""
    rng = np.random.default_rng(21)
    d = np.where(rng.random(n) < 0.5, -1, 1).astype(np.int8)
    k = 333
    x = rng.laplace(0, 0.05, size=(3, n))
    x[:, k] = [3000.0, 2500.0, 2800.0]
    kk, xk = o.calibrate(x)
    assert kk == k
    s = o.build_sign(n, kk, xk, d)
    col = o.hadamard(n)[:, k].astype(np.int64) * int(d[k])
    for t in range(3):
        y0 = o.rotate(x[t:t + 1], d)[0]
        central, h = _central_bins(y0)
        assert (central == 0).all()
        assert h[:4].sum() == (col < 0).sum() and h[-4:].sum() == (col > 0).sum()
        y1 = o.rotate(x[t:t + 1], d, s)[0]
        central, _ = _central_bins(y1)
        assert (central > 0).all()
        assert y1.min() > 0  # the whole crowd sits on the +M/sqrt(n) side


@pytest.mark.parametrize("ratio,bimodal", [(0.5, False), (4.0, True)])
def test_split_threshold_outlier_energy(ratio, bimodal):
    """The split appears once the outlier carries more energy than all other channels combined:
    the rotated row is ~ a 50/50 mixture of N(+/-M/sqrt(n), E_rest/n), bimodal iff M^2 > E_rest."""
    n = 16384
    rng = np.random.default_rng(31)
    d = np.where(rng.random(n) < 0.5, -1, 1).astype(np.int8)
    x = rng.normal(0, 1.0, size=(4, n))
    k = 1234
    x[:, k] = 0.0
    e_rest = (x ** 2).sum(axis=1)
    x[:, k] = np.sqrt(ratio * e_rest)
    y = o.rotate(x, d)
    sd = np.sqrt(e_rest / n)
    mu = x[:, k] / math.sqrt(n)
    z = (y / sd[:, None]).ravel()
    m = float(np.mean(mu / sd))
    centre = np.mean(np.abs(z) < 0.25)
    crowd = 0.5 * (np.mean(np.abs(z - m) < 0.25) + np.mean(np.abs(z + m) < 0.25))
    assert (centre < 0.8 * crowd) if bimodal else (centre > 1.05 * crowd)
