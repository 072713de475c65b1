"""Pins for the oracle's consumer side (the down projection that reads the codes): the offline fold
of D, H and s into the weights, and the W4A4 product with the zero-point correction. Explainer,
"SignRot asks one crowd to walk across the hall" (a diagonal sign matrix is its own inverse; the
flip is folded into the weights offline) and "The flip alone does nothing for a symmetric
quantizer" (the zero-point's correction is the zero-point times a precomputed weight column sum).
None of these compares the oracle with itself: each checks an identity, a brute-force sum or a
closed-form bound."""
import itertools

import numpy as np
import pytest

from oracle import signrot_oracle as o
from rotation_activation_quantization_b200 import synthetic as syn


def _setup(n, T=12, d_out=40, seed=3, outlier=1500.0):
    x, d, _ = syn.random_rows(n, T, "f32", seed=seed, outlier=outlier, sigma=0.3)
    x64 = o.to_f64(x, "f32")
    w = np.random.default_rng(seed + 100).normal(0.0, 1.0 / np.sqrt(n), size=(d_out, n))
    k, xk = o.calibrate(x64)
    return x64, d, w, o.build_sign(n, k, xk, d)


@pytest.mark.parametrize("n", [8, 28, 112, 1024, 344 * 2])
def test_fold_keeps_the_product(n):
    """(W R^T)(R x) = W x: holds only if R is orthogonal and D, H, s sit where the fold puts them."""
    x64, d, w, s = _setup(n)
    for sv in (s, None):
        y = o.rotate(x64, d, sv)
        wf = o.fold_weights(w, d, sv)
        exact = x64 @ w.T
        assert np.allclose(y @ wf.T, exact, rtol=1e-11, atol=1e-11 * np.abs(exact).max())


def test_fold_of_the_flip_is_the_flip_itself():
    """diag(s) is its own inverse: folding s multiplies W' column j by s_j and nothing else."""
    n = 112
    x64, d, w, s = _setup(n)
    assert (o.fold_weights(w, d, s) == o.fold_weights(w, d, None) * s[None, :]).all()


def test_zero_point_correction_brute_force():
    """Integer product minus zero x column sum, against the dequantized product summed by hand."""
    rng = np.random.default_rng(11)
    T, n, d_out = 3, 8, 4
    codes = rng.integers(0, 16, size=(T, n))
    zero = rng.integers(0, 16, size=T).astype(np.float32)
    scale = rng.uniform(0.01, 0.5, size=T).astype(np.float32)
    wcodes = rng.integers(-7, 8, size=(d_out, n))
    wscale = rng.uniform(0.001, 0.05, size=d_out).astype(np.float32)
    got = o.w4a4_matmul(codes, scale, zero, wcodes, wscale)
    for t, oc in itertools.product(range(T), range(d_out)):
        ref = 0.0
        for j in range(n):
            ref += (float(scale[t]) * (int(codes[t, j]) - float(zero[t]))) * (float(wscale[oc]) * int(wcodes[oc, j]))
        assert got[t, oc] == pytest.approx(ref, rel=1e-13, abs=1e-15)
    # a symmetric grid has no correction
    sym = o.w4a4_matmul(codes - 8, scale, None, wcodes, wscale)
    assert np.allclose(sym, (codes - 8) @ wcodes.T * scale[:, None] * wscale[None, :], rtol=1e-14)


@pytest.mark.parametrize("n", [1024, 28 * 64])
def test_w4a4_error_within_the_rounding_bound(n):
    """|out - W x| <= (scale_t / 2) sum_j |w^_oj| + (wscale_o / 2) sum_j |y_j| (+ fp32 slack): each
    activation code is within half a step of y, each weight code within half a step of W'."""
    x64, d, w, s = _setup(n)
    y = o.rotate(x64, d, s)
    codes, scale, zero = o.quantize_asym(y)
    wq, ws = o.quantize_weights_sym(o.fold_weights(w, d, s))
    out = o.w4a4_matmul(codes, scale, zero, wq, ws)
    err = np.abs(out - x64 @ w.T)
    w_hat = wq.astype(np.float64) * ws.astype(np.float64)[:, None]
    bound = (0.5 * scale.astype(np.float64)[:, None] * np.abs(w_hat).sum(axis=1)[None, :]
             + 0.5 * ws.astype(np.float64)[None, :] * np.abs(y).sum(axis=1)[:, None])
    slack = 1e-5 * (np.abs(y).sum(axis=1)[:, None] * np.abs(w_hat).max())
    assert (err <= bound * (1 + 1e-6) + slack).all()
    # and the bound is not vacuous: the error uses a fair part of it
    assert (err / bound).mean() > 0.01


def test_symmetric_grid_gains_nothing_from_the_flip():
    """With a symmetric activation grid the flipped token quantizes to the flipped codes with the
    same scale, and the folded weights undo the flip: the outputs are identical."""
    n = 1024
    x64, d, w, s = _setup(n)
    outs = []
    for sv in (s, None):
        codes, scale = o.quantize_sym(o.rotate(x64, d, sv))
        wq, ws = o.quantize_weights_sym(o.fold_weights(w, d, sv))
        outs.append(o.w4a4_matmul(codes, scale, None, wq, ws))
    assert np.array_equal(outs[0], outs[1])


@pytest.mark.parametrize("n", [1024, 28 * 64, 4096])
def test_flip_with_zero_point_shrinks_the_product_error(n):
    """Asymmetric grid: with s the token's step shrinks, and so does the product's error once the
    weights' own rounding is small (8-bit weights here; with 4-bit round-to-nearest weights on these
    synthetic rows the weights' term, the same with and without s, dominates both)."""
    x64, d, w, s = _setup(n, T=16, d_out=64)
    exact = x64 @ w.T
    err = {}
    for label, sv in (("s", s), ("plain", None)):
        codes, scale, zero = o.quantize_asym(o.rotate(x64, d, sv))
        wq, ws = o.quantize_weights_sym(o.fold_weights(w, d, sv), bits=8)
        err[label] = np.abs(o.w4a4_matmul(codes, scale, zero, wq, ws) - exact).mean()
    assert err["plain"] > 2.0 * err["s"]
