"""GPU tests of the W4A4 down projection (the consumer of the packed codes) against the oracle's
w4a4_matmul, on the same seeded codes and scales.

Explainer, "SignRot asks one crowd to walk across the hall" (the flip folded into the weights
offline) and "The flip alone does nothing for a symmetric quantizer" (the zero-point's correction
is the zero-point times a precomputed column sum of the weights). The integer sums are exact on
both sides; the CUDA epilogue rounds the bracket (sum - zero * colsum) once to fp32 and multiplies
by the two scales, so each output may differ from the float64 oracle by at most three fp32
roundings: |gpu - ref| <= 4 * 2^-24 * |ref|. A wrong integer anywhere moves an output by at least
scale * wscale, far outside that bound.
"""
import numpy as np
import pytest

from oracle import signrot_oracle as o

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

REL = 4 * 2.0 ** -24


@pytest.fixture(scope="module")
def sr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rotation_activation_quantization_b200 import signrot

    signrot.lib()
    signrot.device_error(clear=True)
    return signrot


def pack_signed(codes: np.ndarray) -> np.ndarray:
    """Signed 4-bit codes [R, K] -> two's complement nibbles, element 2i low (the sym4 layout)."""
    c = (np.asarray(codes, dtype=np.int64) & 15).astype(np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def draw(T, K, N, seed, sym=False):
    rng = np.random.default_rng(seed)
    if sym:
        codes = rng.integers(-7, 8, size=(T, K), dtype=np.int8)
        packed = pack_signed(codes)
        zero = None
    else:
        codes = rng.integers(0, 16, size=(T, K), dtype=np.int8)
        packed = o.pack_nibbles(codes.astype(np.uint8))
        zero = rng.integers(-120, 40, size=T).astype(np.float32)
    scale = rng.uniform(0.01, 0.5, size=T).astype(np.float32)
    wcodes = rng.integers(-8, 8, size=(N, K), dtype=np.int8)
    wscale = rng.uniform(1e-3, 2e-2, size=N).astype(np.float32)
    return codes, packed, scale, zero, wcodes, wscale


def cuda(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t if dtype is None else t.to(dtype)).cuda()


def run(sr, packed, scale, zero, wcodes, wscale, K):
    wq8, colsum = sr.w4a4_prepare_weights(cuda(pack_signed(wcodes)), K)
    torch.cuda.synchronize()
    assert (wq8.cpu().numpy() == wcodes).all()
    assert (colsum.cpu().numpy() == wcodes.astype(np.int64).sum(axis=1)).all()
    out = sr.w4a4_matmul(cuda(packed), cuda(scale), None if zero is None else cuda(zero), wq8, cuda(wscale), colsum)
    torch.cuda.synchronize()
    assert sr.device_error() == 0
    return out.cpu().numpy().astype(np.float64)


def check(out, ref):
    err = np.abs(out - ref)
    lim = REL * np.abs(ref) + 1e-30
    assert (err <= lim).all(), f"max excess {float((err - lim).max()):.3e} at {np.unravel_index(np.argmax(err - lim), err.shape)}"
    return float((err / np.maximum(np.abs(ref), 1e-30)).max())


@pytest.mark.parametrize("T,K,N", [(300, 1024, 608), (128, 128, 256), (1, 256, 16), (257, 14336, 512)])
@pytest.mark.parametrize("sym", [False, True])
def test_matches_oracle(sr, T, K, N, sym):
    """Ragged token and output tiles (300 = 2 x 128 + 44 tokens, 608 = 2 x 256 + 96 outputs), one
    full tile, a single token, and the LLaMA-3-8B down projection's K = 14336."""
    codes, packed, scale, zero, wcodes, wscale = draw(T, K, N, seed=T * 7 + K + N + int(sym), sym=sym)
    out = run(sr, packed, scale, zero, wcodes, wscale, K)
    ref = o.w4a4_matmul(codes, scale, zero, wcodes, wscale)
    check(out, ref)


def test_full_size_sampled_rows(sr):
    """LLaMA-3-8B's down projection at the benchmark's token count (T = 8192, K = 14336, N = 4096),
    checked against the oracle on the first and last row of every 128-token tile."""
    T, K, N = 8192, 14336, 4096
    codes, packed, scale, zero, wcodes, wscale = draw(T, K, N, seed=99)
    out = run(sr, packed, scale, zero, wcodes, wscale, K)
    rows = np.unique(np.concatenate([np.arange(0, T, 128), np.arange(127, T, 128)]))
    ref = o.w4a4_matmul(codes[rows], scale[rows], zero[rows], wcodes, wscale)
    check(out[rows], ref)


def test_consumer_of_the_fused_quantizer(sr):
    """End to end through the library: the folded weights W' = rows of W rotated with the same D
    and outlier sign and quantized per row on the symmetric 4-bit grid by the fused kernel,
    prepared, and multiplied with the fused kernel's packed activation codes. Against the oracle
    doing the same from the same seeded x and W (its own calibration, rotation, both grids, fold
    and product): equal up to codes that sit at rounding ties (relative L2 <= 1e-4). Against the
    exact product W x: within the two 4-bit grids' error."""
    from rotation_activation_quantization_b200 import synthetic as syn

    n, T, N = 14336, 64, 256
    x, d, _ = syn.random_rows(n, T, "bf16", seed=5, outlier=1500.0)
    rng = np.random.default_rng(6)
    wb = syn.f32_to_bf16_bits(rng.normal(0, 0.02, size=(N, n)).astype(np.float32))
    x_t = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    w_t = torch.from_numpy(wb.view(np.int16)).view(torch.bfloat16).cuda()
    d_t = cuda(d)
    k, xk, _ = sr.calibrate(x_t)
    q, scale, zero = sr.rotate_quant_outlier(x_t, d_t, k, xk)
    wq4, wscale = sr.rotate_quant_sym_outlier(w_t, d_t, k, xk, bits=4)
    wq8, colsum = sr.w4a4_prepare_weights(wq4, n)
    out = sr.w4a4_matmul(q, scale, zero, wq8, wscale, colsum)
    torch.cuda.synchronize()
    out = out.cpu().numpy().astype(np.float64)

    x64, w64 = o.to_f64(x, "bf16"), o.to_f64(wb, "bf16")
    k_ref, xk_ref = o.calibrate(x64)
    s_ref = o.build_sign(n, k_ref, xk_ref, d)
    codes, sc, z = o.quantize_asym(o.rotate(x64, d, s_ref))
    wcodes, wsc = o.quantize_weights_sym(o.fold_weights(w64, d, s_ref), bits=4)
    ref = o.w4a4_matmul(codes, sc, z, wcodes, wsc)
    rel_ref = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert rel_ref <= 1e-4, rel_ref
    # the product approximates W x: W' R x = W R^T R x = W x up to the two grids' rounding
    exact = x64 @ w64.T
    rel = np.linalg.norm(out - exact) / np.linalg.norm(exact)
    assert rel < 0.5, rel  # 4-bit weights dominate; a wrong fold would leave no correlation (rel ~ 1.4)
