"""GPU tests of the quantizer variants: the asymmetric grid with 8 bits (codes 0..255, one per
byte) and the symmetric grid with 4 and 8 bits (codes -7..7 as two's-complement nibbles, -127..127
as int8; scale = max|y| / L, no zero-point), on the fused kernels (n = 28 * {256, 512, 1024},
16384), the generic kernel (the sign-vector entry at n = 1024 fp32 and 4096) and the short-row
kernels (the outlier entry there), against the float64 oracle. Where both entries run the same
kernel they must give the same bits."""
import numpy as np
import pytest

from oracle import signrot_oracle as o
from rotation_activation_quantization_b200 import synthetic as syn

from parity import check_quant, oracle_sign, record

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

SHAPES = [(1024, "f32"), (4096, "bf16"), (28 * 256, "bf16"), (28 * 512, "bf16"), (16384, "bf16"),
          (28 * 1024, "bf16")]
MODES = [(8, False), (4, True), (8, True)]


@pytest.fixture(scope="module")
def sr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rotation_activation_quantization_b200 import signrot

    signrot.lib()
    signrot.device_error(clear=True)
    return signrot


def to_dev(x_np, dtype):
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x_np).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x_np)).cuda()


def i8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int8)).cuda()


@pytest.mark.parametrize("n,dtype", SHAPES)
def test_quantizer_variants(sr, n, dtype):
    T = 24
    x, d, _ = syn.random_rows(n, T, dtype, seed=7 * n, outlier=1600.0)
    x_t, d_t = to_dev(x, dtype), i8(d)
    k, xk, _ = sr.calibrate(x_t)
    s_t = sr.build_sign(n, k, xk, d_t)
    x64 = o.to_f64(x, dtype)
    s_ref = oracle_sign(x64, d)
    assert (s_t.cpu().numpy() == s_ref).all()
    y_ref = o.rotate(x64, d, s_ref)
    # on the short rows (n = 3584, 4096 bf16; n = 512 .. 2048) the two entries run different
    # kernels: each is checked against the oracle
    same_kernel = not ((dtype == "bf16" and n in (3584, 4096)) or n in (512, 1024, 2048))
    for bits, sym in MODES:
        if sym:
            q1, sc1 = sr.rotate_quant_sym(x_t, d_t, s_t, bits=bits)
            q2, sc2 = sr.rotate_quant_sym_outlier(x_t, d_t, k, xk, bits=bits)
            z1 = z2 = None
            if same_kernel:
                assert torch.equal(q1, q2) and torch.equal(sc1, sc2)
        else:
            q1, sc1, z1 = sr.rotate_quant(x_t, d_t, s_t, bits=bits)
            q2, sc2, z2 = sr.rotate_quant_outlier(x_t, d_t, k, xk, bits=bits)
            if same_kernel:
                assert torch.equal(q1, q2) and torch.equal(sc1, sc2) and torch.equal(z1, z2)
        torch.cuda.synchronize()
        st = check_quant(q2.cpu().numpy(), sc2.cpu().numpy(), None if z2 is None else z2.cpu().numpy(), y_ref,
                         x64=x64, bits=bits, sym=sym)
        record(f"mode_{'sym' if sym else 'asym'}{bits}_{n}", st)
        if not same_kernel:
            check_quant(q1.cpu().numpy(), sc1.cpu().numpy(), None if z1 is None else z1.cpu().numpy(), y_ref,
                        x64=x64, bits=bits, sym=sym)
    assert sr.device_error() == 0


def test_symmetric_one_hot_row(sr):
    """A one-hot row M e_k with its own sign vector rotates to +M/sqrt(n) everywhere: every code is
    +L on the symmetric grid, and the scale is M/sqrt(n)/L."""
    n = 28 * 512
    x = np.zeros((1, n), dtype=np.float32)
    x[0, 4321] = 1200.0
    xb = syn.f32_to_bf16_bits(x)
    d = np.where(np.random.default_rng(1).random(n) < 0.5, -1, 1).astype(np.int8)
    x_t, d_t = to_dev(xb, "bf16"), i8(d)
    k, xk, _ = sr.calibrate(x_t)
    for bits in (4, 8):
        q, sc = sr.rotate_quant_sym_outlier(x_t, d_t, k, xk, bits=bits)
        torch.cuda.synchronize()
        from parity import decode_codes
        codes = decode_codes(q.cpu().numpy(), 1, n, bits, True)
        L = 2 ** (bits - 1) - 1
        assert (codes == L).all()
        _, scale_ref = o.quantize_sym(o.rotate(o.to_f64(xb, "bf16"), d, oracle_sign(o.to_f64(xb, "bf16"), d)), bits=bits)
        # the kernel folds 1/sqrt(n) in as an fp32 multiplier, so y (and max|y|) may differ from the
        # oracle's correctly rounded M/sqrt(n) by an ulp: the scale bar is 1e-5 relative
        assert abs(float(sc.item()) - float(scale_ref[0])) <= 1e-5 * float(scale_ref[0])
