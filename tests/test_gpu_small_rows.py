"""GPU tests of the short-row kernel: n = 512, 1024, 2048 (F = 1), fp32 and bf16 rows, s in its
outlier form, one warp per token with fp64 butterflies and y rounded once to fp32 -- so that the
extremes, and with them the scale, are the oracle's even on rows whose every token carries a
massive outlier (BASELINE config C1: n = 1024, fp32, +/-U[1000, 2000]; there |y| / scale reaches
~700 and a scale one part in 2e5 off moves codes past the tie window). References: the float64
oracle, with k, x_k and s from its own calibration of the same rows."""
import numpy as np
import pytest

from oracle import signrot_oracle as o
from rotation_activation_quantization_b200 import synthetic as syn

from parity import check_quant, check_rotation, record

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

SMALL_N = (512, 1024, 2048)
F64_EPS = 2.0 ** -53  # the kernel's accumulation


@pytest.fixture(scope="module")
def sr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rotation_activation_quantization_b200 import signrot

    signrot.lib()
    signrot.device_error(clear=True)
    return signrot


def dev(x_np, dtype):
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x_np).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x_np, dtype=np.float32)).cuda()


def i8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int8)).cuda()


def reference(x, d, dtype):
    x64 = o.to_f64(x, dtype)
    k_ref, xk_ref = o.calibrate(x64)
    s_ref = o.build_sign(x.shape[1], k_ref, xk_ref, d)
    return x64, (k_ref, xk_ref), o.rotate(x64, d, s_ref)


@pytest.mark.parametrize("n", SMALL_N)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [1, 7, 64, 301])
def test_outlier_entry_against_oracle(sr, n, dtype, T):
    """Token counts below, at and above one CTA (four warps) and around the persistent grid."""
    x, d, _ = syn.random_rows(n, T, dtype, seed=n + T, outlier=2000.0, base="normal")
    x_t, d_t = dev(x, dtype), i8(d)
    k, xk, _ = sr.calibrate(x_t)
    x64, kref, y_ref = reference(x, d, dtype)
    assert (int(k.item()), float(xk.item())) == kref
    st = check_rotation(sr.rotate_outlier(x_t, d_t, k, xk).cpu().numpy(), y_ref)
    q, scale, zero = sr.rotate_quant_outlier(x_t, d_t, k, xk)
    torch.cuda.synchronize()
    st.update(check_quant(q.cpu().numpy(), scale.cpu().numpy(), zero.cpu().numpy(), y_ref, x64=x64, acc_eps=F64_EPS))
    record(f"small_{dtype}_{n}_T{T}", st)
    assert sr.device_error() == 0


@pytest.mark.parametrize("n,dtype", [(1024, "f32"), (512, "bf16"), (2048, "f32")])
def test_quantizer_variants(sr, n, dtype):
    """8-bit asymmetric and 4/8-bit symmetric grids on the same kernel. The grid's multiplier is
    the fp32 reciprocal of the scale, as on the fused kernels; on the 8-bit asymmetric grid
    (|y| / scale ~ 10^4 on these rows) its rounding, not the fp64 rotation, is the dominant error,
    so tokens are classed with the fp32 bound as in the fused kernels' quantizer tests."""
    T = 40
    x, d, _ = syn.random_rows(n, T, dtype, seed=3 * n, outlier=1800.0, base="normal")
    x_t, d_t = dev(x, dtype), i8(d)
    k, xk, _ = sr.calibrate(x_t)
    x64, _, y_ref = reference(x, d, dtype)
    for bits, sym in [(8, False), (4, True), (8, True)]:
        if sym:
            q, sc = sr.rotate_quant_sym_outlier(x_t, d_t, k, xk, bits=bits)
            z = None
        else:
            q, sc, z = sr.rotate_quant_outlier(x_t, d_t, k, xk, bits=bits)
        torch.cuda.synchronize()
        st = check_quant(q.cpu().numpy(), sc.cpu().numpy(), None if z is None else z.cpu().numpy(), y_ref,
                         x64=x64, bits=bits, sym=sym)
        record(f"small_mode_{'sym' if sym else 'asym'}{bits}_{n}", st)
    assert sr.device_error() == 0


@pytest.mark.parametrize("k", [0, 31, 32, 1023])
@pytest.mark.parametrize("sign", ["+", "-"])
def test_outlier_channel_positions(sr, k, sign):
    """The outlier at the first and last channel of a lane's run and of the row, either sign."""
    n, T = 1024, 48
    x, d, _ = syn.random_rows(n, T, "f32", seed=k + (7 if sign == "-" else 0), outlier=1500.0, k=k,
                              base="normal", outlier_sign=sign)
    x_t, d_t = dev(x, "f32"), i8(d)
    kk, xk, _ = sr.calibrate(x_t)
    assert int(kk.item()) == k
    x64, _, y_ref = reference(x, d, "f32")
    q, scale, zero = sr.rotate_quant_outlier(x_t, d_t, kk, xk)
    torch.cuda.synchronize()
    record(f"small_k{k}{sign}", check_quant(q.cpu().numpy(), scale.cpu().numpy(), zero.cpu().numpy(), y_ref,
                                            x64=x64, acc_eps=F64_EPS))


def test_inactive_plan_is_plain_rotation(sr):
    """x_k = 0 (all-zero calibration): no sign adjustment and nothing left out."""
    n, T = 1024, 12
    x, d, _ = syn.random_rows(n, T, "f32", seed=4, outlier=0.0, base="normal")
    x_t, d_t = dev(x, "f32"), i8(d)
    k = torch.tensor([77], dtype=torch.int32, device="cuda")
    xk = torch.zeros(1, dtype=torch.float32, device="cuda")
    y_ref = o.rotate(o.to_f64(x, "f32"), d)
    check_rotation(sr.rotate_outlier(x_t, d_t, k, xk).cpu().numpy(), y_ref)
    q, scale, zero = sr.rotate_quant_outlier(x_t, d_t, k, xk)
    torch.cuda.synchronize()
    check_quant(q.cpu().numpy(), scale.cpu().numpy(), zero.cpu().numpy(), y_ref, x64=o.to_f64(x, "f32"),
                acc_eps=F64_EPS)
    assert sr.device_error() == 0


def test_out_of_range_channel_is_reported(sr):
    n, T = 2048, 5
    x, d, _ = syn.random_rows(n, T, "bf16", seed=8, outlier=0.0)
    x_t, d_t = dev(x, "bf16"), i8(d)
    k = torch.tensor([n], dtype=torch.int32, device="cuda")
    xk = torch.ones(1, dtype=torch.float32, device="cuda")
    y_ref = o.rotate(o.to_f64(x, "bf16"), d)
    check_rotation(sr.rotate_outlier(x_t, d_t, k, xk).cpu().numpy(), y_ref)
    assert sr.device_error(clear=True) == 2
    assert sr.device_error() == 0


def test_strided_rows(sr):
    """Rows inside a wider buffer (ld = n + 64 elements): the row stride is honoured."""
    n, T, pad = 1024, 20, 64
    x, d, _ = syn.random_rows(n, T, "f32", seed=12, outlier=1700.0, base="normal")
    wide = np.zeros((T, n + pad), dtype=np.float32)
    wide[:, :n] = x
    xw = torch.from_numpy(wide).cuda()
    x_t = xw[:, :n]
    d_t = i8(d)
    k, xk, _ = sr.calibrate(dev(x, "f32"))
    x64, _, y_ref = reference(x, d, "f32")
    q, scale, zero = sr.rotate_quant_outlier(x_t, d_t, k, xk)
    torch.cuda.synchronize()
    check_quant(q.cpu().numpy(), scale.cpu().numpy(), zero.cpu().numpy(), y_ref, x64=x64, acc_eps=F64_EPS)
