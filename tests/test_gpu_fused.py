"""GPU tests of the fused tensor-core path (bf16 rows with n = 28 * {128, 256, 512, 1024} or
n = {4096, 8192, 16384, 32768}; the shortest, n = 3584 and 4096, share a 128-column MMA tile four
tokens to a tile): the outlier-channel entry points against the materialised sign vector, token
counts around the persistent grid, a general sign vector, and the device error word."""
import numpy as np
import pytest

from oracle import signrot_oracle as o
from rotation_activation_quantization_b200 import synthetic as syn

from parity import check_quant, check_rotation, oracle_sign, record

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

FUSED_N = [28 * 128, 28 * 256, 28 * 512, 28 * 1024, 4096, 8192, 16384, 32768]


@pytest.fixture(scope="module")
def sr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rotation_activation_quantization_b200 import signrot

    signrot.lib()
    signrot.device_error(clear=True)
    return signrot


def dev_bf16(x_np):
    return torch.from_numpy(np.ascontiguousarray(x_np).view(np.int16)).view(torch.bfloat16).cuda()


def i8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int8)).cuda()


SHORT_N = (28 * 128, 4096)  # four tokens per tile; a sign vector takes the exact generic kernel there


@pytest.mark.parametrize("n", FUSED_N)
def test_outlier_entry_equals_sign_vector_entry(sr, n):
    """Folding s into the rotation gives the same bits as applying the materialised s (on the
    short rows the two entries run different kernels: each is checked against the oracle)."""
    T = 37
    x, d, _ = syn.random_rows(n, T, "bf16", seed=n, outlier=1800.0)
    x_t, d_t = dev_bf16(x), i8(d)
    k, xk, _ = sr.calibrate(x_t)
    s_t = sr.build_sign(n, k, xk, d_t)
    q1, s1, z1 = sr.rotate_quant(x_t, d_t, s_t)
    q2, s2, z2 = sr.rotate_quant_outlier(x_t, d_t, k, xk)
    y1 = sr.rotate(x_t, d_t, s_t)
    y2 = sr.rotate_outlier(x_t, d_t, k, xk)
    if n not in SHORT_N:
        assert torch.equal(q1, q2) and torch.equal(s1, s2) and torch.equal(z1, z2)
        assert torch.equal(y1, y2)
    x64 = o.to_f64(x, "bf16")
    s_ref = oracle_sign(x64, d)
    assert (s_t.cpu().numpy() == s_ref).all()
    y_ref = o.rotate(x64, d, s_ref)
    st = check_rotation(y2.cpu().numpy(), y_ref)
    st.update(check_quant(q2.cpu().numpy(), s2.cpu().numpy(), z2.cpu().numpy(), y_ref, x64=x64))
    record(f"fused_outlier_{n}", st)
    if n in SHORT_N:
        check_rotation(y1.cpu().numpy(), y_ref)
        record(f"fused_vector_{n}", check_quant(q1.cpu().numpy(), s1.cpu().numpy(), z1.cpu().numpy(), y_ref, x64=x64))
    assert sr.device_error() == 0


@pytest.mark.parametrize("n,T", [(14336, 1), (14336, 2), (14336, 147), (14336, 148), (14336, 149), (14336, 297),
                                 (4096, 1), (4096, 3), (4096, 5), (4096, 591), (4096, 592), (4096, 593),
                                 (3584, 7), (3584, 1185)])
def test_token_counts_around_the_grid(sr, n, T):
    """Persistent grids of one CTA per SM (148): token counts around it, and for the shortest rows
    (four tokens per tile) counts that leave a partial last tile."""
    x, d, _ = syn.random_rows(n, T, "bf16", seed=T, outlier=1500.0)
    x_t, d_t = dev_bf16(x), i8(d)
    k, xk, _ = sr.calibrate(x_t)
    q, scale, zero = sr.rotate_quant_outlier(x_t, d_t, k, xk)
    torch.cuda.synchronize()
    rows = sorted({0, T // 2, T - 1, max(T - 2, 0)})
    s = oracle_sign(o.to_f64(x, "bf16"), d)
    x64 = o.to_f64(x[rows], "bf16")
    y_ref = o.rotate(x64, d, s)
    qn, sn, zn = q.cpu().numpy(), scale.cpu().numpy(), zero.cpu().numpy()
    record(f"fused_n{n}_T{T}", check_quant(qn[rows], sn[rows], zn[rows], y_ref, x64=x64))
    assert sr.device_error() == 0


@pytest.mark.parametrize("n", [28 * 128, 4096, 28 * 512, 28 * 1024, 16384])
def test_general_sign_vector_on_fused_path(sr, n):
    T = 9
    x, d, _ = syn.random_rows(n, T, "bf16", seed=3 * n, outlier=900.0)
    s = np.where(np.random.default_rng(n).random(n) < 0.5, -1, 1).astype(np.int8)
    x_t, d_t, s_t = dev_bf16(x), i8(d), i8(s)
    x64 = o.to_f64(x, "bf16")
    y_ref = o.rotate(x64, d, s)
    check_rotation(sr.rotate(x_t, d_t, s_t).cpu().numpy(), y_ref)
    q, scale, zero = sr.rotate_quant(x_t, d_t, s_t)
    check_quant(q.cpu().numpy(), scale.cpu().numpy(), zero.cpu().numpy(), y_ref, x64=x64)
    # and with no sign adjustment at all
    y_ref0 = o.rotate(x64, d)
    q, scale, zero = sr.rotate_quant(x_t, d_t, None)
    check_quant(q.cpu().numpy(), scale.cpu().numpy(), zero.cpu().numpy(), y_ref0, x64=x64)
    assert sr.device_error() == 0


def test_outlier_entry_with_zero_value_is_plain_rotation(sr):
    n, T = 14336, 4
    x, d, _ = syn.random_rows(n, T, "bf16", seed=5)
    x_t, d_t = dev_bf16(x), i8(d)
    k = torch.tensor([123], dtype=torch.int32, device="cuda")
    xk = torch.zeros(1, dtype=torch.float32, device="cuda")
    y = sr.rotate_outlier(x_t, d_t, k, xk)
    assert torch.equal(y, sr.rotate(x_t, d_t, None))


def test_out_of_range_channel_is_reported_not_read(sr):
    n, T = 14336, 3
    x, d, _ = syn.random_rows(n, T, "bf16", seed=6)
    x_t, d_t = dev_bf16(x), i8(d)
    k = torch.tensor([n + 5], dtype=torch.int32, device="cuda")
    xk = torch.ones(1, dtype=torch.float32, device="cuda")
    y = sr.rotate_outlier(x_t, d_t, k, xk)
    assert torch.equal(y, sr.rotate(x_t, d_t, None))
    assert sr.device_error(clear=True) == 2
    assert sr.device_error() == 0


@pytest.mark.parametrize("n,T,chunk", [(14336, 300, 64), (28672, 70, 16), (4096, 33, 8), (4096, 37, 6)])
def test_host_buffer_entry_matches_device_entry(sr, n, T, chunk):
    """Host rows -> chunked device workspace -> host codes equals the device-resident call."""
    x, d, _ = syn.random_rows(n, T, "bf16", seed=11 * T, outlier=1500.0)
    x_t, d_t = dev_bf16(x), i8(d)
    k, xk, _ = sr.calibrate(x_t)
    q, scale, zero = sr.rotate_quant_outlier(x_t, d_t, k, xk)
    xh = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).pin_memory()
    qh = torch.empty((T, n // 2), dtype=torch.uint8).pin_memory()
    sh = torch.empty(T, dtype=torch.float32).pin_memory()
    zh = torch.empty(T, dtype=torch.float32).pin_memory()
    ws = torch.empty(2 * (chunk * sr.host_bytes_per_token(n) + 64), dtype=torch.uint8, device="cuda")
    sr.rotate_quant_host(xh, d_t, qh, sh, zh, ws, k=k, xk=xk)
    torch.cuda.synchronize()
    assert torch.equal(qh, q.cpu()) and torch.equal(sh, scale.cpu()) and torch.equal(zh, zero.cpu())
    # a general sign vector through the same entry equals the device-resident vector call
    s_t = sr.build_sign(n, k, xk, d_t)
    qv, _, _ = sr.rotate_quant(x_t, d_t, s_t)
    sr.rotate_quant_host(xh, d_t, qh, sh, zh, ws, s=s_t)
    torch.cuda.synchronize()
    assert torch.equal(qh, qv.cpu())
    with pytest.raises(sr.SignRotError):
        sr.rotate_quant_host(xh, d_t, qh, sh, zh, ws[:16], k=k, xk=xk)
