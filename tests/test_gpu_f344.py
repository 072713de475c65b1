"""GPU tests of n = 344 * 2^m (H = H_344 kron H_M, Paley over GF(343)) against the float64 oracle.

n = 11008 = 344 * 32 is LLaMA-2-7B's MLP width, the token of the explainer's paragraph "Here is
how it breaks" (outlier M = 1510, shift M / sqrt(n) = 14.39). These shapes run on the generic
kernel; the tests cover calibration, the sign vector, the rotation, every quantizer grid, the
outlier-channel entry points (bit-identical to the materialised sign vector) and the host-buffer
entry point.

The generic kernel accumulates these rows in fp64 (a dense 344-term sum per output), so the parity
checker bounds their rounding with fp64's unit roundoff (F64_EPS) plus the final fp32 rounding.
"""
import math

import numpy as np
import pytest

from oracle import signrot_oracle as o
from rotation_activation_quantization_b200 import synthetic as syn

from parity import check_quant, check_rotation, oracle_sign, record

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
F64_EPS = 2.0 ** -53


@pytest.fixture(scope="module")
def sr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rotation_activation_quantization_b200 import signrot

    signrot.lib()
    return signrot


def dev(x_np, dtype):
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x_np).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x_np)).cuda()


def i8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int8)).cuda()


@pytest.mark.parametrize("n", [344, 688, 5504, 11008])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_f344_parity(sr, n, dtype):
    T = 13
    x, d, _ = syn.random_rows(n, T, dtype, seed=n + 3)
    x_t, d_t = dev(x, dtype), i8(d)
    k, xk, _ = sr.calibrate(x_t)
    s_t = sr.build_sign(n, k, xk, d_t)
    x64 = o.to_f64(x, dtype)
    k_ref, xk_ref = o.calibrate(x64)
    assert (int(k.item()), float(xk.item())) == (k_ref, xk_ref)
    s_ref = o.build_sign(n, k_ref, xk_ref, d)
    assert (s_t.cpu().numpy() == s_ref).all()
    y_ref = o.rotate(x64, d, s_ref)

    y = sr.rotate(x_t, d_t, s_t)
    assert torch.equal(y, sr.rotate_outlier(x_t, d_t, k, xk))
    st = check_rotation(y.cpu().numpy(), y_ref)
    st_plain = check_rotation(sr.rotate(x_t, d_t).cpu().numpy(), o.rotate(x64, d))

    q, scale, zero = sr.rotate_quant(x_t, d_t, s_t)
    q2, scale2, zero2 = sr.rotate_quant_outlier(x_t, d_t, k, xk)
    assert torch.equal(q, q2) and torch.equal(scale, scale2) and torch.equal(zero, zero2)
    st.update(check_quant(q.cpu().numpy(), scale.cpu().numpy(), zero.cpu().numpy(), y_ref, x64=x64,
                          acc_eps=F64_EPS))
    for bits, sym in [(8, False), (4, True), (8, True)]:
        if sym:
            qv, sv = sr.rotate_quant_sym_outlier(x_t, d_t, k, xk, bits=bits)
            zv = None
        else:
            qv, sv, zv = sr.rotate_quant_outlier(x_t, d_t, k, xk, bits=bits)
        torch.cuda.synchronize()
        check_quant(qv.cpu().numpy(), sv.cpu().numpy(), None if zv is None else zv.cpu().numpy(), y_ref,
                    x64=x64, bits=bits, sym=sym, acc_eps=F64_EPS)
    record(f"f344_{dtype}_{n}", {**st, "plain_rel_l2_max": st_plain["rel_l2_max"]})


def test_explainer_llama2_token(sr):
    """The explainer's n = 11008 token with a lone outlier M = 1510: without the sign vector every
    output is +-M/sqrt(n) = +-14.39, half of each sign (the outlier's column of H_344 kron H_32 is
    balanced when its Sylvester index is nonzero); with it every output is +14.39."""
    n, M, k = 11008, 1510.0, 6 * 32 + 5
    x = np.zeros((1, n), dtype=np.float32)  # fp32 rows: 1510 is not a bf16 value (step 8 there)
    x[0, k] = M
    d = np.ones(n, dtype=np.int8)
    x_t, d_t = dev(x, "f32"), i8(d)
    shift = M / math.sqrt(n)
    assert round(shift, 2) == 14.39
    y0 = sr.rotate(x_t, d_t).cpu().numpy()[0].astype(np.float64)
    assert np.allclose(np.abs(y0), shift, rtol=2e-7, atol=0)
    assert (y0 > 0).sum() == n // 2
    kk, xk, _ = sr.calibrate(x_t)
    assert int(kk.item()) == k and float(xk.item()) == M
    y1 = sr.rotate_outlier(x_t, d_t, kk, xk).cpu().numpy()[0]
    assert (y1 == y1[0]).all() and abs(float(y1[0]) - shift) <= 2 * np.spacing(np.float32(shift))


def test_f344_ragged_and_host_buffers(sr):
    n = 11008
    for T in (1, 2, 37):
        x, d, _ = syn.random_rows(n, T, "bf16", seed=T)
        x_t, d_t = dev(x, "bf16"), i8(d)
        k, xk, _ = sr.calibrate(x_t)
        s_t = sr.build_sign(n, k, xk, d_t)
        x64 = o.to_f64(x, "bf16")
        s_ref = oracle_sign(x64, d)
        assert (s_t.cpu().numpy() == s_ref).all()
        y_ref = o.rotate(x64, d, s_ref)
        q, scale, zero = sr.rotate_quant(x_t, d_t, s_t)
        torch.cuda.synchronize()
        check_quant(q.cpu().numpy(), scale.cpu().numpy(), zero.cpu().numpy(), y_ref, x64=x64, acc_eps=F64_EPS)
        xh = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).pin_memory()
        qh = torch.empty((T, n // 2), dtype=torch.uint8).pin_memory()
        sh = torch.empty(T, dtype=torch.float32).pin_memory()
        zh = torch.empty(T, dtype=torch.float32).pin_memory()
        ws = torch.empty(2 * (8 * sr.host_bytes_per_token(n) + 64), dtype=torch.uint8, device="cuda")
        sr.rotate_quant_host(xh, d_t, qh, sh, zh, ws, k=k, xk=xk)
        torch.cuda.synchronize()
        assert torch.equal(qh, q.cpu()) and torch.equal(sh, scale.cpu()) and torch.equal(zh, zero.cpu())
