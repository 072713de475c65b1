"""GPU parity: the CUDA path (through the C ABI) against the float64 CPU oracle on the same seeded
bytes. Tolerances live in tests/parity.py."""
import math

import numpy as np
import pytest

from oracle import signrot_oracle as o
from rotation_activation_quantization_b200 import synthetic as syn

from parity import check_quant, check_rotation, oracle_sign, record

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

POW2_N = [2 ** m for m in range(1, 16)]
P28_N = [28 * 2 ** m for m in range(0, 11)]


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
    return torch.from_numpy(np.ascontiguousarray(x_np, dtype=np.float32)).cuda()


def i8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int8)).cuda()


def gpu_sign(sr, x_t, d_t, n):
    k, xk, _ = sr.calibrate(x_t)
    s = sr.build_sign(n, k, xk, d_t)
    return s, int(k.item()), float(xk.item())


@pytest.mark.parametrize("n", POW2_N + P28_N)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_rotate_and_quant_sweep(sr, n, dtype):
    # enough elements that the 1e-4 tie allowance is several codes, not a fraction of one
    T = 9 if n >= 8192 else max(17, -(-30000 // n))
    x, d, _ = syn.random_rows(n, T, dtype, seed=1)
    x_t, d_t = dev(x, dtype), i8(d)
    s_t, k, xk = gpu_sign(sr, x_t, d_t, n)
    x64 = o.to_f64(x, dtype)
    k_ref, xk_ref = o.calibrate(x64)
    assert (k, xk) == (k_ref, xk_ref)
    s_ref = o.build_sign(n, k_ref, xk_ref, d)
    assert (s_t.cpu().numpy() == s_ref).all()
    y_ref = o.rotate(x64, d, s_ref)
    st = check_rotation(sr.rotate(x_t, d_t, s_t).cpu().numpy(), y_ref)
    q, scale, zero = sr.rotate_quant(x_t, d_t, s_t)
    st.update(check_quant(q.cpu().numpy(), scale.cpu().numpy(), zero.cpu().numpy(), y_ref, x64=x64))
    record(f"sweep_{dtype}_{n}", st)


@pytest.mark.parametrize("n", [2, 28, 56, 1024, 4096, 14336, 28672])
@pytest.mark.parametrize("T", [1, 5, 150])
def test_ragged_token_counts(sr, n, T):
    if n * T > 28672 * 20:
        T = 20
    x, d, _ = syn.random_rows(n, T, "bf16", seed=T)
    x_t, d_t = dev(x, "bf16"), i8(d)
    s_t, _, _ = gpu_sign(sr, x_t, d_t, n)
    x64 = o.to_f64(x, "bf16")
    s_ref = oracle_sign(x64, d)
    assert (s_t.cpu().numpy() == s_ref).all()
    y_ref = o.rotate(x64, d, s_ref)
    q, scale, zero = sr.rotate_quant(x_t, d_t, s_t)
    record(f"ragged_{n}_{T}", check_quant(q.cpu().numpy(), scale.cpu().numpy(), zero.cpu().numpy(), y_ref,
                                          x64=x64))


@pytest.mark.parametrize("n", [2, 28, 4096, 28 * 512, 28 * 1024])
@pytest.mark.parametrize("M", [1510.0, -1510.0])
def test_one_hot_collapses_bit_identically(sr, n, M):
    """M e_k calibrated on itself: all n fp32 outputs identical (= |M|/sqrt(n)); the row is
    constant, so the quantizer takes its hi == lo branch."""
    k = (3 * n) // 5
    x = np.zeros((1, n), dtype=np.float32)
    x[0, k] = M
    xb = syn.f32_to_bf16_bits(x)
    d = np.where(np.arange(n) % 3 == 0, -1, 1).astype(np.int8)
    x_t, d_t = dev(xb, "bf16"), i8(d)
    s_t, kk, xk = gpu_sign(sr, x_t, d_t, n)
    assert kk == k and xk == float(o.bf16_bits_to_f64(xb)[0, k])
    y = sr.rotate(x_t, d_t, s_t).cpu().numpy()[0]
    assert (y == y[0]).all()
    expect = abs(float(o.bf16_bits_to_f64(xb)[0, k])) / math.sqrt(n)
    assert abs(float(y[0]) - expect) <= 2 * np.spacing(np.float32(expect))
    q, scale, zero = sr.rotate_quant(x_t, d_t, s_t)
    assert float(scale.item()) == 1.0 and float(zero.item()) == float(np.rint(-np.float32(y[0])))
    assert (q.cpu().numpy() == 0).all()


@pytest.mark.parametrize("index", [1, 2, 3, 4])
def test_calibration_and_sign_exact(sr, index):
    w = syn.workload(index)
    xc = syn.draw_calibration(w)
    d = syn.draw_d(w)
    k, xk, _ = sr.calibrate(dev(xc, w.dtype))
    k_ref, xk_ref = o.calibrate(o.to_f64(xc, w.dtype))
    assert int(k.item()) == k_ref == syn.channels(w)[0]
    assert float(xk.item()) == xk_ref
    s = sr.build_sign(w.n, k, xk, i8(d)).cpu().numpy()
    assert (s == o.build_sign(w.n, k_ref, xk_ref, d)).all()


def test_calibration_chunked_with_cross_chunk_ties(sr):
    n, T = 4096, 600
    x, _, _ = syn.random_rows(n, T, "bf16", seed=9, outlier=0.0)
    x64 = o.to_f64(x, "bf16")
    # plant equal magnitudes in two chunks and two channels: lowest channel, first token win
    big = syn.f32_to_bf16_bits(np.array([[-1232.0, 1232.0]], dtype=np.float32))[0]  # exact in bf16
    x[450, 3000], x[100, 3000], x[120, 17] = big[1], big[0], big[1]
    x64 = o.to_f64(x, "bf16")
    ref = o.calibrate(x64)
    assert ref == (17, 1232.0)
    x_t = dev(x, "bf16")
    ws = torch.empty(n, dtype=torch.int64, device="cuda")
    for i, (t0, t1) in enumerate([(0, 64), (64, 64), (64, 300), (300, 600)]):
        k, xk, _ = sr.calibrate(x_t[t0:t1], ws=ws, accumulate=i > 0, t_offset=t0)
    assert (int(k.item()), float(xk.item())) == ref
    x[120, 17] = syn.f32_to_bf16_bits(np.array([1.0], dtype=np.float32))[0]
    ref2 = o.calibrate(o.to_f64(x, "bf16"))
    assert ref2 == (3000, -1232.0)
    x_t = dev(x, "bf16")
    for i, (t0, t1) in enumerate([(300, 600), (0, 300)]):  # later chunk first: t_offset decides
        k, xk, _ = sr.calibrate(x_t[t0:t1], ws=ws, accumulate=i > 0, t_offset=t0)
    assert (int(k.item()), float(xk.item())) == ref2


@pytest.mark.parametrize("index", [1, 2, 3, 4])
def test_workload_full_size(sr, index):
    """The workload's full token count through the same call the benchmark times; the oracle
    checks sampled tokens one by one, and every token is checked against the CUDA rotation by
    the quantizer's error bound."""
    w = syn.workload(index)
    x = syn.draw_tokens(w)
    d = syn.draw_d(w)
    x_t, d_t = dev(x, w.dtype), i8(d)
    k, xk, _ = sr.calibrate(dev(syn.draw_calibration(w), w.dtype))
    s_t = sr.build_sign(w.n, k, xk, d_t)
    q, scale, zero = sr.rotate_quant(x_t, d_t, s_t)
    torch.cuda.synchronize()
    rng = np.random.default_rng(index)
    if w.T <= 2048:
        sample = np.arange(w.T)
    else:
        sample = np.unique(np.concatenate([[0, 1, w.T - 1], rng.choice(w.T, 9, replace=False)]))
    s_ref = oracle_sign(o.to_f64(syn.draw_calibration(w), w.dtype), d)
    assert (s_t.cpu().numpy() == s_ref).all()
    y_ref = o.rotate(o.to_f64(x[sample], w.dtype), d, s_ref)
    qn, sn, zn = q.cpu().numpy(), scale.cpu().numpy(), zero.cpu().numpy()
    st = check_quant(qn[sample], sn[sample], zn[sample], y_ref)
    st.update(check_rotation(sr.rotate(x_t[sample.tolist()], d_t, s_t).cpu().numpy(), y_ref))
    record(f"workload_{index}", st)
    # every token: dequantized codes lie within half a step of the CUDA fp32 rotation
    y_all = sr.rotate(x_t, d_t, s_t)
    codes = torch.stack([q & 0xF, q >> 4], dim=-1).reshape(w.T, w.n).float()
    deq = (codes - zero[:, None]) * scale[:, None]
    err = (deq - y_all).abs().amax(dim=1)
    assert bool((err <= scale * 0.5 * (1 + 1e-4) + y_all.abs().amax(dim=1) * 1e-6).all())


@pytest.mark.parametrize("index", [1, 2, 3, 4])
def test_timed_call_full_size(sr, index):
    """The call the benchmark times -- the outlier-channel entry point, sign adjustment folded into
    the rotation -- on the workload's full token count, checked against the oracle on the first
    and the last token of every CTA of the persistent grid (one CTA per SM) plus a seeded sample.
    The reference takes k, x_k and s from the oracle's own calibration of the same batch."""
    w = syn.workload(index)
    x = syn.draw_tokens(w)
    d = syn.draw_d(w)
    xc = syn.draw_calibration(w)
    x_t, d_t = dev(x, w.dtype), i8(d)
    k, xk, _ = sr.calibrate(dev(xc, w.dtype))
    q, scale, zero = sr.rotate_quant_outlier(x_t, d_t, k, xk)
    torch.cuda.synchronize()
    assert sr.device_error() == 0
    k_ref, xk_ref = o.calibrate(o.to_f64(xc, w.dtype))
    assert (int(k.item()), float(xk.item())) == (k_ref, xk_ref)
    s_ref = o.build_sign(w.n, k_ref, xk_ref, d)
    # a CTA takes tiles of tok tokens (four for n = 4096's 32-column rows, else one)
    tok = 4 if w.n == 4096 else 1
    tiles = -(-w.T // tok)
    grid = min(tiles, torch.cuda.get_device_properties(0).multi_processor_count)
    first = np.arange(grid) * tok
    last = (np.arange(grid) + grid * ((tiles - 1 - np.arange(grid)) // grid)) * tok + tok - 1
    last = np.minimum(last, w.T - 1)
    extra = np.random.default_rng(100 + index).choice(w.T, 24, replace=False)
    sample = np.unique(np.concatenate([first, last, extra])) if w.T > 256 else np.arange(w.T)
    x64 = o.to_f64(x[sample], w.dtype)
    y_ref = o.rotate(x64, d, s_ref)
    st = check_quant(q.cpu().numpy()[sample], scale.cpu().numpy()[sample], zero.cpu().numpy()[sample], y_ref,
                     x64=x64)
    st["tokens_checked"] = int(sample.size)
    record(f"timed_call_{index}", st)


def test_edge_rows(sr):
    n = 28 * 64
    rows = np.zeros((6, n), dtype=np.float32)
    rows[1] = 3.0  # constant row before rotation
    rows[2] = np.random.default_rng(0).normal(0, 0.3, n)  # no outlier at all
    rows[3] = rows[2]
    rows[3, 5] = -2500.0  # negative outlier
    rows[4] = np.random.default_rng(1).uniform(-60000, 60000, n)  # large range
    rows[5, 7] = 1.0  # one tiny one-hot
    xb = syn.f32_to_bf16_bits(rows)
    d = np.where(np.random.default_rng(2).random(n) < 0.5, -1, 1).astype(np.int8)
    s = np.where(np.random.default_rng(3).random(n) < 0.5, -1, 1).astype(np.int8)
    x_t, d_t, s_t = dev(xb, "bf16"), i8(d), i8(s)
    x64 = o.to_f64(xb, "bf16")
    y_ref = o.rotate(x64, d, s)
    check_rotation(sr.rotate(x_t, d_t, s_t).cpu().numpy(), y_ref)
    q, scale, zero = sr.rotate_quant(x_t, d_t, s_t)
    check_quant(q.cpu().numpy(), scale.cpu().numpy(), zero.cpu().numpy(), y_ref, x64=x64)
    # s = NULL is the plain rotation
    y_ref0 = o.rotate(x64, d)
    check_rotation(sr.rotate(x_t, d_t, None).cpu().numpy(), y_ref0)
    q, scale, zero = sr.rotate_quant(x_t, d_t, None)
    check_quant(q.cpu().numpy(), scale.cpu().numpy(), zero.cpu().numpy(), y_ref0, x64=x64)


@pytest.mark.parametrize("clip", [1.0, 0.9])
def test_strided_misaligned_and_clip(sr, clip):
    n, T = 28 * 128, 9
    x, d, _ = syn.random_rows(n, T, "bf16", seed=4)
    big = np.zeros((T, n + 24), dtype=np.uint16)
    big[:, 3:3 + n] = x  # rows with ld = n + 24, starting one element off a 16 B boundary
    base = dev(big, "bf16")
    x_t = base[:, 3:3 + n]
    assert x_t.stride(0) == n + 24
    d_t = i8(d)
    s = np.where(np.random.default_rng(5).random(n) < 0.5, -1, 1).astype(np.int8)
    x64 = o.to_f64(x, "bf16")
    y_ref = o.rotate(x64, d, s)
    q, scale, zero = sr.rotate_quant(x_t, d_t, i8(s), clip=clip)
    check_quant(q.cpu().numpy(), scale.cpu().numpy(), zero.cpu().numpy(), y_ref, clip=clip, x64=x64)
    big2 = big.copy()
    big2[:, 8:8 + n] = x
    aligned = dev(big2, "bf16")[:, 8:8 + n]
    q2, scale2, zero2 = sr.rotate_quant(aligned, d_t, i8(s), clip=clip)
    check_quant(q2.cpu().numpy(), scale2.cpu().numpy(), zero2.cpu().numpy(), y_ref, clip=clip, x64=x64)


def test_zero_tokens_is_noop(sr):
    x = torch.empty((0, 1024), dtype=torch.bfloat16, device="cuda")
    d = torch.ones(1024, dtype=torch.int8, device="cuda")
    q, scale, zero = sr.rotate_quant(x, d)
    assert q.shape == (0, 512) and scale.shape == (0,)
    assert sr.rotate(x, d).shape == (0, 1024)
