"""GPU tests of signrot_calibrate's token rules against the oracle: the largest |x| wins, the
lowest channel on equal magnitudes, and the FIRST token attaining it gives x_k its sign. Cases
put the tied tokens inside one of the kernel's token blocks and in different blocks, at a token
count large enough for blocks of hundreds of tokens, and take both fold kernels (16-byte aligned
bf16 rows with n % 8 == 0, and the element-wise kernel for other rows)."""
import numpy as np
import pytest

from oracle import signrot_oracle as o
from rotation_activation_quantization_b200 import synthetic as syn

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rotation_activation_quantization_b200 import signrot

    signrot.lib()
    return signrot


def bf16(vals):
    return syn.f32_to_bf16_bits(np.asarray(vals, dtype=np.float32))


def dev(x_np):
    return torch.from_numpy(np.ascontiguousarray(x_np).view(np.int16)).view(torch.bfloat16).cuda()


def run(sr, x_t):
    k, xk, _ = sr.calibrate(x_t)
    torch.cuda.synchronize()
    return int(k.item()), float(xk.item())


@pytest.mark.parametrize("T,hits", [
    (600, [(5, -1232.0), (7, 1232.0)]),                      # same block: first token (negative) wins
    (600, [(7, 1232.0), (5, -1232.0), (590, -1232.0)]),      # order of planting is irrelevant
    (40000, [(15001, 1232.0), (15003, -1232.0)]),            # same (long) block
    (40000, [(39999, -1232.0), (3, 1232.0), (20000, -1232.0)]),  # different blocks
])
def test_first_token_and_sign_rule(sr, T, hits):
    n = 1024
    x, _, _ = syn.random_rows(n, T, "bf16", seed=T + len(hits), outlier=0.0)
    for t, v in hits:
        x[t, 700] = bf16([v])[0]
    x[T // 2, 900] = bf16([1232.0])[0]  # same magnitude in a higher channel: loses
    ref = o.calibrate(o.to_f64(x, "bf16"))
    t_first = min(t for t, _ in hits)
    assert ref == (700, dict(hits)[t_first])
    assert run(sr, dev(x)) == ref


def test_both_fold_kernels_agree_with_oracle(sr):
    n, T = 4096, 333
    x, _, k0 = syn.random_rows(n, T, "bf16", seed=5, outlier=1500.0)
    x_t = dev(x)
    ref = o.calibrate(o.to_f64(x, "bf16"))
    assert ref[0] == k0
    assert run(sr, x_t) == ref  # 16-byte aligned rows, n % 8 == 0: the vector kernel
    # rows starting 2 bytes past a 16-byte boundary (ld = 4096, n = 1024): the element-wise kernel
    assert run(sr, x_t[:, 1:1025]) == o.calibrate(o.to_f64(x[:, 1:1025], "bf16"))
    # n = 28 (n % 8 != 0): the element-wise kernel
    x28 = np.ascontiguousarray(x[:, :28])
    assert run(sr, dev(x28)) == o.calibrate(o.to_f64(x28, "bf16"))


def test_all_zero_rows(sr):
    x = np.zeros((300, 2048), dtype=np.uint16)
    assert run(sr, dev(x)) == (0, 0.0)


@pytest.mark.parametrize("index", [2, 3])
def test_sharded_calibration_keys_and_merge(sr, index):
    """Two shards of one calibration set folded separately (as two ranks would): each workspace
    holds exactly the keys the header defines (restated in tests/calib_keys.py), their elementwise
    maximum -- what the all-reduce(MAX) of calibrate_sharded computes -- gives the whole set's
    (k, x_k) through the argmax-only call, and calibrate_sharded without a process group equals
    calibrate."""
    from calib_keys import decode, fold_keys

    w = syn.workload(index)
    xc = syn.draw_calibration(w)
    Tc = xc.shape[0]
    half = Tc // 2 + 3  # an uneven split
    x_t = dev(xc)  # both workloads store bf16 rows
    x64 = o.to_f64(xc, w.dtype)
    ws_a = torch.empty(w.n, dtype=torch.int64, device="cuda")
    ws_b = torch.empty(w.n, dtype=torch.int64, device="cuda")
    sr.calibrate(x_t[:half], ws=ws_a, t_offset=0)
    sr.calibrate(x_t[half:], ws=ws_b, t_offset=half)
    torch.cuda.synchronize()
    keys_a = fold_keys(x64[:half], t_offset=0)
    keys_b = fold_keys(x64[half:], t_offset=half)
    assert (ws_a.cpu().numpy().astype(np.uint64) == keys_a).all()
    assert (ws_b.cpu().numpy().astype(np.uint64) == keys_b).all()
    merged = torch.maximum(ws_a, ws_b)
    k, xk = sr.calibrate_finish(merged)
    ref = o.calibrate(x64)
    assert (int(k.item()), float(xk.item())) == ref == decode(np.maximum(keys_a, keys_b))
    k2, xk2, _ = sr.calibrate_sharded(x_t, t_offset=0)
    assert (int(k2.item()), float(xk2.item())) == ref
