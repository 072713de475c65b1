"""signrot_calibrate_static, called through the C ABI, against signrot_calibrate.

The static entry point serves callers that cannot allocate device memory (a start-up memory pool,
a host framework that owns the allocator, latency-bound code that must not risk cudaMalloc's
device synchronisation): it keeps the calibration keys in the library's own fixed device array.
Its results must equal the workspace-taking entry point's exactly, on consecutive calls: a call
that continues a calibration (accumulate = 1) and calls that start a new one (accumulate = 0,
which must clear what the previous call left in the shared array).
"""
import ctypes

import numpy as np
import pytest

from rotation_activation_quantization_b200 import synthetic as syn

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rotation_activation_quantization_b200 import signrot

    return signrot.lib()


def _rows(index, t0, t1):
    w = syn.workload(index)
    x = syn.draw_calibration(w, t0, t1)
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda(), w.n


def _call_static(lib, x, t_offset, accumulate):
    T, n = x.shape
    k = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    xk = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    st = lib.signrot_calibrate_static(x.data_ptr(), 0, T, n, n, t_offset, accumulate, k.data_ptr(),
                                      xk.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 0, lib.signrot_last_error()
    torch.cuda.synchronize()
    return int(k.item()), float(xk.item())


def _call_workspace(lib, x, ws, t_offset, accumulate):
    T, n = x.shape
    k = torch.empty(1, dtype=torch.int32, device="cuda")
    xk = torch.empty(1, dtype=torch.float32, device="cuda")
    st = lib.signrot_calibrate(x.data_ptr(), 0, T, n, n, t_offset, ws.data_ptr(), accumulate, k.data_ptr(),
                               xk.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 0, lib.signrot_last_error()
    torch.cuda.synchronize()
    return int(k.item()), float(xk.item())


def test_two_consecutive_calls_continue_a_calibration(lib):
    a, n = _rows(3, 0, 700)
    b, _ = _rows(3, 700, 2048)
    ws = torch.empty(n, dtype=torch.int64, device="cuda")
    expect1 = _call_workspace(lib, a, ws, 0, 0)
    expect2 = _call_workspace(lib, b, ws, 700, 1)
    assert _call_static(lib, a, 0, 0) == expect1
    assert _call_static(lib, b, 700, 1) == expect2


def test_two_consecutive_fresh_calls_clear_the_shared_array(lib):
    big, n = _rows(4, 0, 512)      # n = 28672: leaves large keys behind in the shared array
    small, m = _rows(2, 0, 512)    # n = 4096: a new calibration must not see them
    ws_big = torch.empty(n, dtype=torch.int64, device="cuda")
    ws_small = torch.empty(m, dtype=torch.int64, device="cuda")
    assert _call_static(lib, big, 0, 0) == _call_workspace(lib, big, ws_big, 0, 0)
    assert _call_static(lib, small, 0, 0) == _call_workspace(lib, small, ws_small, 0, 0)


def test_longest_row_and_no_device_allocation(lib):
    """The longest supported row (n = 32768, the array's full size) equals the workspace entry
    point, and a warmed-up call leaves the device's free memory unchanged: it allocates nothing."""
    n = 32768
    g = torch.Generator().manual_seed(5)
    x = (torch.randn((300, n), generator=g) * 0.3).to(torch.bfloat16)
    x[123, 31000] = 2500.0
    x = x.cuda()
    ws = torch.empty(n, dtype=torch.int64, device="cuda")
    expect = _call_workspace(lib, x, ws, 0, 0)
    assert expect[0] == 31000
    assert _call_static(lib, x, 0, 0) == expect
    k = torch.empty(1, dtype=torch.int32, device="cuda")
    xk = torch.empty(1, dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        st = lib.signrot_calibrate_static(x.data_ptr(), 0, 300, n, n, 0, 0, k.data_ptr(), xk.data_ptr(),
                                          torch.cuda.current_stream().cuda_stream)
        assert st == 0, lib.signrot_last_error()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert int(k.item()) == 31000


def test_rejects_unsupported_rows_before_touching_the_device(lib):
    x = torch.zeros((2, 65536), dtype=torch.bfloat16, device="cuda")
    k = torch.empty(1, dtype=torch.int32, device="cuda")
    xk = torch.empty(1, dtype=torch.float32, device="cuda")
    st = lib.signrot_calibrate_static(x.data_ptr(), 0, 2, 65536, 65536, 0, 0, k.data_ptr(), xk.data_ptr(), None)
    assert st == 2  # the same status signrot_calibrate gives for this n
    assert b"65536" in lib.signrot_last_error()
    st = lib.signrot_calibrate_static(None, 0, 2, 4096, 4096, 0, 0, k.data_ptr(), xk.data_ptr(), None)
    assert st == 1
