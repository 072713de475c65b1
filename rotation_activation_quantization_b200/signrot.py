"""Python binding of the SignRot C ABI (include/signrot.h): argument marshalling only.

Every step of the path runs in the CUDA library ``lib/libsignrot.so``; this module checks tensor
placement, dtypes and strides, allocates outputs with torch when the caller does not pass them,
and forwards raw device pointers and the current CUDA stream. There is no CPU fallback: if the
library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libsignrot.so")
_lib = None

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED_N, ERR_ALIGNMENT, ERR_CUDA, ERR_UNSUPPORTED = range(6)
BF16, F32 = 0, 1

_c_i32, _c_i64, _c_p, _c_f = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_float

_SIGNATURES = {
    "signrot_calibrate": [_c_p, _c_i32, _c_i64, _c_i32, _c_i64, _c_i64, _c_p, _c_i32, _c_p, _c_p, _c_p],
    "signrot_calibrate_static": [_c_p, _c_i32, _c_i64, _c_i32, _c_i64, _c_i64, _c_i32, _c_p, _c_p, _c_p],
    "signrot_build_sign": [_c_i32, _c_p, _c_p, _c_p, _c_p, _c_p],
    "signrot_rotate": [_c_p, _c_i32, _c_i64, _c_i32, _c_i64, _c_p, _c_p, _c_p, _c_i64, _c_p],
    "signrot_rotate_quant": [_c_p, _c_i32, _c_i64, _c_i32, _c_i64, _c_p, _c_p, _c_i32, _c_f,
                             _c_p, _c_p, _c_p, _c_p],
    "signrot_rotate_outlier": [_c_p, _c_i32, _c_i64, _c_i32, _c_i64, _c_p, _c_p, _c_p, _c_p, _c_i64, _c_p],
    "signrot_rotate_quant_outlier": [_c_p, _c_i32, _c_i64, _c_i32, _c_i64, _c_p, _c_p, _c_p, _c_i32, _c_f,
                                     _c_p, _c_p, _c_p, _c_p],
    "signrot_rotate_quant_sym": [_c_p, _c_i32, _c_i64, _c_i32, _c_i64, _c_p, _c_p, _c_i32, _c_p, _c_p, _c_p],
    "signrot_rotate_quant_sym_outlier": [_c_p, _c_i32, _c_i64, _c_i32, _c_i64, _c_p, _c_p, _c_p, _c_i32, _c_p,
                                         _c_p, _c_p],
    "signrot_device_error": [_c_p, _c_i32],
    "signrot_w4a4_prepare_weights": [_c_p, _c_i32, _c_i32, _c_i64, _c_p, _c_i64, _c_p, _c_p],
    "signrot_w4a4_matmul": [_c_p, _c_i64, _c_i32, _c_i64, _c_p, _c_p, _c_p, _c_i32, _c_i64, _c_p, _c_p, _c_p,
                            _c_i64, _c_p],
    "signrot_rotate_quant_host": [_c_p, _c_i32, _c_i64, _c_i32, _c_i64, _c_p, _c_p, _c_p, _c_p, _c_i32, _c_f,
                                  _c_p, _c_p, _c_p, _c_p, ctypes.c_size_t, _c_p],
    "signrot_host_bytes_per_token": [_c_i32, _c_i32],
    "signrot_get_h28": [_c_p],
    "signrot_get_h344": [_c_p],
    "signrot_supported_n": [_c_i32],
    "signrot_status_string": [_c_i32],
    "signrot_last_error": [],
    "signrot_kernel_launches": [],
}

EXPORTED = tuple(_SIGNATURES)


class SignRotError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str):
        super().__init__(f"{fn} failed with status {status}: {detail}")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """Load libsignrot.so (once). Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "`python -m rotation_activation_quantization_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        for name, args in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int32
        L.signrot_status_string.restype = ctypes.c_char_p
        L.signrot_last_error.restype = ctypes.c_char_p
        L.signrot_kernel_launches.restype = ctypes.c_uint64
        L.signrot_host_bytes_per_token.restype = ctypes.c_size_t
        _lib = L
    return _lib


def _check(fn: str, status: int) -> None:
    if status != OK:
        L = lib()
        detail = L.signrot_last_error().decode() or L.signrot_status_string(status).decode()
        raise SignRotError(fn, status, detail)


def _dtype_code(x: torch.Tensor) -> int:
    if x.dtype == torch.bfloat16:
        return BF16
    if x.dtype == torch.float32:
        return F32
    raise TypeError(f"activations must be bfloat16 or float32, got {x.dtype}")


def _rows(x: torch.Tensor) -> tuple[int, int, int]:
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D [T, n] tensor with unit stride along n")
    if not x.is_cuda:
        raise ValueError("x must be a CUDA tensor")
    return x.shape[0], x.shape[1], x.stride(0) if x.shape[0] > 1 else x.shape[1]


def _stream(dev: torch.device, stream) -> int:
    s = torch.cuda.current_stream(dev) if stream is None else stream
    return s.cuda_stream


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, dev, dtype, numel, name):
    if t.device != dev or t.dtype != dtype or t.numel() < numel or not t.is_contiguous():
        raise ValueError(f"{name}: need a contiguous {dtype} tensor with >= {numel} elements on {dev}")


def kernel_launches() -> int:
    """Kernels launched by the library so far in this process."""
    return int(lib().signrot_kernel_launches())


def supported_n(n: int) -> bool:
    return bool(lib().signrot_supported_n(int(n)))


def get_h28() -> np.ndarray:
    out = np.zeros(28 * 28, dtype=np.int8)
    _check("signrot_get_h28", lib().signrot_get_h28(out.ctypes.data))
    return out.reshape(28, 28)


def get_h344() -> np.ndarray:
    out = np.zeros(344 * 344, dtype=np.int8)
    _check("signrot_get_h344", lib().signrot_get_h344(out.ctypes.data))
    return out.reshape(344, 344)


def calibrate(x: torch.Tensor, ws: torch.Tensor | None = None, accumulate: bool = False,
              t_offset: int = 0, k_out: torch.Tensor | None = None,
              xk_out: torch.Tensor | None = None, stream=None):
    """Fold calibration rows x [T, n] into ws [n] (int64 storage of the uint64 keys) and return
    (k, x_k) as 1-element device tensors (int32, float32). Returns (k, x_k, ws)."""
    T, n, ld = _rows(x)
    dev = x.device
    ws = torch.empty(n, dtype=torch.int64, device=dev) if ws is None else ws
    _need(ws, dev, torch.int64, n, "ws")
    k_out = torch.empty(1, dtype=torch.int32, device=dev) if k_out is None else k_out
    xk_out = torch.empty(1, dtype=torch.float32, device=dev) if xk_out is None else xk_out
    with torch.cuda.device(dev):
        st = lib().signrot_calibrate(_ptr(x), _dtype_code(x), T, n, ld, int(t_offset), _ptr(ws),
                                     int(bool(accumulate)), _ptr(k_out), _ptr(xk_out), _stream(dev, stream))
    _check("signrot_calibrate", st)
    return k_out, xk_out, ws


def calibrate_finish(ws: torch.Tensor, k_out: torch.Tensor | None = None,
                     xk_out: torch.Tensor | None = None, stream=None):
    """(k, x_k) from keys ws [n] that are already folded (signrot_calibrate with no rows and
    accumulate = 1: only the argmax runs). Returns (k, x_k)."""
    n = ws.numel()
    dev = ws.device
    _need(ws, dev, torch.int64, n, "ws")
    k_out = torch.empty(1, dtype=torch.int32, device=dev) if k_out is None else k_out
    xk_out = torch.empty(1, dtype=torch.float32, device=dev) if xk_out is None else xk_out
    with torch.cuda.device(dev):
        st = lib().signrot_calibrate(None, BF16, 0, n, n, 0, _ptr(ws), 1, _ptr(k_out), _ptr(xk_out),
                                     _stream(dev, stream))
    _check("signrot_calibrate", st)
    return k_out, xk_out


def calibrate_sharded(x: torch.Tensor, t_offset: int, ws: torch.Tensor | None = None, group=None,
                      stream=None):
    """Calibration over a set split across ranks: this rank's rows x [T, n], whose first row is
    token t_offset of the whole set. Folds the rows into keys (CUDA), merges the keys of all
    ranks by one all-reduce(MAX) over the process group (NCCL), then takes the argmax (CUDA).
    Every rank returns the same (k, x_k), equal to calibrating the whole set at once."""
    from . import sharding

    _, _, ws = calibrate(x, ws=ws, accumulate=False, t_offset=t_offset, stream=stream)
    sharding.merge_calibration(ws, group)
    k, xk = calibrate_finish(ws, stream=stream)
    return k, xk, ws


def calibrate_static(x: torch.Tensor, accumulate: bool = False, t_offset: int = 0,
                     k_out: torch.Tensor | None = None, xk_out: torch.Tensor | None = None, stream=None):
    """calibrate() with the workspace kept in the library's fixed device array (no allocation by
    the library; outputs are allocated here only when not passed). Returns (k, x_k)."""
    T, n, ld = _rows(x)
    dev = x.device
    k_out = torch.empty(1, dtype=torch.int32, device=dev) if k_out is None else k_out
    xk_out = torch.empty(1, dtype=torch.float32, device=dev) if xk_out is None else xk_out
    with torch.cuda.device(dev):
        st = lib().signrot_calibrate_static(_ptr(x), _dtype_code(x), T, n, ld, int(t_offset),
                                            int(bool(accumulate)), _ptr(k_out), _ptr(xk_out), _stream(dev, stream))
    _check("signrot_calibrate_static", st)
    return k_out, xk_out


def build_sign(n: int, k: torch.Tensor, xk: torch.Tensor, d: torch.Tensor,
               s_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    dev = d.device
    _need(d, dev, torch.int8, n, "d")
    _need(k, dev, torch.int32, 1, "k")
    _need(xk, dev, torch.float32, 1, "xk")
    s_out = torch.empty(n, dtype=torch.int8, device=dev) if s_out is None else s_out
    _need(s_out, dev, torch.int8, n, "s_out")
    with torch.cuda.device(dev):
        st = lib().signrot_build_sign(int(n), _ptr(k), _ptr(xk), _ptr(d), _ptr(s_out), _stream(dev, stream))
    _check("signrot_build_sign", st)
    return s_out


def rotate(x: torch.Tensor, d: torch.Tensor, s: torch.Tensor | None = None,
           out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """fp32 y = s (.) H D x / sqrt(n) for every row of x [T, n]."""
    T, n, ld = _rows(x)
    dev = x.device
    _need(d, dev, torch.int8, n, "d")
    if s is not None:
        _need(s, dev, torch.int8, n, "s")
    out = torch.empty((T, n), dtype=torch.float32, device=dev) if out is None else out
    if out.shape != (T, n) or out.stride(1) != 1 or out.dtype != torch.float32 or out.device != dev:
        raise ValueError("out must be a float32 [T, n] tensor with unit stride along n on x's device")
    ldy = out.stride(0) if T > 1 else n
    with torch.cuda.device(dev):
        st = lib().signrot_rotate(_ptr(x), _dtype_code(x), T, n, ld, _ptr(d), _ptr(s), _ptr(out), ldy,
                                  _stream(dev, stream))
    _check("signrot_rotate", st)
    return out


def rotate_quant(x: torch.Tensor, d: torch.Tensor, s: torch.Tensor | None = None, bits: int = 4,
                 clip: float = 1.0, q: torch.Tensor | None = None, scale: torch.Tensor | None = None,
                 zero: torch.Tensor | None = None, stream=None):
    """The fused path: returns (q uint8 [T, n/2] (bits 4) or [T, n] (bits 8), scale f32 [T], zero f32 [T])."""
    T, n, ld = _rows(x)
    dev = x.device
    _need(d, dev, torch.int8, n, "d")
    if s is not None:
        _need(s, dev, torch.int8, n, "s")
    qn = _q_row_bytes(n, bits)
    q = torch.empty((T, qn), dtype=torch.uint8, device=dev) if q is None else q
    scale = torch.empty(T, dtype=torch.float32, device=dev) if scale is None else scale
    zero = torch.empty(T, dtype=torch.float32, device=dev) if zero is None else zero
    _need(q, dev, torch.uint8, T * qn, "q")
    _need(scale, dev, torch.float32, T, "scale")
    _need(zero, dev, torch.float32, T, "zero")
    with torch.cuda.device(dev):
        st = lib().signrot_rotate_quant(_ptr(x), _dtype_code(x), T, n, ld, _ptr(d), _ptr(s), int(bits),
                                        float(clip), _ptr(q), _ptr(scale), _ptr(zero), _stream(dev, stream))
    _check("signrot_rotate_quant", st)
    return q, scale, zero


def rotate_outlier(x: torch.Tensor, d: torch.Tensor, k: torch.Tensor, xk: torch.Tensor,
                   out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """fp32 rotation with the sign vector given by its outlier channel (k, x_k on the device)."""
    T, n, ld = _rows(x)
    dev = x.device
    _need(d, dev, torch.int8, n, "d")
    _need(k, dev, torch.int32, 1, "k")
    _need(xk, dev, torch.float32, 1, "xk")
    out = torch.empty((T, n), dtype=torch.float32, device=dev) if out is None else out
    if out.shape != (T, n) or out.stride(1) != 1 or out.dtype != torch.float32 or out.device != dev:
        raise ValueError("out must be a float32 [T, n] tensor with unit stride along n on x's device")
    ldy = out.stride(0) if T > 1 else n
    with torch.cuda.device(dev):
        st = lib().signrot_rotate_outlier(_ptr(x), _dtype_code(x), T, n, ld, _ptr(d), _ptr(k), _ptr(xk),
                                          _ptr(out), ldy, _stream(dev, stream))
    _check("signrot_rotate_outlier", st)
    return out


def rotate_quant_outlier(x: torch.Tensor, d: torch.Tensor, k: torch.Tensor, xk: torch.Tensor, bits: int = 4,
                         clip: float = 1.0, q: torch.Tensor | None = None, scale: torch.Tensor | None = None,
                         zero: torch.Tensor | None = None, stream=None):
    """The fused path with the sign vector folded in from (k, x_k): (q, scale, zero)."""
    T, n, ld = _rows(x)
    dev = x.device
    _need(d, dev, torch.int8, n, "d")
    _need(k, dev, torch.int32, 1, "k")
    _need(xk, dev, torch.float32, 1, "xk")
    qn = _q_row_bytes(n, bits)
    q = torch.empty((T, qn), dtype=torch.uint8, device=dev) if q is None else q
    scale = torch.empty(T, dtype=torch.float32, device=dev) if scale is None else scale
    zero = torch.empty(T, dtype=torch.float32, device=dev) if zero is None else zero
    _need(q, dev, torch.uint8, T * qn, "q")
    _need(scale, dev, torch.float32, T, "scale")
    _need(zero, dev, torch.float32, T, "zero")
    with torch.cuda.device(dev):
        st = lib().signrot_rotate_quant_outlier(_ptr(x), _dtype_code(x), T, n, ld, _ptr(d), _ptr(k), _ptr(xk),
                                                int(bits), float(clip), _ptr(q), _ptr(scale), _ptr(zero),
                                                _stream(dev, stream))
    _check("signrot_rotate_quant_outlier", st)
    return q, scale, zero


def _q_row_bytes(n: int, bits: int) -> int:
    return n if bits == 8 else n // 2


def rotate_quant_sym(x: torch.Tensor, d: torch.Tensor, s: torch.Tensor | None = None, bits: int = 4,
                     q: torch.Tensor | None = None, scale: torch.Tensor | None = None, stream=None):
    """Symmetric grid (codes -L..L, no zero-point): (q [T, n/2] two's-complement nibbles for bits 4,
    or int8 [T, n] for bits 8, scale f32 [T])."""
    T, n, ld = _rows(x)
    dev = x.device
    _need(d, dev, torch.int8, n, "d")
    if s is not None:
        _need(s, dev, torch.int8, n, "s")
    qn = _q_row_bytes(n, bits)
    q = torch.empty((T, qn), dtype=torch.int8 if bits == 8 else torch.uint8, device=dev) if q is None else q
    scale = torch.empty(T, dtype=torch.float32, device=dev) if scale is None else scale
    _need(q, dev, q.dtype, T * qn, "q")
    _need(scale, dev, torch.float32, T, "scale")
    with torch.cuda.device(dev):
        st = lib().signrot_rotate_quant_sym(_ptr(x), _dtype_code(x), T, n, ld, _ptr(d), _ptr(s), int(bits),
                                            _ptr(q), _ptr(scale), _stream(dev, stream))
    _check("signrot_rotate_quant_sym", st)
    return q, scale


def rotate_quant_sym_outlier(x: torch.Tensor, d: torch.Tensor, k: torch.Tensor, xk: torch.Tensor, bits: int = 4,
                             q: torch.Tensor | None = None, scale: torch.Tensor | None = None, stream=None):
    """Symmetric grid with the sign vector folded in from (k, x_k): (q, scale)."""
    T, n, ld = _rows(x)
    dev = x.device
    _need(d, dev, torch.int8, n, "d")
    _need(k, dev, torch.int32, 1, "k")
    _need(xk, dev, torch.float32, 1, "xk")
    qn = _q_row_bytes(n, bits)
    q = torch.empty((T, qn), dtype=torch.int8 if bits == 8 else torch.uint8, device=dev) if q is None else q
    scale = torch.empty(T, dtype=torch.float32, device=dev) if scale is None else scale
    _need(q, dev, q.dtype, T * qn, "q")
    _need(scale, dev, torch.float32, T, "scale")
    with torch.cuda.device(dev):
        st = lib().signrot_rotate_quant_sym_outlier(_ptr(x), _dtype_code(x), T, n, ld, _ptr(d), _ptr(k), _ptr(xk),
                                                    int(bits), _ptr(q), _ptr(scale), _stream(dev, stream))
    _check("signrot_rotate_quant_sym_outlier", st)
    return q, scale


def w4a4_prepare_weights(wq4: torch.Tensor, K: int, wq8: torch.Tensor | None = None,
                         colsum: torch.Tensor | None = None, stream=None):
    """Offline: packed signed 4-bit weight codes wq4 [N, K/2] (as rotate_quant_sym writes them for
    the rows of the folded weights) -> (wq8 [N, K] int8, colsum [N] int32)."""
    if wq4.dim() != 2 or wq4.dtype != torch.uint8 or wq4.stride(1) != 1 or wq4.shape[1] != K // 2:
        raise ValueError("wq4 must be a uint8 [N, K/2] tensor with unit stride along K")
    N, dev = wq4.shape[0], wq4.device
    wq8 = torch.empty((N, K), dtype=torch.int8, device=dev) if wq8 is None else wq8
    colsum = torch.empty(N, dtype=torch.int32, device=dev) if colsum is None else colsum
    if wq8.shape != (N, K) or wq8.stride(1) != 1 or wq8.dtype != torch.int8 or wq8.device != dev:
        raise ValueError("wq8 must be an int8 [N, K] tensor with unit stride along K")
    _need(colsum, dev, torch.int32, N, "colsum")
    with torch.cuda.device(dev):
        st = lib().signrot_w4a4_prepare_weights(_ptr(wq4), N, int(K), wq4.stride(0) if N > 1 else K // 2,
                                                _ptr(wq8), wq8.stride(0) if N > 1 else K, _ptr(colsum),
                                                _stream(dev, stream))
    _check("signrot_w4a4_prepare_weights", st)
    return wq8, colsum


def w4a4_matmul(q: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor | None, wq8: torch.Tensor,
                wscale: torch.Tensor, colsum: torch.Tensor, out: torch.Tensor | None = None, stream=None):
    """out [T, N] fp32 = scale_t wscale_o (sum_j code_tj wq8[o, j] - zero_t colsum_o) from packed
    activation codes q [T, K/2] (uint8) and int8 weight codes wq8 [N, K]; zero=None takes q as the
    symmetric grid's signed nibbles (no zero term)."""
    if q.dim() != 2 or q.dtype != torch.uint8 or q.stride(1) != 1 or not q.is_cuda:
        raise ValueError("q must be a CUDA uint8 [T, K/2] tensor with unit stride along K")
    T, K = q.shape[0], 2 * q.shape[1]
    if wq8.dim() != 2 or wq8.dtype != torch.int8 or wq8.stride(1) != 1 or wq8.shape[1] != K:
        raise ValueError("wq8 must be an int8 [N, K] tensor with unit stride along K")
    N, dev = wq8.shape[0], q.device
    _need(scale, dev, torch.float32, T, "scale")
    if zero is not None:
        _need(zero, dev, torch.float32, T, "zero")
    _need(wscale, dev, torch.float32, N, "wscale")
    _need(colsum, dev, torch.int32, N, "colsum")
    out = torch.empty((T, N), dtype=torch.float32, device=dev) if out is None else out
    if out.shape != (T, N) or out.stride(1) != 1 or out.dtype != torch.float32 or out.device != dev:
        raise ValueError("out must be a float32 [T, N] tensor with unit stride along N")
    with torch.cuda.device(dev):
        st = lib().signrot_w4a4_matmul(_ptr(q), T, K, q.stride(0) if T > 1 else K // 2, _ptr(scale), _ptr(zero),
                                       _ptr(wq8), N, wq8.stride(0) if N > 1 else K, _ptr(wscale), _ptr(colsum),
                                       _ptr(out), out.stride(0) if T > 1 else N, _stream(dev, stream))
    _check("signrot_w4a4_matmul", st)
    return out


def device_error(clear: bool = True) -> int:
    """The current device's error word (0 = none); synchronous."""
    code = ctypes.c_int32(0)
    _check("signrot_device_error", lib().signrot_device_error(ctypes.byref(code), int(bool(clear))))
    return int(code.value)


def host_bytes_per_token(n: int, dtype: torch.dtype = torch.bfloat16) -> int:
    return int(lib().signrot_host_bytes_per_token(int(n), BF16 if dtype == torch.bfloat16 else F32))


def rotate_quant_host(x: torch.Tensor, d: torch.Tensor, q: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor,
                      workspace: torch.Tensor, s: torch.Tensor | None = None, k: torch.Tensor | None = None,
                      xk: torch.Tensor | None = None, bits: int = 4, clip: float = 1.0, device=None, stream=None):
    """The fused path between host buffers (x, q, scale, zero on the CPU, pinned for overlap),
    streamed through a device workspace. Enqueued on the current stream of ``device``."""
    if x.dim() != 2 or x.stride(1) != 1 or x.is_cuda:
        raise ValueError("x must be a 2-D host tensor with unit stride along n")
    T, n = x.shape
    ld = x.stride(0) if T > 1 else n
    dev = torch.device(device) if device is not None else d.device
    if not workspace.is_cuda or workspace.device != dev:
        raise ValueError("workspace must be a device tensor on the same device as d")
    for t, name in ((q, "q"), (scale, "scale"), (zero, "zero")):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous host tensor")
    with torch.cuda.device(dev):
        st = lib().signrot_rotate_quant_host(
            _ptr(x), _dtype_code(x), T, n, ld, _ptr(d), _ptr(s), _ptr(k), _ptr(xk), int(bits), float(clip),
            _ptr(q), _ptr(scale), _ptr(zero), _ptr(workspace), workspace.numel() * workspace.element_size(),
            _stream(dev, stream))
    _check("signrot_rotate_quant_host", st)
    return q, scale, zero
