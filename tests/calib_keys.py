"""A plain restatement, for the tests, of the per-channel calibration keys the C ABI keeps in its
workspace (include/signrot.h, signrot_calibrate): for every channel i the largest |x_{t,i}|, the
first token attaining it and that value's sign, packed as one 64-bit key

    key = bits(|x| as fp32) << 32  |  (2^31 - 1 - t) << 1  |  sign bit of x

so that the larger key is the larger magnitude, then the earlier token. The outlier channel is
the lowest channel of the largest magnitude; its signed value is rebuilt from the key.
"""
import numpy as np


def fold_keys(x: np.ndarray, t_offset: int = 0) -> np.ndarray:
    """Keys of rows x [T, n] (values exactly representable in fp32), token indices t_offset + t."""
    x32 = np.atleast_2d(np.asarray(x, dtype=np.float64)).astype(np.float32)
    bits = x32.view(np.uint32).astype(np.uint64)
    mag = bits & np.uint64(0x7FFFFFFF)
    sign = bits >> np.uint64(31)
    t = np.arange(x32.shape[0], dtype=np.uint64)[:, None] + np.uint64(t_offset)
    order = (np.uint64(0x7FFFFFFF) - t) << np.uint64(1)
    keys = (mag << np.uint64(32)) | order | sign
    return keys.max(axis=0)


def decode(keys: np.ndarray) -> tuple[int, float]:
    """(k, x_k) from folded keys: the lowest channel of the largest magnitude and its signed value."""
    keys = np.asarray(keys).astype(np.uint64)
    mag = (keys >> np.uint64(32)).astype(np.uint32)
    k = int(np.flatnonzero(mag == mag.max())[0])
    v = float(np.array([mag[k]], dtype=np.uint32).view(np.float32)[0])
    return k, (-v if int(keys[k]) & 1 else v)
