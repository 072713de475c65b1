"""Host-side checks of the C ABI (no GPU needed, no kernel launched): the library loads, exports
every function include/signrot.h declares, its own Paley H_28 equals the oracle's entry by entry,
and argument validation returns status codes before any CUDA call."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from oracle import signrot_oracle as o

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "signrot.h")


@pytest.fixture(scope="module")
def binding():
    from rotation_activation_quantization_b200 import signrot

    if not os.path.exists(signrot.library_path()):
        from rotation_activation_quantization_b200 import build

        build.build()
    return signrot


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(signrot_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_path():
    fns = declared_functions()
    for f in ("signrot_calibrate", "signrot_build_sign", "signrot_rotate", "signrot_rotate_quant"):
        assert f in fns


def test_library_exports_every_declared_symbol(binding):
    lib = binding.lib()
    fns = declared_functions()
    for f in fns:
        assert hasattr(lib, f), f
    out = subprocess.run(["nm", "-D", "--defined-only", binding.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (signrot_[a-z0-9_]+)\b", out))
    assert set(fns) <= exported
    assert set(binding.EXPORTED) == set(fns)


def test_library_h28_equals_oracle_h28(binding):
    assert (binding.get_h28() == o.paley_h28()).all()


def test_library_h344_equals_oracle_h344(binding):
    h = binding.get_h344()
    assert (h == o.paley_h344()).all()
    # and, apart from the oracle: a skew Hadamard matrix with the stated border
    assert (h.astype(np.int64) @ h.T.astype(np.int64) == 344 * np.eye(344, dtype=np.int64)).all()
    assert (h + h.T == 2 * np.eye(344, dtype=np.int8)).all()
    assert (h[0] == 1).all() and (h[1:, 0] == -1).all()


def test_supported_n_matches_oracle(binding):
    for n in list(range(0, 400)) + [688, 1024, 4096, 5504, 11008, 14336, 22016, 28672, 32768, 65536,
                                    28 * 2048]:
        try:
            F, M = o.factor_n(n)
            expect = (F == 1 and n <= 32768) or (F == 28 and M <= 1024) or (F == 344 and M <= 32)
        except ValueError:
            expect = False
        assert binding.supported_n(n) == expect, n


def _rq(lib, **kw):
    a = dict(x=1 << 20, dtype=0, T=4, n=1024, ld=1024, d=1 << 21, s=None, bits=4, clip=1.0,
             q=1 << 22, scale=1 << 23, zero=1 << 24)
    a.update(kw)
    return lib.signrot_rotate_quant(a["x"], a["dtype"], a["T"], a["n"], a["ld"], a["d"], a["s"],
                                    a["bits"], ctypes.c_float(a["clip"]), a["q"], a["scale"],
                                    a["zero"], None)


def test_validation_codes_without_cuda(binding):
    lib = binding.lib()
    assert _rq(lib, n=1000) == binding.ERR_UNSUPPORTED_N
    assert _rq(lib, n=28 * 2048) == binding.ERR_UNSUPPORTED_N
    assert _rq(lib, n=1) == binding.ERR_UNSUPPORTED_N
    assert _rq(lib, bits=5) == binding.ERR_UNSUPPORTED
    assert _rq(lib, bits=2) == binding.ERR_UNSUPPORTED
    assert _rq(lib, clip=0.0) == binding.ERR_UNSUPPORTED
    assert _rq(lib, clip=1.5) == binding.ERR_UNSUPPORTED
    assert _rq(lib, dtype=7) == binding.ERR_INVALID_ARG
    assert _rq(lib, T=-1) == binding.ERR_INVALID_ARG
    assert _rq(lib, ld=512) == binding.ERR_INVALID_ARG
    assert _rq(lib, x=None) == binding.ERR_INVALID_ARG
    assert _rq(lib, d=None) == binding.ERR_INVALID_ARG
    assert _rq(lib, q=None) == binding.ERR_INVALID_ARG
    assert _rq(lib, x=(1 << 20) + 1) == binding.ERR_ALIGNMENT
    assert _rq(lib, dtype=1, x=(1 << 20) + 2) == binding.ERR_ALIGNMENT
    assert _rq(lib, scale=(1 << 23) + 2) == binding.ERR_ALIGNMENT
    assert _rq(lib, T=0) == binding.OK  # a no-op, no CUDA call
    assert lib.signrot_rotate(None, 0, 0, 1000, 1000, 1, None, None, 1000, None) == binding.ERR_UNSUPPORTED_N
    assert lib.signrot_rotate(1 << 20, 0, 2, 64, 64, None, None, 1 << 21, 64, None) == binding.ERR_INVALID_ARG
    assert lib.signrot_rotate(1 << 20, 0, 2, 64, 64, 1 << 22, None, 1 << 21, 32, None) == binding.ERR_INVALID_ARG
    assert lib.signrot_build_sign(100, 1 << 20, 1 << 21, 1 << 22, 1 << 23, None) == binding.ERR_UNSUPPORTED_N
    assert lib.signrot_build_sign(64, None, 1 << 21, 1 << 22, 1 << 23, None) == binding.ERR_INVALID_ARG
    assert lib.signrot_calibrate(1 << 20, 0, 4, 64, 64, 0, None, 0, 1 << 21, 1 << 22, None) == binding.ERR_INVALID_ARG
    assert lib.signrot_calibrate(1 << 20, 0, 4, 64, 64, 0, (1 << 21) + 4, 0, 1 << 22, 1 << 23, None) == binding.ERR_ALIGNMENT
    assert lib.signrot_calibrate(1 << 20, 0, 4, 64, 64, 0x7ffffffe, 1 << 21, 0, 1 << 22, 1 << 23, None) == binding.ERR_INVALID_ARG
    assert lib.signrot_get_h28(None) == binding.ERR_INVALID_ARG
    # the symmetric grid: bits 4 or 8, scale required, no zero-point pointer
    sym = lib.signrot_rotate_quant_sym
    assert sym(1 << 20, 0, 4, 1024, 1024, 1 << 21, None, 6, 1 << 22, 1 << 23, None) == binding.ERR_UNSUPPORTED
    assert sym(1 << 20, 0, 4, 1024, 1024, 1 << 21, None, 4, 1 << 22, None, None) == binding.ERR_INVALID_ARG
    assert sym(1 << 20, 0, 4, 1000, 1000, 1 << 21, None, 4, 1 << 22, 1 << 23, None) == binding.ERR_UNSUPPORTED_N
    assert sym(1 << 20, 0, 0, 1024, 1024, 1 << 21, None, 8, 1 << 22, 1 << 23, None) == binding.OK
    symo = lib.signrot_rotate_quant_sym_outlier
    assert symo(1 << 20, 0, 4, 1024, 1024, 1 << 21, None, 1 << 24, 4, 1 << 22, 1 << 23, None) == binding.ERR_INVALID_ARG


def test_error_messages(binding):
    lib = binding.lib()
    assert _rq(lib, n=1000) == binding.ERR_UNSUPPORTED_N
    assert b"n = 1000" in lib.signrot_last_error()
    for st in range(6):
        assert lib.signrot_status_string(st)


def test_bench_reference_arm_prints_the_contract_line():
    """bench.py --impl reference on the CPU: one JSON line with the contract's keys, K steps."""
    import json
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--config", "2",
                          "--steps", "3", "--warmup", "1"], capture_output=True, text=True, check=True,
                         cwd=root, timeout=600).stdout.strip().splitlines()
    line = json.loads(out[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "impl"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 3 and line["warmup"] == 1
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["config"]["workload"]


def test_bench_bytes_per_token():
    """Algorithmic bytes per token: bf16 row in, codes out, fp32 scale (+ zero). C3 and C4 give the
    35 848 and 71 688 B of the measurement plan; INT8 and symmetric grids move accordingly."""
    import importlib.util

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(root, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    from rotation_activation_quantization_b200 import synthetic as syn

    w3, w4, w1 = syn.workload(3), syn.workload(4), syn.workload(1)
    assert bench.bytes_per_token(w3) == 35848
    assert bench.bytes_per_token(w4) == 71688
    assert bench.bytes_per_token(w1) == 4 * 1024 + 512 + 8  # fp32 rows
    assert bench.bytes_per_token(w3, "asym8") == 2 * 14336 + 14336 + 8
    assert bench.bytes_per_token(w3, "sym4") == 2 * 14336 + 7168 + 4
    assert bench.bytes_per_token(w3, "sym8") == 2 * 14336 + 14336 + 4
