"""The step kernel's correctly rounded scale divisions, checked exhaustively
on the GPU.

New scales s' = RN(A/qmax) and inv = RN(qmax/A) must equal IEEE division bit
for bit (the parity tests compare scales exactly), but the kernel computes
them with Markstein's remainder correction (lrs_device.cuh: div_by_qmax,
div_rn_fast; step_kernel.cuh: new_scales). tests/division_check.cu runs
every binary32 significand at every exponent of the ranges those routines
are used over (A in [2^-100, 2^128), the inverse's fast path up to 2^100,
new_scales' IEEE fallback above it) against __fdiv_rn.
"""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "quantized_recurrent_state_decode_b200", "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")


def _build(tmp):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    so = os.path.join(tmp, "division_check.so")
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O3",
           "-fmad=false", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC", "-shared",
           "-I", CSRC, "-I", INCLUDE, os.path.join(HERE, "division_check.cu"), "-o", so]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return so


def test_scale_divisions_are_correctly_rounded(tmp_path):
    L = ctypes.CDLL(_build(str(tmp_path)))
    L.run_division_check.restype = ctypes.c_int
    checked = ctypes.c_ulonglong(0)
    bad = (ctypes.c_ulonglong * 6)()
    first = (ctypes.c_uint32 * 6)()
    rc = L.run_division_check(-100, 127, ctypes.byref(checked), bad, first)
    assert rc == 0
    assert checked.value == (1 << 23) * 228
    names = ["A/127", "A/7", "127/A", "7/A", "new_scales int8", "new_scales int4"]
    msg = ["%s: %d wrong, first at %s" % (n, b, np.uint32(f).view(np.float32))
           for n, b, f in zip(names, bad, first) if b]
    assert not msg, "; ".join(msg)
