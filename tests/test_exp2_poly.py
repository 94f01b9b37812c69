"""The FMA-pipe exp2 of the attention kernel (csrc/exp2_poly.h), on the CPU.

The header is plain C++ for the host, so it is compiled here with g++ and compared with
the exactly rounded 2^x in fp64: the stated bound is a relative error of 7.5e-5 on
[-125, 8] (the kernel feeds the result to a bf16 rounding of relative size 2^-9).
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "unified_text_pixel_b200", "csrc", "exp2_poly.h")


@pytest.fixture(scope="module")
def poly(tmp_path_factory):
    d = tmp_path_factory.mktemp("exp2")
    src = d / "shim.cpp"
    src.write_text(
        f'#include <cmath>\n#include "{HDR}"\n'
        'extern "C" void run(const float* x, float* y, long n) {\n'
        "  for (long i = 0; i < n; ++i) y[i] = hgx::exp2_poly3(x[i]);\n}\n"
    )
    so = d / "shim.so"
    subprocess.run(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", str(src), "-o", str(so)], check=True)
    lib = ctypes.CDLL(str(so))
    lib.run.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_long]

    def f(x):
        x = np.ascontiguousarray(x, dtype=np.float32)
        y = np.empty_like(x)
        lib.run(x.ctypes.data, y.ctypes.data, x.size)
        return y

    return f


def test_relative_error_bound(poly):
    x = np.linspace(-125.0, 8.0, 4_000_001).astype(np.float32)
    y = poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert (np.abs(y - ref) / ref).max() <= 7.6e-5


def test_integer_powers_and_small_arguments(poly):
    n = np.arange(-120, 9).astype(np.float32)
    y = poly(n).astype(np.float64)
    assert (np.abs(y / np.exp2(n.astype(np.float64)) - 1.0)).max() <= 7.6e-5
    x = (np.random.default_rng(0).random(10000) - 0.5).astype(np.float32) * 1e-3
    assert (np.abs(poly(x) / np.exp2(x.astype(np.float64)) - 1.0)).max() <= 7.6e-5


def test_clamp_below_range(poly):
    y = poly(np.array([-126.0, -1000.0, -np.inf], dtype=np.float32)).astype(np.float64)
    assert np.all(y > 0) and np.all(y < 3e-38)
