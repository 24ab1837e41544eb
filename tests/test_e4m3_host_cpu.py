"""The library's host-side e4m3 weight encoder (``csrc/e4m3_host.h``, which
``ae_model_create`` uses for AE_FP8), built on its own with g++ and checked on
the CPU: against torch's float8_e4m3fn conversion on every grid value, every
midpoint and random values; against the format's saturation; and row by row
against the oracle's quantisation (``oracle.e4m3_rows``), code for code, which
is what the GPU parity of the e4m3 model relies on."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

from oracle import oracle as O

torch = pytest.importorskip("torch")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HARNESS = r"""
#include "e4m3_host.h"
extern "C" void encode(const double *x, unsigned char *out, long n) {
  for (long i = 0; i < n; ++i) out[i] = ae::e4m3_code(x[i]);
}
extern "C" void quantise_rows(const float *w, long rows, long cols, unsigned char *codes, double *scales) {
  for (long r = 0; r < rows; ++r) ae::e4m3_quantise_row(w + r * cols, (size_t)cols, codes + r * cols, scales + r);
}
"""


@pytest.fixture(scope="module")
def lib():
    out = os.path.join(ROOT, "_build", "e4m3_host_test")
    os.makedirs(out, exist_ok=True)
    src, so = os.path.join(out, "harness.cpp"), os.path.join(out, "harness.so")
    with open(src, "w") as f:
        f.write(HARNESS)
    subprocess.run(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-I",
                    os.path.join(ROOT, "log_mel_front_b200", "csrc"), src, "-o", so], check=True)
    L = ctypes.CDLL(so)
    L.encode.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_long]
    L.quantise_rows.argtypes = [ctypes.c_void_p, ctypes.c_long, ctypes.c_long, ctypes.c_void_p, ctypes.c_void_p]
    return L


def _encode(L, x):
    x = np.ascontiguousarray(x, np.float64)
    out = np.zeros(len(x), np.uint8)
    L.encode(x.ctypes.data, out.ctypes.data, len(x))
    return out


def _torch_codes(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_codes_match_torch(lib):
    grid = O.e4m3_decode(np.arange(256, dtype=np.uint8))
    grid = np.unique(grid[np.isfinite(grid)])
    pos = grid[grid >= 0]
    mids = (pos[:-1] + pos[1:]) / 2
    r = np.random.default_rng(13)
    rand = (r.standard_normal(50_000) * np.exp(r.uniform(-14, 6.1, 50_000))).astype(np.float32).astype(np.float64)
    for x in (grid[grid != 0], mids, -mids, rand[np.abs(rand) < 448]):
        assert np.array_equal(_encode(lib, x), _torch_codes(x))


def test_saturation_and_zero(lib):
    c = _encode(lib, np.array([448.0, 460.0, 464.0, 1e9, -1e9, 0.0, -0.0]))
    assert c.tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x00, 0x80]


def test_rows_match_the_oracle_code_for_code(lib):
    r = np.random.default_rng(14)
    W = (0.02 * r.standard_normal((64, 1024))).astype(np.float32)
    W[3] = 0.0
    codes = np.zeros(W.shape, np.uint8)
    scales = np.zeros(W.shape[0])
    lib.quantise_rows(W.ctypes.data, W.shape[0], W.shape[1], codes.ctypes.data, scales.ctypes.data)
    vals, s = O.e4m3_rows(W)
    assert np.array_equal(scales, s)
    assert np.array_equal(O.e4m3_decode(codes), vals)
