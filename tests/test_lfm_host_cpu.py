"""The library's host-side Slaney filterbank builder (``csrc/lfm_host.h``,
which ``ae_lfm_logmel`` uploads as its sparse band table), built on its own
with g++ and checked on the CPU against the oracle's filterbank
(``oracle.lfm.slaney_filterbank``): the dense bank it encodes equals the
oracle's to float32 rounding, for several configurations, and a
configuration whose bands are too wide for the table is refused."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

from oracle import lfm as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HARNESS = r"""
#include "lfm_host.h"
extern "C" int bank(int sr, int n_fft, int n_mels, int max_bins, int *lo, float *w, int *widest) {
  ae_lfm_config c = {};
  c.sample_rate = sr; c.n_fft = n_fft; c.n_mels = n_mels;
  std::vector<int32_t> l; std::vector<float> v;
  if (!ae::lfm_bank(c, l, v, widest, max_bins)) return 0;
  for (int b = 0; b < n_mels; ++b) lo[b] = l[b];
  for (size_t i = 0; i < v.size(); ++i) w[i] = v[i];
  return 1;
}
extern "C" int pack(int sr, int n_fft, int n_mels, int *lo, int *cnt, int *off, float *wp, int *wband) {
  ae_lfm_config c = {};
  c.sample_rate = sr; c.n_fft = n_fft; c.n_mels = n_mels;
  std::vector<int32_t> l; std::vector<float> v; int widest = 0;
  if (!ae::lfm_bank(c, l, v, &widest, 32)) return -1;
  const ae::LfmPackedBank P = ae::lfm_bank_pack(l, v, n_mels, 32, 8);
  for (int b = 0; b < n_mels; ++b) { lo[b] = P.lo[b]; cnt[b] = P.cnt[b]; off[b] = P.off[b]; }
  for (size_t i = 0; i < P.w.size(); ++i) wp[i] = P.w[i];
  for (int i = 0; i < 9; ++i) wband[i] = P.wband[i];
  return (int)P.w.size();
}
"""


@pytest.fixture(scope="module")
def lib():
    out = os.path.join(ROOT, "_build", "lfm_host_test")
    os.makedirs(out, exist_ok=True)
    src, so = os.path.join(out, "harness.cpp"), os.path.join(out, "harness.so")
    with open(src, "w") as f:
        f.write(HARNESS)
    subprocess.run(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-I",
                    os.path.join(ROOT, "log_mel_front_b200", "csrc"), src, "-o", so], check=True)
    lb = ctypes.CDLL(so)
    lb.bank.argtypes = [ctypes.c_int] * 4 + [ctypes.c_void_p] * 3
    lb.pack.argtypes = [ctypes.c_int] * 3 + [ctypes.c_void_p] * 5
    return lb


def _dense(lib, sr, n_fft, n_mels, max_bins=32):
    lo = np.zeros(n_mels, np.int32)
    w = np.zeros(n_mels * max_bins, np.float32)
    widest = np.zeros(1, np.int32)
    ok = lib.bank(sr, n_fft, n_mels, max_bins, lo.ctypes.data, w.ctypes.data, widest.ctypes.data)
    if not ok:
        return None, int(widest[0])
    d = np.zeros((n_mels, n_fft // 2 + 1))
    for b in range(n_mels):
        for q in range(max_bins):
            if lo[b] + q <= n_fft // 2:
                d[b, lo[b] + q] += w[b * max_bins + q]
    return d, int(widest[0])


@pytest.mark.parametrize("sr,n_fft,n_mels", [(16000, 512, 128), (16000, 512, 80), (22050, 512, 96), (16000, 512, 64)])
def test_bank_matches_the_oracle(lib, sr, n_fft, n_mels):
    d, widest = _dense(lib, sr, n_fft, n_mels)
    assert d is not None and 1 <= widest <= 32
    o = L.slaney_filterbank(n_mels, n_fft, sr)
    assert np.max(np.abs(d - o)) <= 2e-7 * o.max()


def test_too_wide_bands_are_refused(lib):
    d, _ = _dense(lib, 16000, 512, 8)
    assert d is None


@pytest.mark.parametrize("sr,n_mels", [(16000, 128), (16000, 80), (22050, 96), (16000, 64)])
def test_packed_bank_and_warp_split(lib, sr, n_mels):
    """The packed table the spectrum kernel reads (first bin, bins up to the last
    nonzero weight, offset into one weight array) encodes the same dense bank,
    and the 8 warps' contiguous band runs cover every band once, each with at
    most its share of the work plus one band."""
    lo, cnt, off = (np.zeros(n_mels, np.int32) for _ in range(3))
    wp = np.zeros(n_mels * 32, np.float32)
    wband = np.zeros(9, np.int32)
    nnz = lib.pack(sr, 512, n_mels, lo.ctypes.data, cnt.ctypes.data, off.ctypes.data, wp.ctypes.data,
                   wband.ctypes.data)
    assert nnz == int(cnt.sum())
    d = np.zeros((n_mels, 257))
    for b in range(n_mels):
        assert off[b] == int(cnt[:b].sum())
        if cnt[b]:
            assert wp[off[b] + cnt[b] - 1] != 0.0
        d[b, lo[b]:lo[b] + cnt[b]] = wp[off[b]:off[b] + cnt[b]]
    ref, _ = _dense(lib, sr, 512, n_mels)
    assert np.array_equal(d, ref)
    assert wband[0] == 0 and wband[8] == n_mels and np.all(np.diff(wband) >= 0)
    work = cnt + 8
    share = work.sum() / 8
    for w in range(8):
        assert work[wband[w]:wband[w + 1]].sum() <= share + work.max()
