"""Plain float64 CPU oracle of the audio input conditioning: channel mixdown
and band-limited resampling to 16 kHz.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: the parity tests and
``bench.py``'s CPU legs call it; the CUDA library never does, and nothing
here is shared with it.

Source: the docs.rs page of cortiq-engine 0.8.49, ``egemma2_audio.rs``, items
``to_mono_16k`` (mixdown, then resample), ``bessel_i0`` and ``resample_hq``
(the polyphase Kaiser-windowed sinc with its constants ``RS_WIDTH`` 64 zero
crossings a side, ``RS_ROLLOFF`` 0.958 of the lower Nyquist, ``RS_BETA``
12.8), and the page's tests ``stereo_mixes_down_and_rates_resample`` and
``resampling_keeps_a_tone_and_its_length``.

What is computed, written as the plain definition rather than in the page's
table-and-span form:

* mono[i] = (x_0[i] + x_1[i] + ... + x_{C-1}[i]) / C, summed in channel order
  in float32 (the page sums and divides float32 values); one channel is
  passed through unchanged;
* with g = gcd(from, to), o = from / g, p = to / g, the output has
  ceil(p N / o) samples; output n sits at input position tau_n = n o / p, and

      y[n] = sum over input samples m with |t| < 64 of
             x[m] * c * sinc(t) * I0(beta sqrt(1 - (t/64)^2)) / I0(beta),
      t = (m - tau_n) * c,   c = 0.958 min(o, p) / o,

  sinc(t) = sin(pi t) / (pi t) (1 at 0), samples outside the clip are zero,
  all in float64, the result rounded to float32;
* equal rates, or an empty input, return the input.

The page evaluates t as ((m - f o) / o - j / p) * 0.958 min(o, p) with
f = n div p and j = n mod p, the same number up to float64 rounding; the page's
phase table and tap span only skip taps whose t is outside the window.

Parity status: pinned by the page's own tests (exact lengths, tones within
1e-4 of the ideal, a tone above the new Nyquist removed to RMS < 1e-4, the
stereo mixdown example, DC level), by I0 against numpy's ``i0``, and by a
brute-force restatement on tiny inputs.
"""
from __future__ import annotations

import math

import numpy as np

RS_WIDTH = 64.0
RS_ROLLOFF = 0.958
RS_BETA = 12.8
OUT_RATE = 16000


def bessel_i0(x: float) -> float:
    """Modified Bessel function of the first kind of order 0 by its power
    series sum_k ((x/2)^2)^k / (k!)^2, summed until the terms stop
    contributing (``bessel_i0``)."""
    q = x * x / 4.0
    term = total = 1.0
    k = 1
    while k < 400:
        term *= q / (k * k)
        total += term
        if term < total * 1e-17:
            break
        k += 1
    return total


def bessel_i0_array(x: np.ndarray) -> np.ndarray:
    """``bessel_i0`` elementwise over an array: the same series, summed for
    every element until each one's terms stop contributing."""
    x = np.asarray(x, np.float64)
    q = x * x / 4.0
    term = np.ones_like(q)
    total = np.ones_like(q)
    for k in range(1, 400):
        term = term * q / (k * k)
        total = total + term
        if np.all(term < total * 1e-17):
            break
    return total


def mixdown(channels: list) -> np.ndarray:
    """``to_mono_16k``'s channel average, float32 as on the page."""
    if len(channels) == 0:
        return np.zeros(0, np.float32)
    if len(channels) == 1:
        return np.asarray(channels[0], np.float32).copy()
    acc = np.asarray(channels[0], np.float32).copy()
    for ch in channels[1:]:
        acc = (acc + np.asarray(ch, np.float32)).astype(np.float32)
    return (acc / np.float32(len(channels))).astype(np.float32)


def reduced_rates(src: int, dst: int) -> tuple[int, int]:
    g = math.gcd(src, dst)
    return src // g, dst // g


def resample_len(n: int, src: int, dst: int = OUT_RATE) -> int:
    """Number of output samples: ceil(p N / o) with the reduced rates; the
    input length itself for equal rates or an empty input."""
    if src == dst or n == 0:
        return n
    o, p = reduced_rates(src, dst)
    return -((-p * n) // o)


def resample(x: np.ndarray, src: int, dst: int = OUT_RATE) -> np.ndarray:
    """``resample_hq`` by its definition (see the module notes)."""
    x = np.asarray(x, np.float32)
    if src == dst or len(x) == 0:
        return x.copy()
    o, p = reduced_rates(src, dst)
    n_in = len(x)
    n_out = resample_len(n_in, src, dst)
    c = RS_ROLLOFF * min(o, p) / o
    half = RS_WIDTH / c  # window half-width in input samples
    i0b = bessel_i0(RS_BETA)
    xd = x.astype(np.float64)
    y = np.zeros(n_out, np.float64)
    # outputs of one phase j = n mod p share their tap values; evaluate them once per phase
    for j in range(min(p, n_out)):
        frac = o * j / p  # tau_n - f o for n = f p + j
        m_lo = math.floor(frac - half)
        m_hi = math.ceil(frac + half)
        d = np.arange(m_lo, m_hi + 1)  # m - f o
        t = (d - frac) * c
        inside = np.abs(t) < RS_WIDTH
        d, t = d[inside], t[inside]
        r = t / RS_WIDTH
        win = bessel_i0_array(RS_BETA * np.sqrt(1.0 - r * r)) / i0b
        pt = math.pi * t
        sinc = np.where(pt == 0.0, 1.0, np.sin(pt) / np.where(pt == 0.0, 1.0, pt))
        taps = sinc * win * c
        f = np.arange((n_out - j + p - 1) // p)  # frames that have phase j
        m = f[:, None] * o + d[None, :]
        valid = (m >= 0) & (m < n_in)
        vals = np.where(valid, xd[np.clip(m, 0, n_in - 1)], 0.0)
        y[f * p + j] = vals @ taps
    return y.astype(np.float32)


def resample_direct(x: np.ndarray, src: int, dst: int = OUT_RATE) -> np.ndarray:
    """The same definition as two plain loops over outputs and inputs, for
    tiny inputs (a brute-force check of ``resample``'s phase grouping)."""
    x = np.asarray(x, np.float32)
    if src == dst or len(x) == 0:
        return x.copy()
    o, p = reduced_rates(src, dst)
    c = RS_ROLLOFF * min(o, p) / o
    i0b = bessel_i0(RS_BETA)
    out = []
    for n in range(resample_len(len(x), src, dst)):
        tau = n * o / p
        acc = 0.0
        for m in range(len(x)):
            t = (m - tau) * c
            if abs(t) >= RS_WIDTH:
                continue
            r = t / RS_WIDTH
            win = bessel_i0(RS_BETA * math.sqrt(1.0 - r * r)) / i0b
            sinc = 1.0 if t == 0.0 else math.sin(math.pi * t) / (math.pi * t)
            acc += float(x[m]) * c * sinc * win
        out.append(acc)
    return np.asarray(out, np.float32)


def to_mono_16k(channels: list, src: int) -> np.ndarray:
    """``to_mono_16k``: mixdown, then resample to 16 kHz."""
    return resample(mixdown(channels), src, OUT_RATE)
