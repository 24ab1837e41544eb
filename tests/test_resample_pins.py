"""Pins of the resampler oracle (``oracle/resample.py``) to facts that do not
come from the oracle itself: the page's own resampler tests (egemma2_audio.rs,
``stereo_mixes_down_and_rates_resample`` and
``resampling_keeps_a_tone_and_its_length``: exact lengths, tones within 1e-4
of the ideal, a tone above the new Nyquist removed), the half-amplitude point
of a windowed-sinc low-pass at its cut-off, the transition band predicted by
the Kaiser window's analytic Fourier transform, numpy's Bessel I0, and a
brute-force double loop on tiny inputs."""
import math

import numpy as np
import pytest

from oracle import resample as R


def _tone(rate, f0, n):
    return np.sin(2 * np.pi * f0 * np.arange(n) / rate).astype(np.float32)


def _amplitude(y, f0, lo, hi, rate=16000):
    seg = np.asarray(y[lo:hi], np.float64)
    t = np.arange(lo, hi) / rate
    a = 2 * np.mean(seg * np.sin(2 * np.pi * f0 * t))
    b = 2 * np.mean(seg * np.cos(2 * np.pi * f0 * t))
    return math.hypot(a, b)


def test_bessel_i0_series_matches_numpy():
    for x in (0.0, 0.5, 1.0, 5.0, 12.8, 20.0, 30.0):
        assert R.bessel_i0(x) == pytest.approx(float(np.i0(x)), rel=1e-14)
    xs = np.linspace(0, 12.8, 57)
    assert np.allclose(R.bessel_i0_array(xs), np.i0(xs), rtol=1e-14, atol=0)


def test_lengths_as_on_the_page():
    for rate in (8000, 44100, 48000, 22050, 44099):
        assert R.resample_len(rate, rate, rate) == rate  # equal rates: unchanged
        assert R.resample_len(rate, rate, 16000) == 16000  # one second
    assert R.resample_len(4800, 48000) == 1600
    assert R.resample_len(0, 48000) == 0
    assert R.resample_len(16001, 16000) == 16001
    # ceil, not floor: 3 samples at 48 kHz are one 16 kHz sample, 4 are two
    assert R.resample_len(3, 48000) == 1 and R.resample_len(4, 48000) == 2
    assert R.resample_len(1, 44100) == 1


@pytest.mark.parametrize("rate,f0", [(8000, 1000.0), (44100, 3000.0), (48000, 7000.0), (22050, 440.0)])
def test_a_tone_comes_out_as_the_ideal_one(rate, f0):
    y = R.resample(_tone(rate, f0, rate), rate)
    assert len(y) == 16000
    want = np.sin(2 * np.pi * f0 * np.arange(16000) / 16000.0)
    assert np.max(np.abs(y[2000:14000] - want[2000:14000])) < 1e-4


def test_a_tone_above_the_new_nyquist_is_removed():
    y = R.resample(_tone(48000, 9000.0, 48000), 48000)
    assert math.sqrt(np.mean(y[2000:14000].astype(np.float64) ** 2)) < 1e-4


def test_stereo_mixdown_and_dc_level():
    assert R.to_mono_16k([[1.0, 0.0, 0.5], [0.0, 1.0, 0.5]], 16000).tolist() == [0.5, 0.5, 0.5]
    m = R.to_mono_16k([np.full(4800, 0.25, np.float32)], 48000)
    assert len(m) == 1600 and abs(m[800] - 0.25) < 1e-4
    # the mixdown is a float32 sum in channel order, then a float32 division
    a = np.float32(0.1)
    b = np.float32(0.2)
    c = np.float32(0.3)
    assert R.mixdown([[a], [b], [c]])[0] == np.float32((np.float32(a + b) + c) / np.float32(3))


def _kaiser_ft(u, T, beta):
    """Fourier transform of I0(beta sqrt(1 - (t/T)^2)) / I0(beta) on |t| <= T."""
    a = 2 * math.pi * u * T
    s = beta * beta - a * a
    if s > 0:
        r = math.sqrt(s)
        v = math.sinh(r) / r
    elif s < 0:
        r = math.sqrt(-s)
        v = math.sin(r) / r
    else:
        v = 1.0
    return 2 * T / float(np.i0(beta)) * v


def _windowed_sinc_response(f, c, width=64.0, beta=12.8):
    """Gain at f (cycles per input sample) of c sinc(c t) w(t): the box of
    width c convolved with the window's transform."""
    from scipy import integrate
    T = width / c
    edge = beta / (2 * math.pi * T)
    val, _ = integrate.quad(lambda u: _kaiser_ft(u, T, beta), f - c / 2, f + c / 2, limit=400,
                            points=[-edge, edge])
    return val


@pytest.mark.parametrize("rate", [48000, 44100])
def test_cutoff_and_transition_band_follow_the_kaiser_window(rate):
    """0.958 of the lower Nyquist is the half-amplitude point, and 3 % either
    side of it the gain is what the Kaiser window (beta 12.8, 64 zero
    crossings) predicts; a different beta, width or roll-off moves these by
    more than 1e-2."""
    c = 0.958 * 16000 / rate  # the page's RS_ROLLOFF, written out: the pin must not follow the oracle's constant
    fc = 0.958 * 8000
    n = 2 * rate
    for f0 in (fc, 0.97 * fc, 1.03 * fc):
        y = R.resample(_tone(rate, f0, n), rate)
        want = _windowed_sinc_response(f0 / rate, c)
        assert abs(_amplitude(y, f0, 4000, 28000) - want) < 2e-4, f0
    assert abs(_amplitude(R.resample(_tone(rate, fc, n), rate), fc, 4000, 28000) - 0.5) < 1e-4


@pytest.mark.parametrize("rate", [48000, 44100, 8000, 22050])
def test_phase_grouping_equals_the_direct_double_loop(rate):
    x = np.random.default_rng(rate).standard_normal(300).astype(np.float32)
    a = R.resample(x, rate)
    b = R.resample_direct(x, rate)
    assert len(a) == len(b) == R.resample_len(300, rate)
    assert np.max(np.abs(a.astype(np.float64) - b)) <= 1e-6


def test_coprime_rate_and_equal_rate():
    x = ((np.arange(44099) % 97) / 97.0 - 0.5).astype(np.float32)
    y = R.resample(x, 44099)
    assert len(y) == 16000 and np.all(np.isfinite(y))
    z = np.arange(10, dtype=np.float32)
    assert np.array_equal(R.resample(z, 16000), z)
    assert len(R.resample(np.zeros(0, np.float32), 48000)) == 0


def test_linear_and_shift_equivariant():
    """The definition is a linear, shift-invariant filter evaluated on a
    lattice: resampling a x + b y gives a R(x) + b R(y), and delaying the input
    by o samples (one lattice period) delays the output by p samples."""
    rng = np.random.default_rng(12)
    for rate in (48000, 44100):
        o, p = R.reduced_rates(rate, 16000)
        n = 3000 + 7 * o
        x = rng.standard_normal(n).astype(np.float32)
        y = rng.standard_normal(n).astype(np.float32)
        lin = R.resample((2 * x - 3 * y).astype(np.float32), rate).astype(np.float64)
        assert np.max(np.abs(lin - (2 * R.resample(x, rate).astype(np.float64)
                                    - 3 * R.resample(y, rate).astype(np.float64)))) < 1e-5
        xs = np.concatenate([np.zeros(o, np.float32), x])
        a = R.resample(x, rate)
        b = R.resample(xs, rate)
        assert np.array_equal(b[p:p + len(a)], a) or np.max(np.abs(b[p:p + len(a)] - a)) < 1e-6


# Every rate the GPU parity tests resample from (``tests/test_gpu_resample.py``).
GPU_TEST_RATES = (8000, 44100, 48000, 22050, 96000, 11025, 32000, 24000, 44099, 10500, 15750, 12600, 5125, 432000,
                  448000, 1000000)


def test_tap_sums_stay_below_the_parity_bound():
    """The GPU parity bound (L / 2 + 2) 2^-24 x 2.7 x max |input| takes 2.7 for
    the absolute sum of one output's taps. Evaluated here from the page's
    definition (numpy's I0, every phase of every rate the GPU tests use), the
    largest sum is about 2.66 (upsampling) and 2.37 to 2.43 otherwise."""
    for rate in GPU_TEST_RATES:
        g = math.gcd(rate, 16000)
        o, p = rate // g, 16000 // g
        c = 0.958 * min(o, p) / o
        half = 64.0 / c
        worst = 0.0
        for j in range(p):
            frac = o * j / p
            d = np.arange(math.floor(frac - half), math.ceil(frac + half) + 1)
            t = (d - frac) * c
            t = t[np.abs(t) < 64.0]
            win = np.i0(12.8 * np.sqrt(1.0 - (t / 64.0) ** 2)) / np.i0(12.8)
            worst = max(worst, float(np.sum(np.abs(np.sinc(t) * win * c))))
        assert 2.0 < worst <= 2.7, (rate, worst)
