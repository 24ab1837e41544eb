"""Pins of the second front-end's oracle (``oracle/lfm.py``) to facts outside
it: torch.stft (frame count, centre padding, window placement, power), the
Slaney mel scale's closed forms, the filters' unit area, pre-emphasis of a
constant signal, and the normalisation's moments. The constants themselves
are readings (the page names but does not give them); these pins fix the
structure around them."""
import math

import numpy as np
import pytest

from oracle import lfm as L

torch = pytest.importorskip("torch")


def _torch_power(y, n_fft=512, hop=160, wl=400):
    t = torch.stft(torch.from_numpy(np.asarray(y, np.float64)), n_fft=n_fft, hop_length=hop, win_length=wl,
                   window=torch.hann_window(wl, periodic=True, dtype=torch.float64), center=True,
                   pad_mode="constant", return_complex=True)
    return (t.abs() ** 2).T.numpy()


def _preemph(x, p):
    x = np.asarray(x, np.float32).astype(np.float64)
    y = x.copy()
    y[1:] -= p * x[:-1]
    return y


@pytest.mark.parametrize("n", [1, 159, 160, 161, 400, 16000, 16001, 48123])
def test_frame_count_and_power_match_torch_stft(n):
    x = np.random.default_rng(n).standard_normal(n).astype(np.float32)
    P = L.power_frames(x)
    T = _torch_power(_preemph(x, 0.97))
    assert P.shape == T.shape == (L.num_frames(n), 257)
    assert np.allclose(P, T, rtol=1e-10, atol=1e-10 * P.max())


def test_window_and_hop_parameters_follow_torch():
    x = np.random.default_rng(3).standard_normal(5000).astype(np.float32)
    cfg = dict(n_fft=256, win_length=200, hop=80, preemph=0.5)
    assert np.allclose(L.power_frames(x, cfg), _torch_power(_preemph(x, 0.5), 256, 80, 200), rtol=1e-10, atol=1e-8)


def test_effective_length_counts_frames_centred_in_the_clip():
    assert [L.effective_len(n) for n in (0, 1, 159, 160, 161, 320)] == [0, 1, 1, 1, 2, 2]
    assert [L.num_frames(n) for n in (0, 1, 159, 160, 161, 320)] == [0, 1, 1, 2, 2, 3]
    for n in (1, 160, 161, 16000, 16001):
        eff, nf = L.effective_len(n), L.num_frames(n)
        assert 1 <= eff <= nf and (eff - 1) * 160 < n <= eff * 160


def test_slaney_scale_closed_forms():
    assert L.hz_to_mel_slaney(1000.0) == pytest.approx(15.0, abs=1e-12)
    assert L.hz_to_mel_slaney(6400.0) == pytest.approx(42.0, abs=1e-12)  # one factor of 6.4 = 27 mels
    assert L.hz_to_mel_slaney(300.0) == pytest.approx(4.5, abs=1e-12)     # linear part: 3 f / 200
    f = np.array([0.0, 50.0, 999.0, 1000.0, 1001.0, 4000.0, 8000.0])
    assert np.allclose(L.mel_to_hz_slaney(L.hz_to_mel_slaney(f)), f, rtol=1e-12, atol=1e-9)


def test_filters_have_unit_area_and_peak_at_their_centres():
    M = L.slaney_filterbank(128, 512, 16000)
    df = 16000 / 512
    pts = L.mel_to_hz_slaney(np.linspace(0.0, L.hz_to_mel_slaney(8000.0), 130))
    for b in range(128):
        width = pts[b + 2] - pts[b]
        if width > 8 * df:  # well resolved by the bins: the discrete area is close to the triangle's
            assert abs(M[b].sum() * df - 1.0) < 0.05, b
            assert abs(np.argmax(M[b]) * df - pts[b + 1]) <= df
    assert np.all(M >= 0) and M[:, -1].max() < 1e-12  # the last triangle ends exactly at Nyquist


def test_preemphasis_of_a_constant_scales_dc_power():
    x = np.full(16000, 0.25, np.float32)
    P0 = L.power_frames(x, dict(preemph=0.0))
    P = L.power_frames(x, dict(preemph=0.97))
    mid = slice(5, 90)  # frames away from both edges
    assert np.allclose(P[mid, 0], P0[mid, 0] * (1 - 0.97) ** 2, rtol=1e-9)


def test_normalisation_moments_and_zero_tail():
    x = (0.1 * np.random.default_rng(7).standard_normal(16000 * 3 + 77)).astype(np.float32)
    F = L.features(x)
    eff, nf = L.effective_len(len(x)), L.num_frames(len(x))
    assert F.shape == (nf, 128) and nf == eff  # the length is not a multiple of the hop
    assert np.all(F[eff:] == 0.0)
    lm = L.log_mel(x)[:eff]
    var = lm.var(axis=0)
    assert np.allclose(F[:eff].mean(axis=0), 0.0, atol=1e-9)
    assert np.allclose(F[:eff].var(axis=0), var / (var + 1e-5), rtol=1e-9)


def test_tone_lands_in_its_band():
    sr = 16000
    x = (0.3 * np.sin(2 * np.pi * 1000.0 * np.arange(sr) / sr)).astype(np.float32)
    lm = L.log_mel(x, dict(preemph=0.0))
    pts = L.mel_to_hz_slaney(np.linspace(0.0, L.hz_to_mel_slaney(8000.0), 130))
    want = int(np.argmin(np.abs(pts[1:-1] - 1000.0)))
    assert abs(int(np.argmax(lm[50])) - want) <= 1


def test_features_do_not_depend_on_the_input_scale():
    """Above the log floor, scaling the clip by a adds 2 ln a to every log-mel
    value, which the per-band normalisation removes. Scaling up keeps every band
    above the floor (scaling down can push the weakest, pre-emphasised low bands
    onto it, where the clamp breaks the identity)."""
    x = (0.1 * np.random.default_rng(9).standard_normal(16000 * 2)).astype(np.float32)
    F = L.features(x)
    for a in (2.0, 4.0, 64.0):
        G = L.features((a * x).astype(np.float32))
        assert np.max(np.abs(G - F)) < 1e-6
        assert np.allclose(L.log_mel((a * x).astype(np.float32)), L.log_mel(x) + 2 * math.log(a), atol=1e-5)
