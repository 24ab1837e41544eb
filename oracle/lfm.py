"""Plain float64 CPU oracle of the second log-mel front-end: the LFM2A audio
encoder's, as the docs.rs page of its GPU port describes it
(``log_mel_spectrogram_gpu`` and the ``AudioEncoderGpuOps`` stages
``stft_frames``, ``power_spec``, ``mel_project``, ``mel_norm``; the
``GpuMelFrontend`` tables).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: the parity tests and
``bench.py``'s CPU legs call it; the CUDA library never does, and nothing here
is shared with it.

What the page fixes: frames of ``n_fft`` samples every ``hop`` samples with
``n_fft / 2`` samples of centre padding per side; pre-emphasis; a periodic
Hann window of the window length centred in an ``n_fft``-wide buffer of
zeros; the power spectrum |X_k|^2 for k = 0 .. n_fft / 2; a Slaney mel
filterbank; the natural log with a floor; per-mel-bin normalisation whose
statistics come from the first ``effective_n_len`` frames, the others set to
zero; output [frames, n_mel], time-major.

What the page leaves open, and the readings taken here (all parameters, with
these defaults):

* the constants: sample rate 16 kHz, n_fft 512, window 400, hop 160, 128
  bands, pre-emphasis 0.97, log floor 2^-24, variance epsilon 1e-5;
* padding is zeros (librosa's constant centre padding); pre-emphasis runs on
  the clip before padding, y[n] = x[n] - p x[n-1] with x[-1] = 0;
* frames: n_frames = 1 + N // hop for N > 0 samples (one frame per hop, as
  centre-padded STFTs count them), 0 for N = 0;
* effective_n_len = ceil(N / hop): the frames whose centre sample lies inside
  the clip;
* the floor is a lower clamp: ln(max(mel, floor));
* normalisation: (v - mean) / sqrt(var + eps) per band, mean and the biased
  variance over the effective frames;
* Slaney filterbank as librosa builds it by default (htk=False,
  norm="slaney"): mel points evenly spaced between mel(0) and mel(sr / 2) on
  the Slaney scale (linear 3 f / 200 below 1 kHz, 15 + 27 ln(f / 1000) /
  ln 6.4 above), triangles over the FFT bin frequencies k sr / n_fft, each
  scaled by 2 / (f_{b+2} - f_b).

Parity status: partly unpinned. The structure is pinned (torch.stft for
framing, padding, window and power; the Slaney scale's closed forms; the
filters' unit area; the normalisation's moments); the constants are
readings, not the page's.
"""
from __future__ import annotations

import math

import numpy as np

DEFAULTS = dict(sample_rate=16000, n_fft=512, win_length=400, hop=160, n_mels=128, preemph=0.97,
                log_floor=2.0 ** -24, var_eps=1e-5)


def num_frames(n: int, hop: int = 160) -> int:
    """1 + N // hop frames for N > 0 samples, none for an empty clip."""
    return 1 + n // hop if n > 0 else 0


def effective_len(n: int, hop: int = 160) -> int:
    """Frames whose centre sample (f hop, with n_fft / 2 of padding) lies in the clip."""
    return -(-n // hop) if n > 0 else 0


def hz_to_mel_slaney(f):
    """Slaney's scale: 3 f / 200 below 1 kHz, 15 + 27 ln(f / 1000) / ln 6.4 above."""
    f = np.asarray(f, np.float64)
    lin = 3.0 * f / 200.0
    log = 15.0 + 27.0 * np.log(np.maximum(f, 1e-300) / 1000.0) / math.log(6.4)
    return np.where(f >= 1000.0, log, lin)


def mel_to_hz_slaney(m):
    m = np.asarray(m, np.float64)
    lin = 200.0 * m / 3.0
    log = 1000.0 * np.exp((m - 15.0) * math.log(6.4) / 27.0)
    return np.where(m >= 15.0, log, lin)


def slaney_filterbank(n_mels: int = 128, n_fft: int = 512, sr: int = 16000) -> np.ndarray:
    """[n_mels, n_fft / 2 + 1] triangles on the Slaney scale, area-normalised."""
    pts = mel_to_hz_slaney(np.linspace(hz_to_mel_slaney(0.0), hz_to_mel_slaney(sr / 2.0), n_mels + 2))
    fk = np.arange(n_fft // 2 + 1) * sr / n_fft
    bank = np.zeros((n_mels, n_fft // 2 + 1))
    for b in range(n_mels):
        lower = (fk - pts[b]) / (pts[b + 1] - pts[b])
        upper = (pts[b + 2] - fk) / (pts[b + 2] - pts[b + 1])
        bank[b] = np.maximum(0.0, np.minimum(lower, upper)) * (2.0 / (pts[b + 2] - pts[b]))
    return bank


def padded_hann(win_length: int = 400, n_fft: int = 512) -> np.ndarray:
    """Periodic Hann of win_length centred in an n_fft-wide buffer of zeros."""
    w = 0.5 - 0.5 * np.cos(2.0 * np.pi * np.arange(win_length) / win_length)
    out = np.zeros(n_fft)
    lo = (n_fft - win_length) // 2
    out[lo:lo + win_length] = w
    return out


def power_frames(wave, cfg: dict | None = None) -> np.ndarray:
    """[n_frames, n_fft / 2 + 1] power spectra of the pre-emphasised,
    centre-padded, windowed frames."""
    c = dict(DEFAULTS, **(cfg or {}))
    x = np.asarray(wave, np.float32).astype(np.float64)
    n, hop, n_fft = len(x), c["hop"], c["n_fft"]
    nf = num_frames(n, hop)
    if nf == 0:
        return np.zeros((0, n_fft // 2 + 1))
    y = x.copy()
    y[1:] -= c["preemph"] * x[:-1]
    pad = np.concatenate([np.zeros(n_fft // 2), y, np.zeros(n_fft // 2 + n_fft)])
    idx = np.arange(nf)[:, None] * hop + np.arange(n_fft)[None, :]
    frames = pad[idx] * padded_hann(c["win_length"], n_fft)[None, :]
    X = np.fft.rfft(frames, axis=1)
    return X.real ** 2 + X.imag ** 2


def log_mel(wave, cfg: dict | None = None) -> np.ndarray:
    """Un-normalised log-mel [n_frames, n_mels]: ln(max(P M^T, floor))."""
    c = dict(DEFAULTS, **(cfg or {}))
    P = power_frames(wave, c)
    M = slaney_filterbank(c["n_mels"], c["n_fft"], c["sample_rate"])
    return np.log(np.maximum(P @ M.T, c["log_floor"]))


def normalise(lm: np.ndarray, eff: int, var_eps: float) -> np.ndarray:
    """Per band: (v - mean) / sqrt(var + eps) over the first eff frames
    (biased variance); frames from eff on are zero."""
    out = np.zeros_like(lm)
    if eff <= 0:
        return out
    v = lm[:eff]
    mean = v.mean(axis=0)
    var = ((v - mean) ** 2).mean(axis=0)
    out[:eff] = (v - mean) / np.sqrt(var + var_eps)
    return out


def features(wave, cfg: dict | None = None) -> np.ndarray:
    """The front-end's output for one clip: [n_frames, n_mels], time-major."""
    c = dict(DEFAULTS, **(cfg or {}))
    lm = log_mel(wave, c)
    return normalise(lm, effective_len(len(wave), c["hop"]), c["var_eps"])
