"""Parity of the second log-mel front-end (``ae_lfm_logmel``, the LFM2A
encoder's) with the float64 oracle (``oracle/lfm.py``), element by element
on the normalised output. Tolerance: max |gpu - oracle| <= 2e-3. The GPU
computes the spectrum in float32 (four-step FFT, float32 twiddles and
window): the error of a power bin is about 1e-6 of the frame's largest bin,
which is a relative error of up to ~1e-3 on the weakest bands of these
signals (the pre-emphasis takes the low bands down by (1 - 0.97)^2), and the
normalisation divides by the band's standard deviation over the clip."""
import numpy as np
import pytest

import synth
from oracle import lfm as L
from tests.helpers import dev, offsets, workspace

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import log_mel_front_b200 as ae  # noqa: E402

TOL = 2e-3


def gpu_lfm(clips, cfg=None, **kw):
    cfg = cfg or ae.lfm_config(**kw)
    flat, off = synth.pack(clips)
    frames = sum(ae.ae_lfm_num_frames(cfg, len(c)) for c in clips)
    d_out = torch.full((max(frames, 1), cfg.n_mels), float("nan"), device="cuda")
    ws = workspace(ae.ae_lfm_workspace_size(cfg, len(clips)))
    ae.ae_lfm_logmel(cfg, dev(flat if len(flat) else np.zeros(1, np.float32)), off, d_out, ws, ws.numel())
    torch.cuda.synchronize()
    assert ae.ae_device_status() == ae.AE_OK
    g = d_out[:frames].cpu().numpy()
    o = offsets([ae.ae_lfm_num_frames(cfg, len(c)) for c in clips])
    return [g[o[i]:o[i + 1]] for i in range(len(clips))]


def _check(g, o, what):
    assert g.shape == o.shape, what
    err = float(np.max(np.abs(g.astype(np.float64) - o))) if o.size else 0.0
    print(f"[parity] {what}: max abs err {err:.3e} (bound {TOL})")
    assert err <= TOL, what


def test_ragged_edge_lengths():
    lens = [0, 1, 159, 160, 161, 400, 16000, 16001, 48123]
    clips = [synth.noise_tones_clip(n, 50, i) for i, n in enumerate(lens)]
    got = gpu_lfm(clips)
    for n, c, g in zip(lens, clips, got):
        _check(g, L.features(c), f"clip of {n} samples")


def test_frontend_workload_full_size_sampled():
    clips = synth.waves("frontend")
    got = gpu_lfm(clips)
    assert sum(len(g) for g in got) == 64 * L.num_frames(480000)
    for i in (0, 31, 63):
        _check(got[i], L.features(clips[i]), f"frontend workload clip {i}")


def test_other_configuration():
    cfg = dict(n_mels=80, win_length=320, hop=100, preemph=0.5, var_eps=1e-3, log_floor=1e-10)
    clips = [synth.noise_tones_clip(n, 51, i) for i, n in enumerate([12345, 999, 100])]
    got = gpu_lfm(clips, **cfg)
    for c, g in zip(clips, got):
        _check(g, L.features(c, cfg), f"{len(c)} samples, n_mels 80, window 320, hop 100")


def test_silence_and_zero_tail():
    got = gpu_lfm([np.zeros(16000, np.float32), synth.noise_tones_clip(32000, 52, 0)])
    assert np.all(got[0] == 0.0)  # constant log floor: zero variance, normalised to 0
    eff = L.effective_len(32000)
    assert eff == 200 and got[1].shape[0] == 201 and np.all(got[1][eff:] == 0.0)


def test_wave_not_16_byte_aligned():
    """With a waveform base 4 bytes off a 16-byte boundary the spectrum kernel
    stages its samples 4 bytes at a time instead of 16: the same rows."""
    clips = [synth.noise_tones_clip(n, 53, i) for i, n in enumerate([16000, 7777, 48123, 161])]
    flat, off = synth.pack(clips)
    cfg = ae.lfm_config()
    frames = sum(ae.ae_lfm_num_frames(cfg, len(c)) for c in clips)
    nb = ae.ae_lfm_workspace_size(cfg, len(clips))
    outs = []
    for shift in (0, 1):
        base = torch.zeros(len(flat) + 8, device="cuda")
        base[shift:shift + len(flat)] = dev(flat)
        d_out = torch.full((frames, cfg.n_mels), float("nan"), device="cuda")
        ws = workspace(nb)
        ae.ae_lfm_logmel(cfg, base[shift:shift + len(flat)], off, d_out, ws, ws.numel())
        torch.cuda.synchronize()
        assert ae.ae_device_status() == ae.AE_OK
        outs.append(d_out.cpu().numpy())
    assert np.array_equal(outs[0], outs[1])
    o = offsets([ae.ae_lfm_num_frames(cfg, len(c)) for c in clips])
    _check(outs[1][o[2]:o[3]], L.features(clips[2]), "48123 samples from an unaligned base")
