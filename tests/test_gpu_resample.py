"""Parity of the library's mixdown and resampler (``ae_resample``, through
the C ABI) with the float64 oracle (``oracle/resample.py``), element by
element, within the bound the arithmetic gives: float32 taps applied with
float32 accumulation in two interleaved partial sums over L taps, error
below (L / 2 + 2) 2^-24 x 2.7 x max |input|, 2.7 bounding the taps' absolute
sum (computed from the definition for every rate used here, in
``test_resample_pins.py``). The tensor-core form (bf16-split inputs and taps,
four products, float32 accumulation) is held to the same bound."""
import math

import numpy as np
import pytest

from oracle import resample as R
from tests.helpers import dev, offsets, workspace

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import log_mel_front_b200 as ae  # noqa: E402


def _bound(rate_in, rate_out=16000):
    o, p = R.reduced_rates(rate_in, rate_out)
    c = R.RS_ROLLOFF * min(o, p) / o
    L = 2 * math.ceil(R.RS_WIDTH / c) + 3
    return (L / 2 + 2) * 2.0 ** -24 * 2.7


def gpu_resample(channels_per_clip, rate_in, rate_out=16000):
    """channels_per_clip: list of clips, each a list of C equal-length arrays."""
    C = len(channels_per_clip[0]) if channels_per_clip else 1
    lens = [len(clip[0]) for clip in channels_per_clip]
    off = offsets(lens)
    total = int(off[-1])
    planes = np.zeros((C, max(total, 1)), np.float32)
    for k, clip in enumerate(channels_per_clip):
        for ch in range(C):
            planes[ch, off[k]:off[k + 1]] = clip[ch]
    outs = [ae.ae_resample_len(n, rate_in, rate_out) for n in lens]
    d_x = dev(planes)
    d_y = torch.full((max(sum(outs), 1),), float("nan"), device="cuda")
    nb = ae.ae_resample_workspace_size(off, rate_in, rate_out, C)
    ws = workspace(nb)
    ae.ae_resample(d_x, C, planes.shape[1], off, rate_in, rate_out, d_y, ws, ws.numel())
    torch.cuda.synchronize()
    assert ae.ae_device_status() == ae.AE_OK
    y = d_y[:sum(outs)].cpu().numpy()
    o = offsets(outs)
    return [y[o[k]:o[k + 1]] for k in range(len(lens))]


def _check(got, want, x_max, rate_in, what):
    assert got.shape == want.shape, what
    err = float(np.max(np.abs(got.astype(np.float64) - want.astype(np.float64)))) if got.size else 0.0
    bound = _bound(rate_in) * max(x_max, 1e-30)
    print(f"[parity] {what}: max abs err {err:.3e} (bound {bound:.3e})")
    assert err <= bound, what


@pytest.mark.parametrize("rate,f0", [(8000, 1000.0), (44100, 3000.0), (48000, 7000.0), (22050, 440.0)])
def test_tones_as_on_the_page(rate, f0):
    x = np.sin(2 * np.pi * f0 * np.arange(rate) / rate).astype(np.float32)
    (y,) = gpu_resample([[x]], rate)
    assert len(y) == 16000
    want = np.sin(2 * np.pi * f0 * np.arange(16000) / 16000.0)
    assert np.max(np.abs(y[2000:14000] - want[2000:14000])) < 1e-4
    _check(y, R.resample(x, rate), 1.0, rate, f"tone {f0} Hz from {rate}")


def test_alias_removed_and_stereo_mixdown():
    x = np.sin(2 * np.pi * 9000.0 * np.arange(48000) / 48000).astype(np.float32)
    (y,) = gpu_resample([[x]], 48000)
    assert math.sqrt(np.mean(y[2000:14000].astype(np.float64) ** 2)) < 1e-4
    (m,) = gpu_resample([[np.array([1.0, 0.0, 0.5], np.float32), np.array([0.0, 1.0, 0.5], np.float32)]], 16000)
    assert m.tolist() == [0.5, 0.5, 0.5]
    (m,) = gpu_resample([[np.full(4800, 0.25, np.float32)]], 48000)
    assert len(m) == 1600 and abs(m[800] - 0.25) < 1e-4


def test_ragged_stereo_batch_at_44k1():
    rng = np.random.default_rng(44)
    lens = [0, 1, 2, 441, 1000, 44100, 100003]
    clips = [[(0.5 * rng.standard_normal(n)).astype(np.float32) for _ in range(2)] for n in lens]
    got = gpu_resample(clips, 44100)
    for k, clip in enumerate(clips):
        mono = R.mixdown(clip)
        want = R.resample(mono, 44100)
        xm = float(np.max(np.abs(mono))) if len(mono) else 0.0
        _check(got[k], want, xm, 44100, f"stereo 44.1 kHz clip of {lens[k]} samples")


@pytest.mark.parametrize("rate", [96000, 11025, 32000, 24000])
def test_other_rates(rate):
    rng = np.random.default_rng(rate)
    clips = [[rng.uniform(-1, 1, n).astype(np.float32)] for n in (rate // 3, 777)]
    got = gpu_resample(clips, rate)
    for k, clip in enumerate(clips):
        _check(got[k], R.resample(clip[0], rate), float(np.max(np.abs(clip[0]))), rate, f"{rate} Hz clip {k}")


# Each tile width the tensor-core form takes besides 16 and 160 (a row of
# N = 32, 64, 80 and 128 outputs), its longest window (432 kHz: 4032 inputs
# per row, the most it takes being 4096), and the per-tile FIR for the rates
# past that window (448 kHz, taps staged in shared memory; 1 MHz, the highest
# rate taken, taps read from global memory), each over several tiles and a
# ragged tail, beside a short clip.
TILE_EDGE_RATES = {10500: 10513, 15750: 15763, 12600: 12613, 5125: 15388, 432000: 108000, 448000: 112000,
                   1000000: 60000}


@pytest.mark.parametrize("rate", sorted(TILE_EDGE_RATES))
def test_every_tile_width_and_the_widest_windows(rate):
    rng = np.random.default_rng(rate + 1)
    clips = [[rng.uniform(-1, 1, n).astype(np.float32)] for n in (TILE_EDGE_RATES[rate], 777)]
    got = gpu_resample(clips, rate)
    for k, clip in enumerate(clips):
        _check(got[k], R.resample(clip[0], rate), float(np.max(np.abs(clip[0]))), rate, f"{rate} Hz clip {k}")


def test_coprime_rate_reads_global_memory():
    x = ((np.arange(44099) % 97) / 97.0 - 0.5).astype(np.float32)
    (y,) = gpu_resample([[x]], 44099)
    assert len(y) == 16000
    _check(y, R.resample(x, 44099), 0.5, 44099, "co-prime 44099 Hz")


def test_three_channels_mix_in_order():
    rng = np.random.default_rng(3)
    chans = [rng.standard_normal(5000).astype(np.float32) for _ in range(3)]
    (y,) = gpu_resample([chans], 48000)
    mono = R.mixdown(chans)
    _check(y, R.resample(mono, 48000), float(np.max(np.abs(mono))), 48000, "three channels from 48 kHz")
    (same,) = gpu_resample([chans], 16000)
    assert np.array_equal(same, mono)


def test_refusals_enqueue_nothing():
    off = np.array([0, 100], np.int64)
    x = torch.zeros(100, device="cuda")
    y = torch.zeros(100, device="cuda")
    ws = workspace(1 << 20)
    for args, st in [((x, 1, 100, off, 0, 16000), ae.AE_EINVAL), ((x, 0, 100, off, 48000, 16000), ae.AE_EINVAL),
                     ((x, 2, 50, off, 48000, 16000), ae.AE_EINVAL),
                     ((x, 1, 100, off, 999983, 999979), ae.AE_EUNSUPPORTED)]:
        with pytest.raises(ae.AEError) as e:
            ae.ae_resample(*args, y, ws, ws.numel())
        assert e.value.status == st
    with pytest.raises(ae.AEError) as e:
        ae.ae_resample(x, 1, 100, off, 48000, 16000, y, ws, 64)
    assert e.value.status == ae.AE_EWORKSPACE
    torch.cuda.synchronize()
