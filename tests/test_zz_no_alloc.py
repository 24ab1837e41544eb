"""ae_logmel_noalloc: the log-mel front-end for callers that cannot allocate
device memory (a real-time audio callback, a host whose device memory all
belongs to its own pool allocator, a plugin handed only its buffers). It
keeps its clip tables in a fixed array inside the library instead of a
caller workspace; its output must match ae_logmel's.

Collected last (file name) so that a run stopping at the first failure has
already run every other test.
"""
import numpy as np
import pytest

import synth
from tests.helpers import LOGMEL_ABS, dev, workspace

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import log_mel_front_b200 as ae  # noqa: E402


def _frames(clips):
    return sum(ae.ae_num_frames(len(c)) for c in clips)


def _with_workspace(clips):
    flat, off = synth.pack(clips)
    F = _frames(clips)
    out = torch.full((F, 128), float("nan"), device="cuda")
    ws = workspace(ae.ae_workspace_size(None, len(clips), F, 0))
    ae.ae_logmel(dev(flat), off, out, ws, ws.numel())
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _without_workspace(clips):
    flat, off = synth.pack(clips)
    F = _frames(clips)
    out = torch.full((F, 128), float("nan"), device="cuda")
    ae.ae_logmel_noalloc(dev(flat), off, out)
    torch.cuda.synchronize()
    assert ae.ae_device_status() == ae.AE_OK
    return out.cpu().numpy()


def test_noalloc_matches_logmel_on_two_calls_in_a_row():
    rng = np.random.default_rng(2024)
    # first call: a ragged batch; second call: fewer, longer clips, so stale
    # table entries from the first call would show up as wrong rows
    first = [(0.3 * rng.standard_normal(n)).astype(np.float32) for n in (16000, 161, 72825, 321, 480001, 1000)]
    second = synth.waves("frontend", [0, 5, 9])
    for clips in (first, second):
        want = _with_workspace(clips)
        got = _without_workspace(clips)
        assert got.shape == want.shape == (_frames(clips), 128)
        assert np.all(np.isfinite(got))
        err = float(np.max(np.abs(got - want)))
        print(f"[parity] ae_logmel_noalloc vs ae_logmel: max abs diff {err:.3e} (bound {LOGMEL_ABS})")
        assert err <= LOGMEL_ABS


def test_noalloc_refuses_too_many_clips():
    off = np.arange(4002, dtype=np.int64) * 16000
    with pytest.raises(ae.AEError) as e:
        ae.ae_logmel_noalloc(0, off, 0)
    assert e.value.status == ae.AE_EINVAL and "at most 4000 clips" in str(e.value)


def test_noalloc_at_the_clip_limit():
    """4000 clips, the most one call takes: the clip tables come closest to
    filling the fixed array here. Short clips of 161 to 400 samples (one or two
    frames each) keep the call small; its rows must equal ae_logmel's."""
    rng = np.random.default_rng(4000)
    lens = rng.integers(161, 401, size=4000)
    clips = [(0.3 * rng.standard_normal(int(n))).astype(np.float32) for n in lens]
    want = _with_workspace(clips)
    got = _without_workspace(clips)
    assert got.shape == want.shape == (_frames(clips), 128)
    assert np.all(np.isfinite(got))
    err = float(np.max(np.abs(got - want)))
    print(f"[parity] ae_logmel_noalloc at 4000 clips vs ae_logmel: max abs diff {err:.3e} (bound {LOGMEL_ABS})")
    assert err <= LOGMEL_ABS
