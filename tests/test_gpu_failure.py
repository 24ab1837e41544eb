"""Failure detection on the GPU without a fault. Every wait in the library's
kernels is bounded; a kernel that gives one up records it in the library's
status word and leaves, and ae_device_status reports it (AE_EDEVICE) and
clears it. ae_selftest_bounded_wait runs that same bounded wait on a barrier
that nothing completes, with a short limit, so the path is exercised without
hanging or faulting anything; afterwards the context must still compute."""
import numpy as np
import pytest

import synth
from oracle import oracle as O
from tests.helpers import assert_logmel, dev, workspace

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import log_mel_front_b200 as ae  # noqa: E402


def test_wait_that_nothing_completes_is_reported_once():
    torch.cuda.synchronize()
    assert ae.ae_device_status() == ae.AE_OK
    ae.ae_selftest_bounded_wait(2000)  # gives up after 2 ms
    assert ae.ae_device_status() == ae.AE_EDEVICE
    assert ae.ae_device_status() == ae.AE_OK  # reported once, then cleared


def test_completed_wait_reports_nothing():
    ae.ae_selftest_bounded_wait(1000000, arrive=True)
    assert ae.ae_device_status() == ae.AE_OK


def test_context_still_computes_after_a_timeout():
    ae.ae_selftest_bounded_wait(1000)
    assert ae.ae_device_status() == ae.AE_EDEVICE
    clip = synth.pr1_wave()
    flat, off = synth.pack([clip])
    frames = O.num_frames(len(clip))
    d_mel = torch.full((frames, 128), float("nan"), device="cuda")
    ws = workspace(ae.ae_workspace_size(None, 1, frames, 0))
    ae.ae_logmel(dev(flat), off, d_mel, ws, ws.numel())
    torch.cuda.synchronize()
    assert ae.ae_device_status() == ae.AE_OK
    assert_logmel(d_mel.cpu().numpy(), O.log_mel(clip), "log-mel after a reported timeout")
