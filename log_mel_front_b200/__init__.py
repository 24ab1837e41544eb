"""B200 (sm_100a) audio-encoder forward: 16 kHz waveform -> log-mel -> stem ->
Conformer layers -> 512-d embedding rows, behind the C ABI of include/ae.h.

Importing this package loads libae.so and raises ImportError if it has not
been built (``python -m log_mel_front_b200.build``): there is no other
implementation to fall back to.
"""
from .abi import *  # noqa: F401,F403
from .abi import EXPORTS, LIB_PATH, Model, lib  # noqa: F401

__version__ = "0.1.0"
