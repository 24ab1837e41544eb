"""B200 (sm_100a) audio-encoder forward: 16 kHz waveform -> log-mel -> stem ->
Conformer layers -> 512-d embedding rows, behind the C ABI of include/ae.h.

The first use of any name of this package loads libae.so and raises
ImportError if it has not been built (``python -m log_mel_front_b200.build``):
there is no other implementation to fall back to. Importing the package
alone (for instance to run the build module) does not load the library.
"""
import importlib

__version__ = "0.1.0"


def __getattr__(name):
    if name.startswith("__"):
        raise AttributeError(name)
    if name in ("abi", "build", "gen_htk_bank"):
        return importlib.import_module(f"{__name__}.{name}")
    abi = importlib.import_module(f"{__name__}.abi")  # loads libae.so; ImportError if it is missing
    return getattr(abi, name)
