"""CPU oracle of the gemma4_audio encoder forward.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.
"""
from .oracle import *  # noqa: F401,F403
