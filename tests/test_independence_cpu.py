"""The oracle and the CUDA path are independent: no module of ``oracle/``
imports the package or reads its sources, no file of the package (Python,
CUDA, headers) refers to ``oracle``, the seeded-input module imports neither,
and only the tests, ``__graft_entry__.py`` and ``bench.py`` import the
oracle."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _files(sub, exts):
    out = []
    for d, _, fs in os.walk(os.path.join(ROOT, sub)):
        if "__pycache__" in d:
            continue
        out += [os.path.join(d, f) for f in fs if f.endswith(exts)]
    return out


def test_oracle_does_not_touch_the_package():
    for p in _files("oracle", (".py", ".c", ".h")):
        src = open(p).read()
        assert "log_mel_front_b200" not in src and "csrc" not in src and "libae" not in src, p


def test_package_does_not_touch_the_oracle():
    for p in _files("log_mel_front_b200", (".py", ".cu", ".cuh", ".h", ".cpp")) + _files("include", (".h",)):
        src = open(p).read()
        assert not re.search(r"\boracle\b", src), p


def test_input_generators_hold_no_method_code():
    for p in _files("synth", (".py",)):
        src = open(p).read()
        assert "import oracle" not in src and "from oracle" not in src and "log_mel_front_b200" not in src, p


def test_only_tests_entry_and_bench_import_the_oracle():
    allowed = {"bench.py", "__graft_entry__.py"}
    product = [os.path.join(ROOT, f) for f in os.listdir(ROOT) if f.endswith(".py") and f not in allowed]
    product += _files("log_mel_front_b200", (".py",)) + _files("synth", (".py",))
    for p in product:
        src = open(p).read()
        assert not re.search(r"^\s*(from|import)\s+oracle\b", src, re.M), p
