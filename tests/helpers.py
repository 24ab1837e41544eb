"""Shared pieces of the tests: error metrics, tolerances, device buffers."""
from __future__ import annotations

import numpy as np

# Tolerances (fixed by the benchmark spec of the workloads):
#   log-mel, float32:                max |gpu - oracle| <= 1e-3
#   float32 tower stages:            max |gpu - oracle| / max |oracle| <= 1e-3
#   bf16 tensor-core tower stages:   cosine >= 0.999 and max |gpu - oracle| / max |oracle| <= 2e-2
LOGMEL_ABS = 1e-3
F32_REL = 1e-3
BF16_COS = 0.999
BF16_REL = 2e-2


def rel_err(g, o) -> float:
    """Norm-wise relative error: max |g - o| / max |o|."""
    g, o = np.asarray(g, np.float64), np.asarray(o, np.float64)
    den = np.max(np.abs(o))
    return float(np.max(np.abs(g - o)) / (den if den > 0 else 1.0))


def cosine(g, o) -> float:
    g, o = np.asarray(g, np.float64).ravel(), np.asarray(o, np.float64).ravel()
    return float(g @ o / (np.linalg.norm(g) * np.linalg.norm(o) + 1e-300))


def assert_f32(g, o, what=""):
    e = rel_err(g, o)
    print(f"[parity] {what}: rel err {e:.3e} (bound {F32_REL})")
    assert e <= F32_REL, f"{what}: rel err {e:.3e} > {F32_REL}"
    return e


def assert_bf16(g, o, what=""):
    e, c = rel_err(g, o), cosine(g, o)
    print(f"[parity] {what}: rel err {e:.3e} (bound {BF16_REL}), cosine {c:.7f} (bound {BF16_COS})")
    assert e <= BF16_REL and c >= BF16_COS, f"{what}: rel err {e:.3e} (<= {BF16_REL}), cosine {c:.6f} (>= {BF16_COS})"
    return e, c


def assert_logmel(g, o, what=""):
    e = float(np.max(np.abs(np.asarray(g, np.float64) - np.asarray(o, np.float64)))) if np.size(o) else 0.0
    print(f"[parity] {what}: max abs err {e:.3e} (bound {LOGMEL_ABS})")
    assert e <= LOGMEL_ABS, f"{what}: max abs err {e:.3e} > {LOGMEL_ABS}"
    return e


def offsets(lengths) -> np.ndarray:
    off = np.zeros(len(lengths) + 1, np.int64)
    off[1:] = np.cumsum(lengths)
    return off


def dev(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def workspace(nbytes: int):
    import torch
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device="cuda")
