"""GPU parity where the model's bounds bind: every ClipLin's input and output
clamp, the three q/k/v output segments, SiLU's second clamp, the row passes'
next-input clamp, and the tanh soft-cap of the attention logits.

The workloads' bounds (+-8) never bind with N(0, 0.02) weights, so these cases
set their own (egemma2_audio.rs, ClipLin / Gemma4ClippableLinear: clamp the
input, x W^T, clamp the output; ``attention``: cap tanh(z / cap) on
q.k + q.R). BIND bounds every projection differently, tightly enough that
each clamp changes a sizeable share of its elements; q, k and v share their
input bounds (one fused projection) and differ in their output bounds; the
FFN W2 input bounds have lo above -0.279, SiLU's minimum, so the clamp after
SiLU binds too. CAP additionally scales the q and k weights by 32 (a power of
two keeps bf16 weights exact) with output bounds near +-8, so that most
dot-0 logits lie beyond the cap of 50.

The oracle run is instrumented on the CPU (its ``clip_lin`` and attention
core wrapped, values unchanged) to print and assert the share of elements
each clamp changes and the share of logits beyond the cap.

Tolerances: the library's float32 bound (1e-3) and the bf16 bound (2e-2 and
cosine 0.999) where they apply. With the cap saturated, the attention is a
high-gain stage: its softmax over logits near 50 turns any perturbation of q
or k into an output change. Emulating only the bf16 storage of the
projections' operands and outputs in the oracle moves one CAP layer by max
rel 0.078 (cosine 0.99992), so no bf16 implementation meets 2e-2 there; the
bf16 CAP layer is held to cosine 0.999 and max rel 0.15 (twice that
emulation), and the saturated cap is checked at the strict bounds in float32
and in the attention core alone, where both sides read the same bf16 q, k, v.
e4m3 uses the bounds set from its own sensitivity: a relative 1e-4
perturbation of the input moves the oracle's e4m3 BIND layer by max rel 0.029
(cosine 0.99988) and a two-layer encode by 0.062-0.077 (cosine 0.9992), so the
layer keeps the library's e4m3 layer bound (cosine 0.9995, max rel 5e-2) and
the two-layer encode takes cosine 0.998, max rel 0.15.
"""
import contextlib

import numpy as np
import pytest

import synth
from oracle import oracle as O
from tests.helpers import assert_bf16, assert_f32, cosine, dev, offsets, rel_err, workspace

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import log_mel_front_b200 as ae  # noqa: E402

BIND = {
    "ff1.w1": (-1.5, 1.5, -0.6, 0.5),
    "ff1.w2": (-0.15, 0.4, -0.25, 0.2),
    "q": (-1.25, 1.25, -0.5, 0.6),
    "k": (-1.25, 1.25, -0.7, 0.45),
    "v": (-1.25, 1.25, -0.4, 0.45),
    "post": (-0.3, 0.35, -0.15, 0.12),
    "lc_start": (-1.5, 1.4, -0.55, 0.5),
    "lc_end": (-0.2, 1.0, -0.3, 0.3),
    "ff2.w1": (-1.4, 1.6, -0.5, 0.6),
    "ff2.w2": (-0.1, 0.3, -0.2, 0.25),
}
CAP = dict(BIND, q=(-1.25, 1.25, -8.0, 7.0), k=(-1.25, 1.25, -6.0, 8.0))
QK_SCALE = 32.0

E4M3_LAYER_COS, E4M3_LAYER_REL = 0.9995, 5e-2
E4M3_ENC_COS, E4M3_ENC_REL = 0.998, 0.15
CAP_BF16_COS, CAP_BF16_REL = 0.999, 0.15


def _sync():
    torch.cuda.synchronize()
    assert ae.ae_device_status() == ae.AE_OK


def weights(kind, bounds, n_layers, qk_scale=1.0):
    w = synth.model_weights("pr1" if kind == "f32" else "tower", n_layers=n_layers)
    w["bounds"] = [dict(bounds) for _ in range(n_layers)]
    for ly in w["layers"]:
        for n in ("q", "k"):
            ly[n] = (ly[n] * np.float32(qk_scale)).astype(np.float32)
    return w


DTYPES = {"f32": ae.AE_F32, "bf16": ae.AE_BF16, "e4m3": ae.AE_FP8}


def oracle_weights(w, kind):
    return O.fp8_weights(w) if kind == "e4m3" else w


@contextlib.contextmanager
def instrumented(monkeypatch, layers):
    """Counts, per projection kind, the elements each clamp changes in the
    oracle run inside the block, and the share of distance-0 logits beyond
    the cap (the values the oracle computes are unchanged)."""
    names = {id(ly[n]): n for ly in layers for n in synth.CLIP_NAMES}
    stats = {n: np.zeros(5, np.int64) for n in synth.CLIP_NAMES}
    cap = {"beyond": 0, "total": 0}
    clip_lin, core = O.clip_lin, O.local_attention_core

    def counting_clip_lin(x, W, b=(-np.inf, np.inf, -np.inf, np.inf), fp8=False):
        n = names.get(id(W))
        if n is not None:
            xc = np.clip(x, b[0], b[1])
            y = xc @ np.asarray(W, np.float64).T
            s = stats[n]
            s += [int(((x < b[0]) | (x > b[1])).sum()), x.size, int((x < b[0]).sum()),
                  int(((y < b[2]) | (y > b[3])).sum()), y.size]
        return clip_lin(x, W, b, fp8)

    def counting_core(q, k, v, pos, R, qd, heads, left, cap_v):
        T, H = q.shape
        hd = H // heads
        qs = (q * O.q_scale_of(hd) * np.tile(np.asarray(qd, np.float64), heads)[None, :]).reshape(T, heads, hd)
        ks = (k * O.k_scale_of()).reshape(T, heads, hd)
        z = (qs * ks).sum(-1) + (qs * np.asarray(R[0], np.float64).reshape(heads, hd)[None]).sum(-1)
        cap["beyond"] += int((np.abs(z) > cap_v).sum())
        cap["total"] += z.size
        return core(q, k, v, pos, R, qd, heads, left, cap_v)

    monkeypatch.setattr(O, "clip_lin", counting_clip_lin)
    monkeypatch.setattr(O, "local_attention_core", counting_core)
    try:
        yield stats, cap
    finally:
        monkeypatch.setattr(O, "clip_lin", clip_lin)
        monkeypatch.setattr(O, "local_attention_core", core)


def report(stats, cap, what, cap_expected=False):
    for n in synth.CLIP_NAMES:
        x_out, x_n, x_lo, y_out, y_n = stats[n]
        print(f"[clamps] {what}: {n}: input {x_out}/{x_n} clamped ({x_lo} below lo), output {y_out}/{y_n} clamped")
        assert x_out > 0 and y_out > 0, f"{what}: a clamp of {n} never binds"
    for n in ("ff1.w2", "ff2.w2"):
        assert stats[n][2] > 0, f"{what}: SiLU's second clamp (the {n} input's lower bound) never binds"
    share = cap["beyond"] / max(cap["total"], 1)
    print(f"[softcap] {what}: {cap['beyond']}/{cap['total']} distance-0 logits beyond the cap ({share:.1%})")
    if cap_expected:
        assert share > 0.2, f"{what}: the soft-cap barely binds"


def gpu_layer(model, h, toks):
    T = sum(toks)
    d_h = dev(h.astype(np.float32))
    ws = workspace(model.workspace_size(len(toks), 0, T))
    ae.ae_conformer_layer(model, 0, d_h, offsets(toks), ws, ws.numel())
    _sync()
    return d_h.cpu().numpy()


def gpu_encode(model, clips):
    flat, off = synth.pack(clips)
    frames = sum(O.num_frames(len(c)) for c in clips)
    toks = [O.num_tokens(len(c)) for c in clips]
    d_out = torch.full((sum(toks) + 1, 512), float("nan"), device="cuda")   # one sentinel row
    ws = workspace(model.workspace_size(len(clips), frames, sum(toks)))
    ae.ae_encode(model, dev(flat), off, d_out, ws, ws.numel())
    _sync()
    g = d_out.cpu().numpy()
    assert np.all(np.isnan(g[-1])), "rows written beyond the batch's token count"
    return g[:-1]


TOKS = [5, 130, 300, 1, 11]


def _layer_input(seed=12):
    return np.random.default_rng(seed).standard_normal((sum(TOKS), 1024)).astype(np.float32)


@pytest.mark.parametrize("kind,bounds,qk", [("f32", "BIND", 1.0), ("f32", "CAP", QK_SCALE),
                                            ("bf16", "BIND", 1.0), ("bf16", "CAP", QK_SCALE),
                                            ("e4m3", "BIND", 1.0)])
def test_layer_with_binding_bounds(kind, bounds, qk, monkeypatch):
    w = weights(kind, {"BIND": BIND, "CAP": CAP}[bounds], 1, qk)
    h = _layer_input()
    m = ae.Model(w, DTYPES[kind])
    try:
        g = gpu_layer(m, h, TOKS)
    finally:
        m.close()
    wo = oracle_weights(w, kind)
    with instrumented(monkeypatch, wo["layers"]) as (stats, cap):
        o = O.conformer_layer(h.astype(np.float64), O.positions(TOKS), wo["layers"][0], w["bounds"][0], w["shape"],
                              fp8=(kind == "e4m3"))
    what = f"{kind} layer, {bounds} bounds"
    report(stats, cap, what, cap_expected=(bounds == "CAP"))
    assert np.all(np.isfinite(g))
    if kind == "f32":
        assert_f32(g, o, what)
    elif kind == "bf16" and bounds == "BIND":
        assert_bf16(g, o, what)
    else:
        c_min, r_max = (E4M3_LAYER_COS, E4M3_LAYER_REL) if kind == "e4m3" else (CAP_BF16_COS, CAP_BF16_REL)
        e, c = rel_err(g, o), cosine(g, o)
        print(f"[parity] {what}: rel err {e:.3e} (bound {r_max}), cosine {c:.7f} (bound {c_min})")
        assert e <= r_max and c >= c_min


def _clips():
    return [synth.noise_tones_clip(16000, 7, 0), synth.noise_tones_clip(40000, 7, 1)]


@pytest.mark.parametrize("kind,bounds,qk", [("f32", "CAP", QK_SCALE), ("bf16", "BIND", 1.0), ("e4m3", "BIND", 1.0)])
def test_encode_with_binding_bounds(kind, bounds, qk, monkeypatch):
    """Two short clips (1 s and 2.5 s) through the whole forward with two layers."""
    w = weights(kind, {"BIND": BIND, "CAP": CAP}[bounds], 2, qk)
    clips = _clips()
    m = ae.Model(w, DTYPES[kind])
    try:
        g = gpu_encode(m, clips)
    finally:
        m.close()
    wo = oracle_weights(w, kind)
    with instrumented(monkeypatch, wo["layers"]) as (stats, cap):
        o = np.concatenate(O.encode(clips, wo))
    what = f"{kind} encode, {bounds} bounds"
    report(stats, cap, what, cap_expected=(bounds == "CAP"))
    assert g.shape == o.shape and np.all(np.isfinite(g))
    if kind == "f32":
        assert_f32(g, o, what)
    elif kind == "bf16":
        assert_bf16(g, o, what)
    else:
        e, c = rel_err(g, o), cosine(g, o)
        print(f"[parity] {what}: rel err {e:.3e} (bound {E4M3_ENC_REL}), cosine {c:.7f} (bound {E4M3_ENC_COS})")
        assert e <= E4M3_ENC_REL and c >= E4M3_ENC_COS


def test_attention_core_softcap_saturated_bf16():
    """The attention kernel alone with q and k of N(0, 8^2) (bf16 values shared
    by both sides): most logits lie far beyond the cap of 50, so tanh
    saturates; every token is compared at the bf16 bound."""
    p = synth.attention_params()
    rng = np.random.default_rng(50)
    toks = [3, 12, 140, 200]
    T = sum(toks)
    q, k = (synth.round_to_bf16((8.0 * rng.standard_normal((T, 1024))).astype(np.float32)) for _ in range(2))
    v = synth.round_to_bf16(rng.standard_normal((T, 1024)).astype(np.float32))
    R, qs, ks = ae.ae_attention_tables(p["relk"], p["pds"])
    out = torch.full((T, 1024), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = workspace(ae.ae_workspace_size(None, len(toks), 0, T))
    ae.ae_local_attention(dev(q).to(torch.bfloat16), dev(k).to(torch.bfloat16), dev(v).to(torch.bfloat16), 1024,
                          ae.AE_BF16, dev(R), dev(qs), ks, 50.0, offsets(toks), out, 1024, ws, ws.numel())
    _sync()
    Ro = O.relative_keys(p["relk"], 12, 1024)
    qd = O.softplus(p["pds"])
    z = ((q * O.q_scale_of(128) * np.tile(qd, 8)).reshape(T, 8, 128) * (k * O.k_scale_of()).reshape(T, 8, 128)).sum(-1)
    share = float((np.abs(z) > 50.0).mean())
    print(f"[softcap] attention core: {share:.1%} of distance-0 logits beyond the cap")
    assert share > 0.5
    o = O.local_attention_core(q.astype(np.float64), k.astype(np.float64), v.astype(np.float64),
                               O.positions(toks), Ro, qd, 8, 12, 50.0)
    assert_bf16(out.float().cpu().numpy(), o, "attention core, saturated soft-cap")
