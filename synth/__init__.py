"""Seeded synthetic inputs shared by the oracle, the tests and the bench.

This module only draws random numbers and lays them out. It holds none of
the encoder's arithmetic: no framing, no FFT, no normalisation, no
projection. Both sides of every parity check (the CUDA library and the CPU
oracle) receive exactly the arrays produced here.

Workloads (the synthetic stand-ins for the clips the encoder sees; the pages
publish no dataset):

* ``pr1``       one clip of 1.0 s, ``0.5 sin(2 pi 440 t) + 0.1 N(0,1)``, seed 0;
                float32 weights, one Conformer layer.
* ``frontend``  64 clips x 30 s of ``N(0, 0.3)`` noise plus three random
                sinusoids (100-7900 Hz, amplitude U(0.05, 0.5), phase U(0, 2 pi)).
* ``tower``     16 clips x 30 s of the same noise-and-tone recipe; bf16
                weights, 12 layers and the embedding head.
* ``ragged``    256 clips with lengths drawn uniformly from whole samples in
                [16000, 480000], same recipe, 12 layers, bf16.
* ``attention`` 32 sequences x 8192 tokens of ``N(0,1)`` q/k/v (bf16 values),
                a random 1024x1024 relative-key projection and per-dim scales.

Weights: every matrix and convolution ``N(0, 0.02)``, ``per_dim_scale``
``N(0, 0.1)``, every norm gain ``1 + N(0, 0.02)``, the output bias and the
depthwise taps ``N(0, 0.02)``, clamp bounds +-8 on every clippable
projection. In the bf16 workloads every weight value is rounded to the
nearest bf16 (ties to even) here, so that the bf16 weights *are* the model.
"""
from __future__ import annotations

import numpy as np

SAMPLE_RATE = 16000
MAX_SAMPLES = 480000

# Shape of the release tower (gemma4_audio): the sizes the kernels are built for.
MODEL_SHAPE = dict(
    n_mels=128,
    c0=128,
    c1=32,
    hidden=1024,
    heads=8,
    ffn=4096,
    left=12,
    kernel=5,
    out_dim=1536,
    embed_dim=512,
    softcap=50.0,
    residual_weight=0.5,
)

# Names of the clippable projections of one layer, in a fixed order.
CLIP_NAMES = ("ff1.w1", "ff1.w2", "q", "k", "v", "post", "lc_start", "lc_end", "ff2.w1", "ff2.w2")

WORKLOADS = {
    "pr1": dict(config_index=0, n_layers=1, dtype="f32"),
    "frontend": dict(config_index=1, n_layers=0, dtype="f32"),
    "tower": dict(config_index=2, n_layers=12, dtype="bf16"),
    "ragged": dict(config_index=3, n_layers=12, dtype="bf16"),
    "attention": dict(config_index=4, n_layers=0, dtype="bf16"),
}


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """float32 array -> float32 array of the nearest bf16 values (ties to even)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    out = (r & 0xFFFFFFFF).astype(np.uint32).view(np.float32)
    return out.reshape(a.shape)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 array holding bf16 values -> uint16 bit patterns (exact)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


# ----------------------------------------------------------------- waveforms

def pr1_wave() -> np.ndarray:
    """One second: 0.5 sin(2 pi 440 t) + 0.1 N(0,1), seed 0."""
    rng = _rng(0)
    t = np.arange(SAMPLE_RATE, dtype=np.float64) / SAMPLE_RATE
    x = 0.5 * np.sin(2 * np.pi * 440.0 * t) + 0.1 * rng.standard_normal(SAMPLE_RATE)
    return x.astype(np.float32)


def noise_tones_clip(n: int, seed: int, index: int) -> np.ndarray:
    """N(0, 0.3) noise plus three sinusoids, 100-7900 Hz, amp U(0.05, 0.5), phase U(0, 2 pi)."""
    rng = _rng(seed, index)
    t = np.arange(n, dtype=np.float64) / SAMPLE_RATE
    x = 0.3 * rng.standard_normal(n)
    f = rng.uniform(100.0, 7900.0, 3)
    amp = rng.uniform(0.05, 0.5, 3)
    ph = rng.uniform(0.0, 2 * np.pi, 3)
    for j in range(3):
        x += amp[j] * np.sin(2 * np.pi * f[j] * t + ph[j])
    return x.astype(np.float32)


def clip_lengths(workload: str) -> list[int]:
    if workload == "pr1":
        return [SAMPLE_RATE]
    if workload == "frontend":
        return [MAX_SAMPLES] * 64
    if workload == "tower":
        return [MAX_SAMPLES] * 16
    if workload == "ragged":
        rng = _rng(WORKLOADS["ragged"]["config_index"], 999_999)
        return [int(v) for v in rng.integers(16000, 480000, size=256, endpoint=True)]
    raise ValueError(workload)


def global_lengths(workload: str, n_batches: int) -> list[int]:
    """Clip lengths of a global batch of n_batches times the workload's batch
    (the data-parallel runs split it over devices): batch 0 is the workload's
    own clips, batch b > 0 draws the same way with its own seed."""
    lens = list(clip_lengths(workload))
    for b in range(1, n_batches):
        if workload == "ragged":
            rng = _rng(WORKLOADS["ragged"]["config_index"], 999_999, b)
            lens += [int(v) for v in rng.integers(16000, 480000, size=256, endpoint=True)]
        else:
            lens += list(clip_lengths(workload))
    return lens


def global_waves(workload: str, lengths: list[int], clips: list[int]) -> list[np.ndarray]:
    """Clips (by global index) of a global batch with these lengths; for the
    indices of batch 0 these are exactly ``waves(workload)``'s clips."""
    seed = WORKLOADS[workload]["config_index"]
    return [noise_tones_clip(lengths[i], seed, i) for i in clips]


def waves(workload: str, clips: list[int] | None = None) -> list[np.ndarray]:
    """The workload's clips (or the listed subset of them), float32 each."""
    if workload == "pr1":
        return [pr1_wave()]
    lens = clip_lengths(workload)
    idx = range(len(lens)) if clips is None else clips
    seed = WORKLOADS[workload]["config_index"]
    return [noise_tones_clip(lens[i], seed, i) for i in idx]


def pack(clips: list[np.ndarray]) -> tuple[np.ndarray, np.ndarray]:
    """Clips back to back without padding, and int64 offsets [n_clips + 1]."""
    off = np.zeros(len(clips) + 1, dtype=np.int64)
    for i, c in enumerate(clips):
        off[i + 1] = off[i] + len(c)
    flat = np.concatenate(clips).astype(np.float32) if clips else np.zeros(0, np.float32)
    return flat, off


# ----------------------------------------------------------------- weights

def _normal(rng, shape, std, mean=0.0):
    return (mean + std * rng.standard_normal(shape, dtype=np.float32)).astype(np.float32)


def model_weights(workload: str, n_layers: int | None = None, bf16: bool | None = None,
                  shape: dict | None = None, clamp: float = 8.0) -> dict:
    """Random-init weights of the tower, in the checkpoint's tensor layout.

    Returns ``{"stem": {...}, "layers": [{...}, ...], "head": {...},
    "bounds": [{name: (lo_in, hi_in, lo_out, hi_out)}, ...]}``; matrices are
    ``[out, in]`` row-major float32.
    """
    w = WORKLOADS[workload]
    s = dict(MODEL_SHAPE if shape is None else shape)
    L = w["n_layers"] if n_layers is None else n_layers
    use_bf16 = (w["dtype"] == "bf16") if bf16 is None else bf16
    seed = 1000 + w["config_index"]
    H, F, C0, C1 = s["hidden"], s["ffn"], s["c0"], s["c1"]
    hd = H // s["heads"]

    r = _rng(seed, 0)
    stem = {
        "conv0": _normal(r, (C0, 9), 0.02),
        "ln0": _normal(r, (C0,), 0.02, 1.0),
        "conv1": _normal(r, (C1, C0, 3, 3), 0.02),
        "ln1": _normal(r, (C1,), 0.02, 1.0),
        "in_proj": _normal(r, (H, C1 * (s["n_mels"] // 4)), 0.02),
    }
    layers, bounds = [], []
    for i in range(L):
        r = _rng(seed, 1 + i)
        ly = {}
        for f in ("ff1", "ff2"):
            ly[f + ".pre"] = _normal(r, (H,), 0.02, 1.0)
            ly[f + ".w1"] = _normal(r, (F, H), 0.02)
            ly[f + ".w2"] = _normal(r, (H, F), 0.02)
            ly[f + ".post"] = _normal(r, (H,), 0.02, 1.0)
        ly["norm_pre_attn"] = _normal(r, (H,), 0.02, 1.0)
        ly["norm_post_attn"] = _normal(r, (H,), 0.02, 1.0)
        ly["norm_out"] = _normal(r, (H,), 0.02, 1.0)
        for p in ("q", "k", "v", "post"):
            ly[p] = _normal(r, (H, H), 0.02)
        ly["pds"] = _normal(r, (hd,), 0.1)
        ly["relk"] = _normal(r, (H, H), 0.02)
        ly["lc_pre"] = _normal(r, (H,), 0.02, 1.0)
        ly["lc_start"] = _normal(r, (2 * H, H), 0.02)
        ly["lc_dw"] = _normal(r, (H, s["kernel"]), 0.02)
        ly["lc_norm"] = _normal(r, (H,), 0.02, 1.0)
        ly["lc_end"] = _normal(r, (H, H), 0.02)
        layers.append(ly)
        bounds.append({n: (-clamp, clamp, -clamp, clamp) for n in CLIP_NAMES})
    r = _rng(seed, 10_000)
    head = {
        "out_proj": _normal(r, (s["out_dim"], H), 0.02),
        "out_bias": _normal(r, (s["out_dim"],), 0.02),
        "embed": _normal(r, (s["embed_dim"], s["out_dim"]), 0.02),
    }
    out = {"stem": stem, "layers": layers, "head": head, "bounds": bounds, "shape": s,
           "bf16": use_bf16}
    if use_bf16:
        for d in [stem, head] + layers:
            for k in d:
                d[k] = round_to_bf16(d[k])
    return out


# ----------------------------------------------------------------- attention microbench

# Input conditioning (mixdown + resampling to 16 kHz): 64 stereo clips of 30 s
# at 44.1 kHz, the common consumer source rate, each channel N(0, 0.2) noise
# plus three sinusoids of 50-20000 Hz (some above the new Nyquist).
RS_CLIPS = 64
RS_RATE = 44100
RS_SECONDS = 30


def resample_clip(index: int, n: int | None = None, rate: int = RS_RATE, channels: int = 2) -> list[np.ndarray]:
    """One clip of the resampling workload: a list of `channels` float32 arrays."""
    n = rate * RS_SECONDS if n is None else n
    rng = _rng(9, index)
    t = np.arange(n, dtype=np.float64) / rate
    out = []
    for _ in range(channels):
        x = 0.2 * rng.standard_normal(n)
        for _ in range(3):
            f = rng.uniform(50.0, 20000.0)
            x = x + rng.uniform(0.05, 0.3) * np.sin(2 * np.pi * f * t + rng.uniform(0, 2 * np.pi))
        out.append(x.astype(np.float32))
    return out


ATT_SEQS = 32
ATT_T = 8192


def attention_params(hidden: int = 1024, heads: int = 8) -> dict:
    """Relative-key projection [hidden, hidden] N(0, 0.02) and per_dim_scale N(0, 0.1)."""
    r = _rng(WORKLOADS["attention"]["config_index"], 0)
    return {"relk": _normal(r, (hidden, hidden), 0.02),
            "pds": _normal(r, (hidden // heads,), 0.1)}


def attention_qkv(seq: int, T: int = ATT_T, hidden: int = 1024) -> tuple[np.ndarray, ...]:
    """q, k, v of one sequence: [T, hidden] float32 holding bf16 values of N(0,1)."""
    r = _rng(WORKLOADS["attention"]["config_index"], 1 + seq)
    return tuple(round_to_bf16(r.standard_normal((T, hidden), dtype=np.float32)) for _ in range(3))


# ----------------------------------------------------------------- LFM2A encoder body

# The LFM2A Conformer encoder's shape as the library reads it (17 blocks of
# width 512 with 8 heads; the other sizes are readings, the page names them
# without values).
LENC_SHAPE = dict(n_mels=128, n_embd=512, n_head=8, n_layers=17, n_ff=2048, conv_k=9, stem_ch=256,
                  adapter_ff=2048, llm_hidden=2048, eps=1e-5)

LENC_BLOCK_VECTORS = ("ffn1.norm_b", "ffn1.down_b", "ln1_b", "attn_q_b", "attn_k_b", "attn_v_b", "attn_o_b",
                      "pos_bias_u", "pos_bias_v", "norm_conv_b", "conv_dw_b", "conv_norm_b", "conv_pw2_b",
                      "ffn2.norm_b", "ffn2.down_b", "ln2_b")


def lfm_encoder_weights(n_layers: int | None = None, shape: dict | None = None, seed: int = 5000) -> dict:
    """Random-init weights of the LFM2A encoder body in the page's tensor
    layouts (matrices [out, in], stem convolutions [C_out][C_in/groups][kh][kw],
    the depthwise conv1d taps [k][C]). Stem convolutions and pre_encode_out
    N(0, 1 / fan_in), so the activations keep their scale through the ReLUs;
    block and adapter matrices N(0, 0.02); LayerNorm gains and the conv
    module's channel scale 1 + N(0, 0.02); biases and the depthwise taps
    N(0, 0.02) and N(0, 1 / k). Every matrix the tensor cores multiply (the
    pointwise stem convolutions, pre_encode_out, the block and adapter
    matrices, linear_pos) is rounded to bf16 here, so the bf16 values are the
    model; vectors and the 3x3 stem taps stay float32."""
    s = dict(LENC_SHAPE if shape is None else shape)
    L = s["n_layers"] if n_layers is None else n_layers
    s["n_layers"] = L
    D, F, C, K = s["n_embd"], s["n_ff"], s["stem_ch"], s["conv_k"]
    r = _rng(seed, 0)
    W = {"cfg": s, "layers": []}
    for i, (dw, k, cin) in enumerate(((False, 3, 1), (True, 3, C), (False, 1, C), (True, 3, C), (False, 1, C))):
        fan = (1 if dw else cin) * k * k
        w = _normal(r, (C, 1 if dw else cin, k, k), fan ** -0.5)
        W[f"stem{i}.w"] = w if k == 3 else round_to_bf16(w)
        W[f"stem{i}.b"] = _normal(r, (C,), 0.02)
    fq = s["n_mels"] // 8
    W["pre_w"] = round_to_bf16(_normal(r, (D, C * fq), (C * fq) ** -0.5))
    W["pre_b"] = _normal(r, (D,), 0.02)
    for l in range(L):
        r = _rng(seed, 1 + l)
        ly = {}
        for f in ("ffn1", "ffn2"):
            ly[f + ".norm_w"] = _normal(r, (D,), 0.02, 1.0)
            ly[f + ".norm_b"] = _normal(r, (D,), 0.02)
            ly[f + ".up_w"] = round_to_bf16(_normal(r, (F, D), 0.02))
            ly[f + ".up_b"] = _normal(r, (F,), 0.02)
            ly[f + ".down_w"] = round_to_bf16(_normal(r, (D, F), 0.02))
            ly[f + ".down_b"] = _normal(r, (D,), 0.02)
        for n in ("ln1", "ln2", "norm_conv"):
            ly[n + "_w"] = _normal(r, (D,), 0.02, 1.0)
            ly[n + "_b"] = _normal(r, (D,), 0.02)
        for c in "qkvo":
            ly[f"attn_{c}_w"] = round_to_bf16(_normal(r, (D, D), 0.02))
            ly[f"attn_{c}_b"] = _normal(r, (D,), 0.02)
        ly["linear_pos_w"] = round_to_bf16(_normal(r, (D, D), 0.02))
        ly["pos_bias_u"] = _normal(r, (D,), 0.02)
        ly["pos_bias_v"] = _normal(r, (D,), 0.02)
        ly["conv_pw1_w"] = round_to_bf16(_normal(r, (2 * D, D), 0.02))
        ly["conv_pw1_b"] = _normal(r, (2 * D,), 0.02)
        ly["conv_dw_w"] = _normal(r, (K, D), K ** -0.5)
        ly["conv_dw_b"] = _normal(r, (D,), 0.02)
        ly["conv_norm_w"] = _normal(r, (D,), 0.02, 1.0)
        ly["conv_norm_b"] = _normal(r, (D,), 0.02)
        ly["conv_pw2_w"] = round_to_bf16(_normal(r, (D, D), 0.02))
        ly["conv_pw2_b"] = _normal(r, (D,), 0.02)
        W["layers"].append(ly)
    r = _rng(seed, 100_000)
    W["ad_norm_w"] = _normal(r, (D,), 0.02, 1.0)
    W["ad_norm_b"] = _normal(r, (D,), 0.02)
    W["ad_up_w"] = round_to_bf16(_normal(r, (s["adapter_ff"], D), 0.02))
    W["ad_up_b"] = _normal(r, (s["adapter_ff"],), 0.02)
    W["ad_down_w"] = round_to_bf16(_normal(r, (s["llm_hidden"], s["adapter_ff"]), 0.02))
    W["ad_down_b"] = _normal(r, (s["llm_hidden"],), 0.02)
    return W
