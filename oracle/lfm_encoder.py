"""Plain, slow, float64 CPU oracle of the LFM2A Conformer audio encoder body.

TEST INFRASTRUCTURE ONLY: the parity tests, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU legs call it; the CUDA library never does, and this file
shares no code, table or constant generator with it.

Source: the docs.rs page of cera 0.5.3, ``audio_encoder_gpu.rs`` ("GPU
forward pass for the LFM2A Conformer audio encoder"): ``encode_audio_gpu``
(the stem, 17 blocks, the adapter), ``macaron_ffn``, ``conv_stem_gpu`` with
``STEM_LAYER_MODES`` and ``STEM_RELU_AFTER``, the ``AudioEncoderGpuOps``
trait (what ``layernorm``, ``linear``, ``glu_split``, ``chan_affine_silu``,
``gelu_erf`` and ``xl_attention`` compute) and ``validate_block`` (the
weight shapes). Everything is float64 with direct definitions: convolutions
as sums over their taps, projections as matrix products, the attention as an
explicit loop over the query rows.

Readings of what the page leaves open (listed again in the design notes):

* Sizes the page names without values: ``n_ff`` = 4 n_embd (2048),
  ``conv_dw_k`` = 9, ``POS_EMB_DIM`` = n_embd, the stem's 256 channels, the
  adapter's intermediate width 2048 and ``llm_hidden_size`` 2048, LayerNorm
  eps 1e-5. The page fixes 17 blocks, 8 heads and head_dim 64 (n_embd 512).
* ``relative_pos_emb(t)`` (2t - 1 rows, not shown): row r holds relative
  position t - 1 - r (from t - 1 down to -(t - 1)) as interleaved
  sin/cos pairs, [sin(p w_i), cos(p w_i)] for w_i = 10000^(-2i / d).
* ``xl_attention`` (the shader is not shown): the Transformer-XL score of
  query i and key j is ((q_i + bias_u) . k_j + (q_i + bias_v) . p_{t-1-i+j})
  / sqrt(head_dim), i.e. the position row of relative distance i - j, then a
  softmax over all keys of the clip and the weighted sum of v.
* The stem's flatten: (channel, time, freq) to (time, channel * f_out + f),
  as ``conv_stem_gpu`` permutes it, then ``pre_encode_out`` with its bias.
* The depthwise conv1d of the conv module pads (k - 1) / 2 on the left and
  the rest on the right (the page's split), within each clip; its weights are
  stored kernel-first, [k][channels] (``validate_block``).
* A batch of clips is encoded clip by clip (the page encodes one chunk).

Parity status: pinned by ``tests/test_lfm_encoder_pins.py`` (brute-force
convolutions on tiny inputs, the stem's output geometry, the position
table's closed form, attention against torch's scaled_dot_product_attention
when the position terms vanish, the relative shift's Toeplitz structure and
distance-0 row, GELU against math.erf, LayerNorm moments, the depthwise
conv's impulse response, the macaron half weight). The readings above are
readings: the page prints no value that fixes them.
"""
from __future__ import annotations

import math

import numpy as np

# cera 0.5.3, audio_encoder_gpu.rs: STEM_LAYER_MODES (depthwise, stride, pad),
# with the kernel sizes its comments give, and STEM_RELU_AFTER
STEM_MODES = ((False, 2, 1, 3), (True, 2, 1, 3), (False, 1, 0, 1), (True, 2, 1, 3), (False, 1, 0, 1))
STEM_RELU = (True, False, True, False, True)

DEFAULTS = dict(n_mels=128, n_embd=512, n_head=8, n_layers=17, n_ff=2048, conv_k=9, stem_ch=256,
                adapter_ff=2048, llm_hidden=2048, eps=1e-5)


def conv2d(x: np.ndarray, w: np.ndarray, b: np.ndarray, stride: int, pad: int, groups: int) -> np.ndarray:
    """Direct 2D convolution (the trait's ``conv2d``): x [C_in][H][W], w
    [C_out][C_in/groups][kh][kw], b [C_out]; zero padding ``pad`` on every
    side; output [C_out][H_out][W_out], H_out = (H + 2 pad - kh) // stride + 1."""
    x = np.asarray(x, np.float64)
    w = np.asarray(w, np.float64)
    cin, H, W = x.shape
    cout, cpg, kh, kw = w.shape
    ho, wo = (H + 2 * pad - kh) // stride + 1, (W + 2 * pad - kw) // stride + 1
    xp = np.zeros((cin, H + 2 * pad, W + 2 * pad))
    xp[:, pad:pad + H, pad:pad + W] = x
    out = np.zeros((cout, ho, wo))
    opg = cout // groups
    for g in range(groups):
        xs = xp[g * cpg:(g + 1) * cpg]
        for dh in range(kh):
            for dw in range(kw):
                patch = xs[:, dh:dh + stride * (ho - 1) + 1:stride, dw:dw + stride * (wo - 1) + 1:stride]
                # [cpg, ho, wo] x [opg, cpg] -> [opg, ho, wo]
                out[g * opg:(g + 1) * opg] += np.einsum("chw,oc->ohw", patch, w[g * opg:(g + 1) * opg, :, dh, dw])
    return out + np.asarray(b, np.float64)[:, None, None]


def stem(mel: np.ndarray, W: dict) -> np.ndarray:
    """``conv_stem_gpu``: five convolutions (ReLU after the 1st, 3rd and 5th),
    the (channel, time, freq) -> (time, channel * freq) flatten and
    ``pre_encode_out`` with its bias. mel [F][n_mels] -> [T][n_embd]."""
    x = np.asarray(mel, np.float64)[None]               # [1][F][n_mels]: channel, time, freq
    for i, (dw, stride, pad, k) in enumerate(STEM_MODES):
        groups = x.shape[0] if dw else 1
        x = conv2d(x, W[f"stem{i}.w"], W[f"stem{i}.b"], stride, pad, groups)
        if STEM_RELU[i]:
            x = np.maximum(x, 0.0)
    c, t, f = x.shape
    flat = x.transpose(1, 0, 2).reshape(t, c * f)
    return flat @ np.asarray(W["pre_w"], np.float64).T + np.asarray(W["pre_b"], np.float64)


def stem_len(frames: int) -> int:
    """Rows after the stem: three 3x3 stride-2 pad-1 convolutions, each
    ceil(n / 2)."""
    n = frames
    for _ in range(3):
        n = (n + 2 - 3) // 2 + 1 if n > 0 else 0
    return n


def layer_norm(x: np.ndarray, w, b, eps: float) -> np.ndarray:
    """The trait's ``layernorm``: (x - mean) / sqrt(var + eps) * w + b per row
    (biased variance)."""
    x = np.asarray(x, np.float64)
    m = x.mean(-1, keepdims=True)
    v = ((x - m) ** 2).mean(-1, keepdims=True)
    return (x - m) / np.sqrt(v + eps) * np.asarray(w, np.float64) + np.asarray(b, np.float64)


def silu(x):
    return x / (1.0 + np.exp(-x))


def gelu_erf(x):
    """The erf form of GELU (``gelu_erf``): x (1 + erf(x / sqrt 2)) / 2."""
    x = np.asarray(x, np.float64)
    erf = np.vectorize(math.erf, otypes=[np.float64])
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def linear(x, w, b=None):
    y = np.asarray(x, np.float64) @ np.asarray(w, np.float64).T
    return y if b is None else y + np.asarray(b, np.float64)


def relative_pos_emb(t: int, d: int) -> np.ndarray:
    """[2t - 1][d]: row r is relative position p = t - 1 - r, columns 2i and
    2i + 1 are sin(p w_i) and cos(p w_i), w_i = 10000^(-2i / d)."""
    p = (t - 1 - np.arange(2 * t - 1, dtype=np.float64))[:, None]
    w = np.exp(-np.arange(0, d, 2, dtype=np.float64) * (math.log(10000.0) / d))[None, :]
    out = np.zeros((2 * t - 1, d))
    out[:, 0::2] = np.sin(p * w)
    out[:, 1::2] = np.cos(p * w)
    return out


def xl_attention(q, k, v, p, bu, bv, heads: int) -> np.ndarray:
    """``xl_attention``: per head, score(i, j) = ((q_i + bu) . k_j +
    (q_i + bv) . p_{t-1-i+j}) / sqrt(hd); softmax over j < t; sum of v.
    q, k, v [t][heads*hd], p [2t-1][heads*hd]."""
    t, H = q.shape
    hd = H // heads
    qu = (q + bu).reshape(t, heads, hd)
    qv = (q + bv).reshape(t, heads, hd)
    kh = k.reshape(t, heads, hd)
    vh = v.reshape(t, heads, hd)
    ph = p.reshape(2 * t - 1, heads, hd)
    out = np.zeros((t, heads, hd))
    scale = 1.0 / math.sqrt(hd)
    for i in range(t):
        rows = t - 1 - i + np.arange(t)                  # position row of distance i - j, j = 0..t-1
        s = (np.einsum("hd,jhd->hj", qu[i], kh) + np.einsum("hd,jhd->hj", qv[i], ph[rows])) * scale
        s = s - s.max(-1, keepdims=True)
        e = np.exp(s)
        a = e / e.sum(-1, keepdims=True)
        out[i] = np.einsum("hj,jhd->hd", a, vh)
    return out.reshape(t, H)


def depthwise_conv1d(x: np.ndarray, w: np.ndarray, b) -> np.ndarray:
    """The conv module's depthwise conv along time: x [t][C], w [k][C]
    (kernel first), pad (k - 1) // 2 on the left and the rest on the right:
    y[i][c] = b[c] + sum_m w[m][c] x[i + m - (k - 1) // 2][c]."""
    x = np.asarray(x, np.float64)
    w = np.asarray(w, np.float64)
    t, C = x.shape
    k = w.shape[0]
    lo = (k - 1) // 2
    xp = np.zeros((t + k - 1, C))
    xp[lo:lo + t] = x
    y = np.zeros((t, C))
    for m in range(k):
        y += w[m][None, :] * xp[m:m + t]
    return y + np.asarray(b, np.float64)[None, :]


def macaron_ffn(x, ly, f: str, eps: float) -> np.ndarray:
    """``macaron_ffn``: x + 0.5 (W_down silu(W_up LN(x) + b_up) + b_down)."""
    n = layer_norm(x, ly[f + ".norm_w"], ly[f + ".norm_b"], eps)
    mid = silu(linear(n, ly[f + ".up_w"], ly[f + ".up_b"]))
    return x + 0.5 * linear(mid, ly[f + ".down_w"], ly[f + ".down_b"])


def block(x, ly: dict, pos_emb: np.ndarray, cfg: dict) -> np.ndarray:
    """One Conformer block of ``encode_audio_gpu``."""
    eps, heads = cfg["eps"], cfg["n_head"]
    x = macaron_ffn(x, ly, "ffn1", eps)
    n = layer_norm(x, ly["ln1_w"], ly["ln1_b"], eps)
    q, k, v = (linear(n, ly[f"attn_{c}_w"], ly[f"attn_{c}_b"]) for c in "qkv")
    p = linear(pos_emb, ly["linear_pos_w"])                       # no bias
    a = xl_attention(q, k, v, p, np.asarray(ly["pos_bias_u"], np.float64), np.asarray(ly["pos_bias_v"], np.float64),
                     heads)
    x = x + linear(a, ly["attn_o_w"], ly["attn_o_b"])
    n = layer_norm(x, ly["norm_conv_w"], ly["norm_conv_b"], eps)
    g = linear(n, ly["conv_pw1_w"], ly["conv_pw1_b"])
    C = g.shape[1] // 2
    g = g[:, :C] / (1.0 + np.exp(-g[:, C:]))                      # glu_split: first half times sigma(second)
    c = depthwise_conv1d(g, ly["conv_dw_w"], ly["conv_dw_b"])
    c = silu(c * np.asarray(ly["conv_norm_w"], np.float64) + np.asarray(ly["conv_norm_b"], np.float64))
    x = x + linear(c, ly["conv_pw2_w"], ly["conv_pw2_b"])
    x = macaron_ffn(x, ly, "ffn2", eps)
    return layer_norm(x, ly["ln2_w"], ly["ln2_b"], eps)


def adapter(x, W: dict, eps: float) -> np.ndarray:
    """Stage 4 of ``encode_audio_gpu``: LN, up + bias, erf GELU, down + bias."""
    n = layer_norm(x, W["ad_norm_w"], W["ad_norm_b"], eps)
    return linear(gelu_erf(linear(n, W["ad_up_w"], W["ad_up_b"])), W["ad_down_w"], W["ad_down_b"])


def encode(mel: np.ndarray, W: dict, trace: dict | None = None) -> np.ndarray:
    """``encode_audio_gpu`` for one clip's spectrogram [F][n_mels]:
    [stem_len(F)][llm_hidden] (empty for a clip too short for the stem)."""
    cfg = W["cfg"]
    if stem_len(mel.shape[0]) == 0:
        return np.zeros((0, cfg["llm_hidden"]))
    x = stem(mel, W)
    if trace is not None:
        trace["stem"] = x.copy()
        trace["blocks"] = []
    pe = relative_pos_emb(x.shape[0], cfg["n_embd"])
    for ly in W["layers"]:
        x = block(x, ly, pe, cfg)
        if trace is not None:
            trace["blocks"].append(x.copy())
    return adapter(x, W, cfg["eps"])
