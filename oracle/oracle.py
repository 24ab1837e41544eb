"""Plain, slow, float64 CPU oracle of the gemma4_audio encoder forward.

TEST INFRASTRUCTURE ONLY: the parity tests, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline legs call it; the CUDA library never does, and
this file shares no code, table or constant generator with it.

Source: the docs.rs page of cortiq-engine 0.8.49, ``egemma2_audio.rs``
("EmbeddingGemma 2 audio: the gemma4_audio tower"), and the RMS-norm helpers
of ``ltxdit.rs`` (cortiq-engine 0.5.94) that the same crate uses. Each
function names the item of the page it restates. Everything is computed in
float64 with direct definitions: a naive DFT (a matrix product with an
explicit twiddle table), direct 3x3 convolutions, plain matrix products for
the projections, and the windowed attention as an explicit loop over the
twelve distances.

Readings of points the page leaves open (listed again in the design notes):

* RMS norm is ``x * w / sqrt(mean(x^2) + 1e-6)`` with float64 statistics
  (``rms_rows``/``rms_into`` are imported from a module the pages do not
  show; the module's ``EPS`` and the ``rms_w``/``rms_plain`` helpers of
  ``ltxdit.rs`` fix the form).
* Only the ten ``ClipLin`` projections per layer clamp; ``in_proj``,
  ``relative_k_proj``, ``out_proj`` and ``embed`` are plain matrices.
* The softmax uses the natural exponential (``attention``), although the
  logits carry log2 scale factors.
* Relative-key rows 0..left-1 are used (13 are built).
* The window product, the FFT magnitude and the sinusoid table stay in
  float64 here (the page rounds some of them to float32; the difference is
  far below every tolerance).

The e4m3 projections (``e4m3_round`` .. ``fp8_weights``) are the library's
own low-precision variant, not the page's arithmetic: the page only keeps a
quantized pack's kernels as an option. They are pinned by torch's
``float8_e4m3fn`` conversion, the format's special values and invariants of
the row quantisation.

Parity status: every stage is pinned by the ``-m "not gpu"`` tests (page
values, closed forms, invariants, brute force), the head and the input
projection included (a hand-worked head example, the weightless norm's scale
invariance, and a non-symmetric ``input_proj_linear`` that fixes which axis of
the stored matrix is the output). The composition of a full layer and of the
tower is pinned only by a tiny-size brute-force restatement and by packing
invariance; no end-to-end value is printed on the pages.
"""
from __future__ import annotations

import math

import numpy as np

# egemma2_audio.rs, "sizes" / module constants
SAMPLE_RATE = 16000
MAX_SAMPLES = 480000
FRAME = 320
HOP = 160
N_FFT = 512
N_MELS = 128
MEL_FLOOR = 1e-3
EPS = 1e-6

__all__ = [
    "num_frames", "num_tokens", "linspace_exact", "hz_to_mel", "mel_to_hz",
    "mel_filter_bank", "hann_periodic", "frames_of", "dft_magnitude", "log_mel",
    "conv0_raw", "conv0_ln_relu", "conv1_raw", "conv1_ln_relu", "stem", "subsample", "rms", "clip_lin",
    "silu", "sigmoid", "softplus", "sinusoids", "relative_keys", "q_scale_of",
    "k_scale_of", "ffn", "local_attention_core", "attention", "glu", "dwconv",
    "light_conv", "conformer_layer", "head", "positions", "encode",
    "layer_tables", "e4m3_round", "e4m3_decode", "linear_e4m3", "e4m3_rows", "e4m3_dequant_rows", "input_scale", "quantize_input",
    "fp8_weights", "FP8_MATRICES",
]


# ------------------------------------------------------------------ sizes

def num_frames(n: int) -> int:
    """``num_frames``: frames of a clip of n samples after the 30 s cut."""
    n = min(int(n), MAX_SAMPLES)
    return 0 if n <= HOP else -(-(n - HOP) // HOP)


def num_tokens(n: int) -> int:
    """``num_tokens``: two stride-2 convolutions over the frames."""
    f = num_frames(n)
    return -(-(-(-f // 2)) // 2)


# ------------------------------------------------------------------ log-mel

def linspace_exact(a: float, b: float, n: int) -> np.ndarray:
    """``linspace``: a + i*step, the last point set to b exactly."""
    step = (b - a) / (n - 1)
    v = a + np.arange(n, dtype=np.float64) * step
    v[-1] = b
    return v


def hz_to_mel(f):
    """HTK mel scale: 2595 log10(1 + f/700)."""
    return 2595.0 * np.log10(1.0 + np.asarray(f, dtype=np.float64) / 700.0)


def mel_to_hz(m):
    return 700.0 * (10.0 ** (np.asarray(m, dtype=np.float64) / 2595.0) - 1.0)


def mel_filter_bank(n_fft: int = N_FFT, n_mels: int = N_MELS, sr: int = SAMPLE_RATE) -> np.ndarray:
    """``mel_filter_bank``: HTK triangles, no normalisation, [257 freq][128 mel]."""
    n_freq = n_fft // 2 + 1
    mels = linspace_exact(float(hz_to_mel(0.0)), float(hz_to_mel(sr / 2)), n_mels + 2)
    ff = mel_to_hz(mels)
    fft = linspace_exact(0.0, sr / 2, n_freq)
    out = np.zeros((n_freq, n_mels), dtype=np.float64)
    for m in range(n_mels):
        down = -(ff[m] - fft) / (ff[m + 1] - ff[m])
        up = (ff[m + 2] - fft) / (ff[m + 2] - ff[m + 1])
        out[:, m] = np.maximum(0.0, np.minimum(down, up))
    return out


def hann_periodic(n: int = FRAME) -> np.ndarray:
    """``MelFrontend::new``: periodic Hann, 0.5 - 0.5 cos(2 pi j / n)."""
    j = np.arange(n, dtype=np.float64)
    return 0.5 - 0.5 * np.cos(2.0 * np.pi * j / n)


def frames_of(wave: np.ndarray) -> np.ndarray:
    """``MelFrontend::log_mel`` framing: frame i, sample j < 320 is
    wave[i*160 + j - 160] (zero before the clip), times the window. [F, 320]."""
    w = np.asarray(wave, dtype=np.float64)[:MAX_SAMPLES]
    nf = num_frames(len(w))
    padded = np.concatenate([np.zeros(HOP), w])
    idx = np.arange(nf)[:, None] * HOP + np.arange(FRAME)[None, :]
    return padded[idx] * hann_periodic()[None, :]


def _twiddles(n_in: int = FRAME, n_fft: int = N_FFT):
    """cos/sin of 2 pi ((k n) mod 512) / 512 for n < n_in, k <= 256, in float64."""
    n = np.arange(n_in)[:, None]
    k = np.arange(n_fft // 2 + 1)[None, :]
    m = (n * k) % n_fft
    ang = 2.0 * np.pi * m / n_fft
    return np.cos(ang), np.sin(ang)


def dft_magnitude(frames: np.ndarray) -> np.ndarray:
    """|X_k| = |sum_n x_n exp(-2 pi i k n / 512)|, k = 0..256 (naive DFT of the
    zero-padded frame; the page's rfft magnitude, not power)."""
    c, s = _twiddles(frames.shape[1])
    re = frames @ c
    im = -(frames @ s)
    return np.hypot(re, im)


def log_mel(wave: np.ndarray, bank: np.ndarray | None = None) -> np.ndarray:
    """``MelFrontend::log_mel``: ln(sum_k |X_k| M[k][b] + 0.001), [F, 128]."""
    m = mel_filter_bank() if bank is None else bank
    fr = frames_of(wave)
    if fr.shape[0] == 0:
        return np.zeros((0, N_MELS))
    out = np.empty((fr.shape[0], m.shape[1]))
    step = 8192
    for s in range(0, fr.shape[0], step):
        mag = dft_magnitude(fr[s:s + step])
        out[s:s + step] = np.log(mag @ m + MEL_FLOOR)
    return out


# ------------------------------------------------------------------ stem

def _layer_norm_relu(x: np.ndarray, g: np.ndarray) -> np.ndarray:
    """``layer_norm_relu``: bias-free LayerNorm over the last axis (mean and
    biased variance, eps 1e-6), times the gain, then ReLU."""
    mean = x.mean(axis=-1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=-1, keepdims=True)
    y = (x - mean) / np.sqrt(var + EPS) * np.asarray(g, np.float64)
    return np.maximum(y, 0.0)


def conv0_raw(mel: np.ndarray, w0: np.ndarray) -> np.ndarray:
    """``subsample`` layer 0 before its norm: 3x3 stride-2 conv, zero pad 1,
    1 -> C0 channels, no bias; tap (dt, df) reads mel[2t+dt-1][2f+df-1].
    mel [F, 128] -> [ceil(F/2), 64, C0]."""
    F, nm = mel.shape
    t1, f1 = -(-F // 2), -(-nm // 2)
    w0 = np.asarray(w0, np.float64).reshape(w0.shape[0], 9)
    P = np.zeros((2 * t1 + 2, 2 * f1 + 2))
    P[1:F + 1, 1:nm + 1] = mel
    acc = np.zeros((t1, f1, w0.shape[0]))
    for dt in range(3):
        for df in range(3):
            patch = P[dt:dt + 2 * t1:2, df:df + 2 * f1:2]
            acc += patch[:, :, None] * w0[None, None, :, dt * 3 + df]
    return acc


def conv0_ln_relu(mel: np.ndarray, w0: np.ndarray, g0: np.ndarray) -> np.ndarray:
    """``subsample`` layer 0: conv, LayerNorm over channels, ReLU."""
    return _layer_norm_relu(conv0_raw(mel, w0), g0)


def conv1_raw(y0: np.ndarray, w1: np.ndarray) -> np.ndarray:
    """``subsample`` layer 1 before its norm: 3x3 stride-2 conv, zero pad 1,
    C0 -> C1 channels, weight [C1][C0][dt][df]. [t1, 64, C0] -> [t2, 32, C1]."""
    t1, f1, c0 = y0.shape
    t2, f2 = -(-t1 // 2), -(-f1 // 2)
    w1 = np.asarray(w1, np.float64)
    Q = np.zeros((2 * t2 + 2, 2 * f2 + 2, c0))
    Q[1:t1 + 1, 1:f1 + 1] = y0
    acc = np.zeros((t2, f2, w1.shape[0]))
    for dt in range(3):
        for df in range(3):
            patch = Q[dt:dt + 2 * t2:2, df:df + 2 * f2:2]
            acc += patch @ w1[:, :, dt, df].T
    return acc


def conv1_ln_relu(y0: np.ndarray, w1: np.ndarray, g1: np.ndarray) -> np.ndarray:
    """``subsample`` layer 1: conv, LayerNorm over channels, ReLU, flattened
    frequency-major (index f*C1 + c) to [T, 32*C1]."""
    acc = conv1_raw(y0, w1)
    y = _layer_norm_relu(acc, g1)
    return y.reshape(acc.shape[0], acc.shape[1] * acc.shape[2])


def stem(mel: np.ndarray, W: dict) -> np.ndarray:
    """Both convolutions of one clip, before the input projection: [T, 1024]."""
    if mel.shape[0] == 0:
        return np.zeros((0, W["conv1"].shape[0] * (N_MELS // 4)))
    y0 = conv0_ln_relu(mel, W["conv0"], W["ln0"])
    return conv1_ln_relu(y0, W["conv1"], W["ln1"])


def subsample(mel: np.ndarray, W: dict) -> np.ndarray:
    """Stem plus ``input_proj_linear`` (no bias, no clamp): [T, hidden]."""
    return stem(mel, W) @ np.asarray(W["in_proj"], np.float64).T


# ------------------------------------------------------------------ tower pieces

def rms(x: np.ndarray, w: np.ndarray | None = None) -> np.ndarray:
    """RMS norm per row: x / sqrt(mean(x^2) + 1e-6), times the weight plainly."""
    y = x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + EPS)
    return y if w is None else y * np.asarray(w, np.float64)


def clip_lin(x: np.ndarray, W: np.ndarray, b=(-np.inf, np.inf, -np.inf, np.inf), fp8: bool = False) -> np.ndarray:
    """``ClipLin::apply`` (Gemma4ClippableLinear): clamp the input, x W^T
    (no bias), clamp the output. With ``fp8`` the clamped input is replaced by
    its e4m3 value at the input scale (``quantize_input``) and W is expected
    to hold the dequantised e4m3 rows (``e4m3_dequant_rows``)."""
    lo_in, hi_in, lo_out, hi_out = b
    xc = np.clip(x, lo_in, hi_in)
    if fp8:
        xc = quantize_input(xc, input_scale(b))
    y = xc @ np.asarray(W, np.float64).T
    return np.clip(y, lo_out, hi_out)


# ------------------------------------------------------------------ e4m3 projections
#
# The low-precision variant of the projections (the page keeps a quantized
# pack's kernels as an option, AudioTower::load with CMF_EGEMMA2_LOWMEM, but
# gives no format): OCP 8-bit floating point E4M3, per-row weight scales and
# an input scale fixed by the ClipLin input clamp. This arithmetic is the
# library's own definition of its AE_FP8 model, written out here plainly.

E4M3_MAX = 448.0


def e4m3_round(x) -> np.ndarray:
    """Nearest E4M3 value, ties to even, magnitudes beyond 448 saturated to
    448. E4M3: sign, 4 exponent bits with bias 7, 3 mantissa bits; normal
    values (1 + m/8) 2^(e-7) for e = 1..15 (the pattern e = 15, m = 7 is NaN,
    so the largest finite value is 1.75 x 2^8 = 448); subnormals m 2^-9.
    The grid spacing at |x| in [2^e, 2^(e+1)) is 2^(e-3) for e >= -6 and
    2^-9 below 2^-6."""
    x = np.asarray(x, np.float64)
    a = np.abs(x)
    _, ex = np.frexp(a)                       # a = f 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, -6)                # binade of a, subnormals share the lowest spacing
    q = np.ldexp(1.0, e - 3)
    r = np.minimum(np.round(a / q) * q, E4M3_MAX)   # np.round: half to even
    return np.copysign(r, x)


def e4m3_decode(codes) -> np.ndarray:
    """Values of E4M3 bit patterns (uint8): sign bit 7, exponent field e in
    bits 3-6, mantissa m in bits 0-2; e = 0 gives m 2^-9, otherwise
    (1 + m/8) 2^(e-7); e = 15 with m = 7 is NaN."""
    c = np.asarray(codes, np.uint8).astype(np.int64)
    e, m = (c >> 3) & 15, c & 7
    v = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, e - 7))
    v = np.where((e == 15) & (m == 7), np.nan, v)
    return np.where(c & 128, -v, v)


def linear_e4m3(x_codes, w_codes, cs, lo: float, hi: float, silu_q: tuple | None = None) -> np.ndarray:
    """One e4m3 projection by its definition: acc = x W^T over the decoded
    codes (float64), times cs per output column, clamped to [lo, hi]; with
    ``silu_q = (lo2, hi2, q)`` the output is e4m3_round(clamp(silu(v), lo2,
    hi2) q) instead (grid values)."""
    acc = e4m3_decode(x_codes) @ e4m3_decode(w_codes).T
    v = np.clip(acc * np.asarray(cs, np.float64)[None, :], lo, hi)
    if silu_q is None:
        return v
    lo2, hi2, q = silu_q
    return e4m3_round(np.clip(silu(v), lo2, hi2) * q)


def e4m3_rows(W) -> tuple[np.ndarray, np.ndarray]:
    """Per-row quantisation of a weight matrix [out, in]: s_n = max_k
    |W[n, k]| / 448 (1 for an all-zero row), values e4m3_round(W[n, k] / s_n)
    in float64. Returns (grid values, s)."""
    W = np.asarray(W, np.float64)
    amax = np.max(np.abs(W), axis=1) if W.size else np.zeros(W.shape[0])
    s = np.where(amax > 0, amax / E4M3_MAX, 1.0)
    return e4m3_round(W / s[:, None]), s


def e4m3_dequant_rows(W) -> np.ndarray:
    """The matrix the e4m3 model multiplies by: grid values times row scales."""
    v, s = e4m3_rows(W)
    return v * s[:, None]


def input_scale(b) -> float:
    """Scale of an e4m3 projection input clamped to [lo_in, hi_in]: 448 over
    the larger bound (the clamp maps onto the format's finite range)."""
    return E4M3_MAX / max(abs(float(b[0])), abs(float(b[1])))


def quantize_input(x, q: float) -> np.ndarray:
    """x replaced by e4m3_round(x q) / q."""
    return e4m3_round(np.asarray(x, np.float64) * q) / q


FP8_MATRICES = ("ff1.w1", "ff1.w2", "ff2.w1", "ff2.w2", "q", "k", "v", "lc_start")


def fp8_weights(W: dict) -> dict:
    """The e4m3 model's weights: a copy of W whose FP8_MATRICES are replaced
    by their dequantised e4m3 rows (the other matrices stay as given)."""
    out = dict(W)
    out["layers"] = []
    for ly in W["layers"]:
        d = dict(ly)
        for k in FP8_MATRICES:
            d[k] = e4m3_dequant_rows(ly[k])
        out["layers"].append(d)
    out["fp8"] = True
    return out


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def silu(x):
    """``silu_slice``: x * sigma(x)."""
    return x * sigmoid(x)


def softplus(x):
    """``AudioTower::load``: softplus as torch computes it, x > 20 passes
    through, otherwise ln(1 + e^x)."""
    x = np.asarray(x, np.float64)
    return np.where(x > 20.0, x, np.log1p(np.exp(np.minimum(x, 20.0))))


def sinusoids(hidden: int, n_dist: int) -> np.ndarray:
    """``AudioTower::load``: relative-distance sinusoids, row d =
    [sin(d inv_i) | cos(d inv_i)], inv_i = exp(-i ln(1e4) / (hidden/2 - 1))."""
    n_ts = hidden // 2
    incr = math.log(10000.0) / (max(n_ts, 2) - 1)
    inv = np.exp(-np.arange(n_ts, dtype=np.float64) * incr)
    d = np.arange(n_dist, dtype=np.float64)[:, None]
    return np.concatenate([np.sin(d * inv), np.cos(d * inv)], axis=1)


def relative_keys(relk: np.ndarray, left: int, hidden: int, chunk: int = 12, ctx_left: int = 13) -> np.ndarray:
    """R = pe relative_k_proj^T, rows for distances 0..left-1 (no clamp)."""
    n_dist = (chunk + ctx_left - 1) // 2 + 1
    pe = sinusoids(hidden, max(n_dist, left))
    return (pe @ np.asarray(relk, np.float64).T)[:left]


def q_scale_of(head_dim: int) -> float:
    """(1/sqrt(head_dim)) / ln 2 = log2(e)/sqrt(head_dim)."""
    return (head_dim ** -0.5) / math.log(2.0)


def k_scale_of() -> float:
    """ln(1 + e) / ln 2 = log2(1 + e)."""
    return math.log(1.0 + math.e) / math.log(2.0)


def layer_tables(ly: dict, shape: dict) -> dict:
    """Load-time tables of one layer: R and softplus(per_dim_scale)."""
    H = shape["hidden"]
    return {"R": relative_keys(ly["relk"], shape["left"], H),
            "qd": softplus(ly["pds"])}


def ffn(h: np.ndarray, ly: dict, f: str, bounds: dict, rw: float, fp8: bool = False) -> np.ndarray:
    """``ffn``: h + rw * rms_post(W2 silu(W1 rms_pre(h))), W1/W2 clippable."""
    a = rms(h, ly[f + ".pre"])
    u = silu(clip_lin(a, ly[f + ".w1"], bounds[f + ".w1"], fp8))
    y = clip_lin(u, ly[f + ".w2"], bounds[f + ".w2"], fp8)
    return h + rw * rms(y, ly[f + ".post"])


def local_attention_core(q: np.ndarray, k: np.ndarray, v: np.ndarray, pos: np.ndarray,
                         R: np.ndarray, qd: np.ndarray, heads: int, left: int,
                         cap: float) -> np.ndarray:
    """The attention core of ``attention`` on the clamped projections:
    q <- q * q_scale * softplus(pds)[j mod head_dim], k <- k * k_scale;
    for dist 0..min(pos, left-1): z = q.k_{t-dist} + q.R[dist] per head,
    z = cap tanh(z / cap), natural-exp softmax over the distances,
    o = sum_dist p v_{t-dist}. Inputs [T, hidden]; output [T, hidden]."""
    T, H = q.shape
    hd = H // heads
    qs = q * q_scale_of(hd) * np.tile(np.asarray(qd, np.float64), heads)[None, :]
    ks = k * k_scale_of()
    qh = qs.reshape(T, heads, hd)
    z = np.full((T, heads, left), -np.inf)
    for dist in range(left):
        ok = pos >= dist
        src = np.arange(T) - dist
        kk = np.zeros((T, heads, hd))
        kk[ok] = ks.reshape(T, heads, hd)[src[ok]]
        rr = R[dist].reshape(heads, hd)
        zz = (qh * kk).sum(-1) + (qh * rr[None]).sum(-1)
        zz = np.tanh(zz / cap) * cap
        z[ok, :, dist] = zz[ok]
    mx = z.max(axis=-1, keepdims=True)
    e = np.exp(z - mx)
    p = e / e.sum(axis=-1, keepdims=True)
    o = np.zeros((T, heads, hd))
    for dist in range(left):
        ok = pos >= dist
        src = np.arange(T) - dist
        vv = np.zeros((T, heads, hd))
        vv[ok] = v.reshape(T, heads, hd)[src[ok]]
        o += p[:, :, dist:dist + 1] * vv
    return o.reshape(T, H)


def attention(h: np.ndarray, pos: np.ndarray, ly: dict, tb: dict, bounds: dict,
              shape: dict, fp8: bool = False) -> np.ndarray:
    """Attention block: h + rms_post_attn(post(core(q, k, v of rms_pre_attn(h))))."""
    a = rms(h, ly["norm_pre_attn"])
    q = clip_lin(a, ly["q"], bounds["q"], fp8)
    k = clip_lin(a, ly["k"], bounds["k"], fp8)
    v = clip_lin(a, ly["v"], bounds["v"], fp8)
    o = local_attention_core(q, k, v, pos, tb["R"], tb["qd"], shape["heads"], shape["left"],
                             shape["softcap"])
    y = clip_lin(o, ly["post"], bounds["post"])
    return h + rms(y, ly["norm_post_attn"])


def glu(g: np.ndarray) -> np.ndarray:
    """``glu``: [n, 2d] -> [n, d], first half times sigma(second half)."""
    d = g.shape[1] // 2
    return g[:, :d] * sigmoid(g[:, d:])


def dwconv(x: np.ndarray, w: np.ndarray, pos: np.ndarray) -> np.ndarray:
    """``dwconv``: causal depthwise conv, tap k reads row t - (K-1-k), skipped
    where that reaches before the clip start (K-1-k > pos[t])."""
    T, d = x.shape
    K = w.shape[1]
    w = np.asarray(w, np.float64)
    out = np.zeros((T, d))
    for k in range(K):
        back = K - 1 - k
        ok = pos >= back
        src = np.arange(T) - back
        out[ok] += w[None, :, k] * x[src[ok]]
    return out


def light_conv(h: np.ndarray, pos: np.ndarray, ly: dict, bounds: dict, fp8: bool = False) -> np.ndarray:
    """Light conv block: h + lc_end(silu(rms_conv_norm(dwconv(glu(lc_start(
    rms_lc_pre(h))))))) (no norm on this residual)."""
    a = rms(h, ly["lc_pre"])
    g = clip_lin(a, ly["lc_start"], bounds["lc_start"], fp8)
    c = dwconv(glu(g), ly["lc_dw"], pos)
    c = silu(rms(c, ly["lc_norm"]))
    return h + clip_lin(c, ly["lc_end"], bounds["lc_end"])


def conformer_layer(h: np.ndarray, pos: np.ndarray, ly: dict, bounds: dict, shape: dict,
                    tb: dict | None = None, fp8: bool = False) -> np.ndarray:
    """One layer of ``encode_locked``: FFN1, attention, light conv, FFN2,
    RMS(norm_out). ``fp8``: the e4m3 model (ly from ``fp8_weights``)."""
    tb = layer_tables(ly, shape) if tb is None else tb
    rw = shape["residual_weight"]
    h = ffn(h, ly, "ff1", bounds, rw, fp8)
    h = attention(h, pos, ly, tb, bounds, shape, fp8)
    h = light_conv(h, pos, ly, bounds, fp8)
    h = ffn(h, ly, "ff2", bounds, rw, fp8)
    return rms(h, ly["norm_out"])


def head(h: np.ndarray, W: dict) -> np.ndarray:
    """``encode_locked`` tail: out_proj + bias, weightless RMS, embed_audio."""
    o = h @ np.asarray(W["out_proj"], np.float64).T + np.asarray(W["out_bias"], np.float64)
    return rms(o) @ np.asarray(W["embed"], np.float64).T


def positions(tokens_per_clip) -> np.ndarray:
    """Index of every packed row inside its clip."""
    return np.concatenate([np.arange(t) for t in tokens_per_clip]) if len(tokens_per_clip) \
        else np.zeros(0, np.int64)


def encode(clips: list, weights: dict, trace: bool = False, mels: list | None = None):
    """``encode_locked`` over packed clips: per-clip log-mel and stem, rows
    back to back, input projection, the layers, the head, split per clip.

    Returns a list of [T_i, embed_dim] arrays (and a dict of packed per-stage
    arrays when ``trace``)."""
    shape = weights["shape"]
    bank = mel_filter_bank()
    if mels is None:
        mels = [log_mel(c, bank) for c in clips]
    xs = [subsample(m, weights["stem"]) for m in mels]
    lens = [x.shape[0] for x in xs]
    T = sum(lens)
    tr = {"mels": mels}
    if T == 0:
        return ([np.zeros((0, shape["embed_dim"])) for _ in lens], tr) if trace else \
            [np.zeros((0, shape["embed_dim"])) for _ in lens]
    h = np.concatenate(xs, axis=0)
    pos = positions(lens)
    tr["subsample"] = h.copy()
    tr["layers"] = []
    fp8 = bool(weights.get("fp8", False))
    for ly, bd in zip(weights["layers"], weights["bounds"]):
        h = conformer_layer(h, pos, ly, bd, shape, fp8=fp8)
        if trace:
            tr["layers"].append(h.copy())
    e = head(h, weights["head"])
    out, off = [], 0
    for t in lens:
        out.append(e[off:off + t])
        off += t
    return (out, tr) if trace else out
