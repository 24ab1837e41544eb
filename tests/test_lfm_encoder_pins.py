"""Pins of the LFM2A encoder oracle (``oracle/lfm_encoder.py``) to facts
outside itself, on the CPU: brute-force convolutions on tiny inputs, the
stem's geometry and flatten, the position table's closed form, the attention
against torch's scaled_dot_product_attention where the position terms
vanish, the direction of the relative shift, GELU against math.erf,
LayerNorm's moments, the depthwise conv's impulse response and the macaron
half weight (cera 0.5.3, audio_encoder_gpu.rs)."""
import math

import numpy as np
import pytest
import torch

from oracle import lfm_encoder as E


def _conv_brute(x, w, b, stride, pad, groups):
    cin, H, W = x.shape
    cout, cpg, kh, kw = w.shape
    ho, wo = (H + 2 * pad - kh) // stride + 1, (W + 2 * pad - kw) // stride + 1
    opg = cout // groups
    out = np.zeros((cout, ho, wo))
    for o in range(cout):
        g = o // opg
        for i in range(ho):
            for j in range(wo):
                acc = b[o]
                for c in range(cpg):
                    for dh in range(kh):
                        for dw in range(kw):
                            r, s = i * stride + dh - pad, j * stride + dw - pad
                            if 0 <= r < H and 0 <= s < W:
                                acc += w[o, c, dh, dw] * x[g * cpg + c, r, s]
                out[o, i, j] = acc
    return out


@pytest.mark.parametrize("groups,stride,pad,k", [(1, 2, 1, 3), (4, 2, 1, 3), (1, 1, 0, 1)])
def test_conv2d_matches_brute_force(groups, stride, pad, k):
    rng = np.random.default_rng(groups * 10 + stride)
    cin = 4
    x = rng.standard_normal((cin, 7, 6))
    w = rng.standard_normal((4, cin // groups, k, k))
    b = rng.standard_normal(4)
    got = E.conv2d(x, w, b, stride, pad, groups)
    assert np.allclose(got, _conv_brute(x, w, b, stride, pad, groups), rtol=0, atol=1e-12)


def _tiny_stem(rng, ch=4, d=8):
    W = {}
    cin = 1
    for i, (dw, _, _, k) in enumerate(E.STEM_MODES):
        W[f"stem{i}.w"] = rng.standard_normal((ch, 1 if dw else cin, k, k)) * 0.5
        W[f"stem{i}.b"] = rng.standard_normal(ch) * 0.1
        cin = ch
    W["pre_w"] = rng.standard_normal((d, ch * 16)) * 0.1
    W["pre_b"] = rng.standard_normal(d) * 0.1
    return W


def test_stem_geometry_and_flatten():
    rng = np.random.default_rng(5)
    W = _tiny_stem(rng)
    for F in (1, 2, 7, 8, 9, 23):
        mel = rng.standard_normal((F, 128))
        want_t = -(-(-(-(-(-F // 2)) // 2)) // 2)
        assert E.stem_len(F) == want_t
        assert E.stem(mel, W).shape == (want_t, 8)
    # the flatten is (time, channel * 16 + freq): a pre_encode_out row that
    # picks (channel 2, freq 5) returns that stem feature
    mel = rng.standard_normal((40, 128))
    x = mel[None]
    for i, (dw, stride, pad, _) in enumerate(E.STEM_MODES):
        x = _conv_brute(x, W[f"stem{i}.w"], W[f"stem{i}.b"], stride, pad, x.shape[0] if dw else 1)
        if E.STEM_RELU[i]:
            x = np.maximum(x, 0.0)
    pick = dict(W, pre_w=np.zeros((1, 64)), pre_b=np.zeros(1))
    pick["pre_w"][0, 2 * 16 + 5] = 1.0
    assert np.allclose(E.stem(mel, pick)[:, 0], x[2, :, 5], rtol=0, atol=1e-12)


def test_relative_position_table_closed_form():
    t, d = 5, 8
    pe = E.relative_pos_emb(t, d)
    assert pe.shape == (2 * t - 1, d)
    assert np.allclose(pe[t - 1], [0, 1] * (d // 2), atol=0)          # relative position 0
    for r in (0, 3, 8):
        p = t - 1 - r
        for i in range(d // 2):
            w = 10000.0 ** (-2 * i / d)
            assert abs(pe[r, 2 * i] - math.sin(p * w)) < 1e-15 and abs(pe[r, 2 * i + 1] - math.cos(p * w)) < 1e-15


def test_attention_without_position_terms_is_plain_attention():
    rng = np.random.default_rng(9)
    t, heads, hd = 11, 2, 4
    q, k, v = (rng.standard_normal((t, heads * hd)) for _ in range(3))
    p = np.zeros((2 * t - 1, heads * hd))
    got = E.xl_attention(q, k, v, p, np.zeros(heads * hd), np.zeros(heads * hd), heads)
    th = lambda a: torch.from_numpy(a.reshape(t, heads, hd).transpose(1, 0, 2).copy())
    want = torch.nn.functional.scaled_dot_product_attention(th(q), th(k), th(v)).numpy().transpose(1, 0, 2)
    assert np.allclose(got, want.reshape(t, heads * hd), rtol=0, atol=1e-12)
    # bias_u adds (bias_u . k_j) to every query's score of key j
    bu = rng.standard_normal(heads * hd)
    got_u = E.xl_attention(q, k, v, p, bu, np.zeros(heads * hd), heads)
    want_u = torch.nn.functional.scaled_dot_product_attention(th(q + bu), th(k), th(v)).numpy().transpose(1, 0, 2)
    assert np.allclose(got_u, want_u.reshape(t, heads * hd), rtol=0, atol=1e-12)


@pytest.mark.parametrize("dist", [0, 1, -2])
def test_relative_shift_direction(dist):
    """With k = 0 the scores come from the position rows alone. A table whose
    only nonzero row is relative distance i - j = dist, large along q + bias_v,
    makes query i attend to key i - dist alone, so the output is v_{i - dist}
    wherever that key exists (and a plain mean where it does not)."""
    t, heads, hd = 9, 1, 4
    rng = np.random.default_rng(3)
    q = np.zeros((t, hd))
    bv = np.array([1.0, 0.0, 0.0, 0.0])
    v = rng.standard_normal((t, hd))
    p = np.zeros((2 * t - 1, hd))
    p[t - 1 - dist, 0] = 400.0                 # row of relative distance dist
    out = E.xl_attention(q, np.zeros((t, hd)), v, p, np.zeros(hd), bv, heads)
    for i in range(t):
        j = i - dist
        if 0 <= j < t:
            assert np.allclose(out[i], v[j], rtol=0, atol=1e-9), (i, j)
        else:
            assert np.allclose(out[i], v.mean(0), rtol=0, atol=1e-9), i


def test_gelu_is_the_erf_form():
    for x in (-3.0, -0.7, 0.0, 0.3, 1.0, 2.5):
        want = 0.5 * x * (1.0 + math.erf(x / math.sqrt(2.0)))
        assert abs(E.gelu_erf(np.array([x]))[0] - want) < 1e-15
    # differs from the tanh approximation
    x = 1.0
    tanh_form = 0.5 * x * (1 + math.tanh(math.sqrt(2 / math.pi) * (x + 0.044715 * x ** 3)))
    assert abs(E.gelu_erf(np.array([x]))[0] - tanh_form) > 1e-5


def test_layer_norm_moments_and_affine():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((3, 32)) * 5 + 2
    y = E.layer_norm(x, np.ones(32), np.zeros(32), 1e-5)
    assert np.allclose(y.mean(1), 0, atol=1e-12)
    assert np.allclose((y ** 2).mean(1), x.var(1) / (x.var(1) + 1e-5), rtol=1e-12)
    w, b = rng.standard_normal(32), rng.standard_normal(32)
    assert np.allclose(E.layer_norm(x, w, b, 1e-5), y * w + b, atol=1e-12)


@pytest.mark.parametrize("k", [9, 4])
def test_depthwise_conv_impulse_response(k):
    rng = np.random.default_rng(k)
    t, C = 20, 3
    w = rng.standard_normal((k, C))
    x = np.zeros((t, C))
    t0 = 10
    x[t0, 1] = 1.0
    y = E.depthwise_conv1d(x, w, np.zeros(C))
    lo = (k - 1) // 2
    want = np.zeros((t, C))
    for m in range(k):
        want[t0 + lo - m, 1] = w[m, 1]         # y[i] = sum_m w[m] x[i + m - lo]
    assert np.allclose(y, want, rtol=0, atol=0)
    # a clip edge: an impulse in the first row reaches back only k - 1 - lo rows after it
    x = np.zeros((t, C))
    x[0, 0] = 1.0
    y = E.depthwise_conv1d(x, w, np.zeros(C))
    assert np.allclose(y[:lo + 1, 0], w[lo::-1, 0]) and np.all(y[lo + 1:, 0] == 0)


def test_macaron_ffn_half_weight():
    rng = np.random.default_rng(6)
    d, f = 8, 16
    ly = {"ffn1.norm_w": np.ones(d), "ffn1.norm_b": np.zeros(d), "ffn1.up_w": np.zeros((f, d)),
          "ffn1.up_b": np.zeros(f), "ffn1.down_w": rng.standard_normal((d, f)), "ffn1.down_b": rng.standard_normal(d)}
    x = rng.standard_normal((4, d))
    # silu(0) = 0, so the block adds half the down bias
    assert np.allclose(E.macaron_ffn(x, ly, "ffn1", 1e-5), x + 0.5 * ly["ffn1.down_b"], atol=1e-12)
