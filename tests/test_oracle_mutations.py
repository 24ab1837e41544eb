"""The pins catch plausible mistakes. Each case plants one mistake in the
oracle on the CPU (one of its functions or constants is replaced for the
duration of the case) and checks that at least one of the pins written
against it fails. A mutant that every listed pin accepts would mean the pins
cannot tell that mistake from the definition."""
import math

import numpy as np
import pytest

from oracle import lfm as LF
from oracle import lfm_encoder as LE
from oracle import oracle as O
from oracle import resample as RS
from tests import test_fp8_pins as P8
from tests import test_lfm_encoder_pins as PE
from tests import test_lfm_pins as PL
from tests import test_oracle_pins as P
from tests import test_resample_pins as PR


def _symmetric_hann(n=O.FRAME):
    return 0.5 - 0.5 * np.cos(2.0 * np.pi * np.arange(n) / (n - 1))


def _wrap(name, fn):
    orig = getattr(O, name)
    return lambda *a, **k: fn(orig, *a, **k)


MUTANTS = {
    # counts
    "frame count floors instead of ceiling": (
        O, "num_frames", lambda: (lambda n: 0 if min(n, O.MAX_SAMPLES) <= O.HOP
                                  else (min(n, O.MAX_SAMPLES) - O.HOP) // O.HOP),
        [P.test_token_counts_match_the_page_table, P.test_frame_count_closed_form_matches_enumeration]),
    # window, log-mel
    "symmetric Hann window": (
        O, "hann_periodic", lambda: _symmetric_hann, [P.test_hann_periodic_closed_form]),
    "log10 instead of ln": (
        O, "log_mel", lambda: _wrap("log_mel", lambda f, *a, **k: f(*a, **k) / math.log(10.0)),
        [P.test_silence_is_the_mel_floor]),
    "mel floor 1e-6 instead of 1e-3": (
        O, "log_mel", lambda: _wrap("log_mel", lambda f, *a, **k: np.log(np.exp(f(*a, **k)) - 1e-3 + 1e-6)),
        [P.test_silence_is_the_mel_floor]),
    # norms, projections, constants
    "RMS norm weight 1 + w": (
        O, "rms", lambda: (lambda x, w=None: x / np.sqrt((x * x).mean(-1, keepdims=True) + O.EPS)
                           * (1.0 if w is None else 1.0 + np.asarray(w))),
        [P.test_rms_norm_invariants]),
    "RMS norm without epsilon": (
        O, "rms", lambda: (lambda x, w=None: x / np.sqrt(np.maximum((x * x).mean(-1, keepdims=True), 1e-300))
                           * (1.0 if w is None else np.asarray(w))),
        [P.test_rms_norm_invariants]),
    "ClipLin without its input clamp": (
        O, "clip_lin", lambda: _wrap("clip_lin", lambda f, x, W, b=(-np.inf, np.inf, -np.inf, np.inf), fp8=False:
                                     f(x, W, (-np.inf, np.inf, b[2], b[3]), fp8)),
        [P.test_matrix_product_matches_triple_loop_and_clamps]),
    "k scale log2(e) instead of log2(1 + e)": (
        O, "k_scale_of", lambda: (lambda: math.log2(math.e)), [P.test_scalar_constants_closed_form]),
    "softplus threshold applied at >= 20": (
        O, "softplus", lambda: (lambda x: np.where(np.asarray(x, np.float64) >= 20.0, np.asarray(x, np.float64),
                                                   np.log1p(np.exp(np.minimum(np.asarray(x, np.float64), 20.0))))),
        [P.test_scalar_constants_closed_form]),
    # attention
    "attention window of 11": (
        O, "local_attention_core", lambda: _wrap("local_attention_core",
                                                 lambda f, q, k, v, pos, R, qd, heads, left, cap:
                                                 f(q, k, v, pos, R, qd, heads, left - 1, cap)),
        [P.test_attention_mask_is_causal_width_12_per_clip, P.test_attention_with_zero_query_is_window_mean]),
    "no soft cap": (
        O, "local_attention_core", lambda: _wrap("local_attention_core",
                                                 lambda f, q, k, v, pos, R, qd, heads, left, cap:
                                                 f(q, k, v, pos, R, qd, heads, left, 1e30)),
        [P.test_attention_two_token_hand_computation]),
    # light conv
    "GLU halves swapped": (
        O, "glu", lambda: (lambda g: g[:, g.shape[1] // 2:] * O.sigmoid(g[:, :g.shape[1] // 2])),
        [P.test_glu_closed_form]),
    "depthwise taps reversed": (
        O, "dwconv", lambda: _wrap("dwconv", lambda f, x, w, pos: f(x, np.asarray(w)[:, ::-1], pos)),
        [P.test_dwconv_impulse_response_and_clip_start]),
    # stem projection and head (encode_locked)
    "in_proj applied transposed": (
        O, "subsample", lambda: (lambda mel, W: O.stem(mel, W) @ np.asarray(W["in_proj"], np.float64)),
        [P.test_in_proj_rows_are_output_features]),
    "head without out_bias": (
        O, "head", lambda: (lambda h, W: O.rms(h @ np.asarray(W["out_proj"], np.float64).T)
                            @ np.asarray(W["embed"], np.float64).T),
        [P.test_head_hand_computation, P.test_head_norm_is_weightless_and_scale_invariant]),
    "head without the weightless RMS norm": (
        O, "head", lambda: (lambda h, W: (h @ np.asarray(W["out_proj"], np.float64).T
                                          + np.asarray(W["out_bias"], np.float64))
                            @ np.asarray(W["embed"], np.float64).T),
        [P.test_head_hand_computation, P.test_head_norm_is_weightless_and_scale_invariant]),
    "head RMS norm with 1e-3 instead of 1e-6": (
        O, "head", lambda: (lambda h, W: ((lambda o: o / np.sqrt((o * o).mean(-1, keepdims=True) + 1e-3))(
            h @ np.asarray(W["out_proj"], np.float64).T + np.asarray(W["out_bias"], np.float64)))
                            @ np.asarray(W["embed"], np.float64).T),
        [P.test_head_hand_computation]),
    # layer composition
    "FFN half-residual ignored": (
        O, "ffn", lambda: _wrap("ffn", lambda f, h, ly, name, bounds, rw, fp8=False: f(h, ly, name, bounds, 1.0, fp8)),
        [P.test_layer_matches_scalar_restatement]),
}

MODULE_MUTANTS = {
    "e4m3 ties rounded away from zero": (
        O, "e4m3_round", lambda: (lambda x: _e4m3_half_up(x)),
        [P8.test_rounding_matches_torch_on_grid_midpoints_and_random_values, P8.test_special_values]),
    "e4m3 row scale amax / 240": (
        O, "e4m3_rows", lambda: (lambda W: _rows_240(W)), [P8.test_row_quantisation_invariants]),
    "resampler roll-off 0.9": (
        RS, "RS_ROLLOFF", lambda: 0.9, [lambda: PR.test_cutoff_and_transition_band_follow_the_kaiser_window(48000)]),
    "resampler Kaiser beta 8.6": (
        RS, "RS_BETA", lambda: 8.6, [lambda: PR.test_cutoff_and_transition_band_follow_the_kaiser_window(48000)]),
    "Slaney scale replaced by HTK": (
        LF, "hz_to_mel_slaney", lambda: (lambda f: 2595.0 * np.log10(1.0 + np.asarray(f, np.float64) / 700.0)),
        [PL.test_slaney_scale_closed_forms]),
    "second front-end without pre-emphasis": (
        LF, "DEFAULTS", lambda: dict(LF.DEFAULTS, preemph=0.0), [lambda: PL.test_frame_count_and_power_match_torch_stft(400)]),
    # LFM2A encoder body
    "XL relative shift reversed (p row t-1+i-j)": (
        LE, "xl_attention", lambda: (lambda q, k, v, p, bu, bv, heads:
                                     LE_ORIG["xl_attention"](q, k, v, p[::-1].copy(), bu, bv, heads)),
        [lambda: PE.test_relative_shift_direction(1)]),
    "macaron FFN at full weight": (
        LE, "macaron_ffn", lambda: (lambda x, ly, f, eps: 2.0 * LE_ORIG["macaron_ffn"](x, ly, f, eps) - x),
        [PE.test_macaron_ffn_half_weight]),
    "GELU in its tanh form": (
        LE, "gelu_erf", lambda: (lambda x: 0.5 * np.asarray(x) * (1 + np.tanh(math.sqrt(2 / math.pi) *
                                                                             (np.asarray(x) + 0.044715 * np.asarray(x) ** 3)))),
        [PE.test_gelu_is_the_erf_form]),
    "stem flattened frequency-major": (
        LE, "stem", lambda: (lambda mel, W: _stem_freq_major(mel, W)), [PE.test_stem_geometry_and_flatten]),
    "depthwise conv made causal": (
        LE, "depthwise_conv1d", lambda: (lambda x, w, b: _causal_dw(x, w, b)),
        [lambda: PE.test_depthwise_conv_impulse_response(9)]),
}


LE_ORIG = {"xl_attention": LE.xl_attention, "macaron_ffn": LE.macaron_ffn}


def _stem_freq_major(mel, W):
    x = np.asarray(mel, np.float64)[None]
    for i, (dw, stride, pad, k) in enumerate(LE.STEM_MODES):
        x = LE.conv2d(x, W[f"stem{i}.w"], W[f"stem{i}.b"], stride, pad, x.shape[0] if dw else 1)
        if LE.STEM_RELU[i]:
            x = np.maximum(x, 0.0)
    c, t, f = x.shape
    flat = x.transpose(1, 2, 0).reshape(t, f * c)
    return flat @ np.asarray(W["pre_w"], np.float64).T + np.asarray(W["pre_b"], np.float64)


def _causal_dw(x, w, b):
    x, w = np.asarray(x, np.float64), np.asarray(w, np.float64)
    t, C = x.shape
    k = w.shape[0]
    xp = np.zeros((t + k - 1, C))
    xp[k - 1:] = x
    y = np.zeros((t, C))
    for m in range(k):
        y += w[m][None, :] * xp[m:m + t]
    return y + np.asarray(b, np.float64)[None, :]


def _e4m3_half_up(x):
    x = np.asarray(x, np.float64)
    a = np.abs(x)
    _, ex = np.frexp(a)
    q = np.ldexp(1.0, np.maximum(ex - 1, -6) - 3)
    return np.copysign(np.minimum(np.floor(a / q + 0.5) * q, 448.0), x)


def _rows_240(W):
    W = np.asarray(W, np.float64)
    amax = np.max(np.abs(W), axis=1)
    s = np.where(amax > 0, amax / 240.0, 1.0)
    return O.e4m3_round(W / s[:, None]), s


def _caught(pins):
    for pin in pins:
        try:
            pin()
        except AssertionError:
            return True
    return False


@pytest.mark.parametrize("name", sorted(MUTANTS) + sorted(MODULE_MUTANTS))
def test_pins_catch_the_planted_mistake(name, monkeypatch):
    mod, attr, make, pins = {**MUTANTS, **MODULE_MUTANTS}[name]
    monkeypatch.setattr(mod, attr, make())
    assert _caught(pins), f"no pin caught: {name}"


def test_pins_pass_on_the_unmutated_oracle():
    """The same pins accept the oracle as committed (the cases above are not
    failing for a reason of their own)."""
    for _, (_, _, _, pins) in {**MUTANTS, **MODULE_MUTANTS}.items():
        assert not _caught(pins)
