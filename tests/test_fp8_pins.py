"""Pins of the oracle's e4m3 projection arithmetic (``oracle.e4m3_round`` ..
``oracle.fp8_weights``) to facts outside the oracle: torch's float8_e4m3fn
conversion (an implementation of the OCP 8-bit floating-point format), the
format's special values and value count, and exact rational arithmetic on
inputs that already lie on the grid."""
from fractions import Fraction

import numpy as np
import pytest

from oracle import oracle as O

torch = pytest.importorskip("torch")


def _torch_e4m3(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def _grid():
    """Every finite e4m3 value, decoded by torch from the 256 bit patterns."""
    v = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return np.unique(v[np.isfinite(v)])


def test_grid_has_the_format_value_count():
    g = _grid()
    pos = g[g >= 0]
    # 0, 7 subnormals, 15 binades x 8 mantissas minus the NaN pattern
    assert len(pos) == 127 and pos.max() == 448.0 and pos[1] == 2.0 ** -9
    assert np.array_equal(O.e4m3_round(g), g)


def test_rounding_matches_torch_on_grid_midpoints_and_random_values():
    g = _grid()
    pos = g[g >= 0]
    mids = (pos[:-1] + pos[1:]) / 2  # ties: to the even code
    r = np.random.default_rng(8)
    rand = r.standard_normal(200_000) * np.exp(r.uniform(-14, 6.1, 200_000))
    for x in (mids, -mids, rand.astype(np.float32).astype(np.float64)):
        x = x[np.abs(x) < 448]
        assert np.array_equal(O.e4m3_round(x), _torch_e4m3(x))


def test_special_values():
    R = O.e4m3_round
    assert R(448.0) == 448.0 and R(463.9) == 448.0  # below the 448/480 midpoint
    assert R(464.0) == 448.0 and R(1e6) == 448.0 and R(-1e6) == -448.0  # saturated, not infinite
    assert R(2.0 ** -9) == 2.0 ** -9 and R(2.0 ** -10) == 0.0  # tie between 0 and 2^-9: even is 0
    assert R(3 * 2.0 ** -10) == 2.0 ** -8  # tie between 1 and 2 steps: even is 2
    assert R(1.0 + 1 / 16) == 1.0 and R(1.0 + 3 / 16) == 1.25  # ties at mantissa 0/1 and 1/2 -> 0 and 2
    assert R(0.0) == 0.0 and np.signbit(R(-0.0))
    assert R(15.0 / 8 * 2 ** 7) == 240.0 and R(2.0 ** -6) == 2.0 ** -6


def test_row_quantisation_invariants():
    r = np.random.default_rng(3)
    W = r.standard_normal((64, 300)) * 0.02
    W[5] = 0.0
    W[7, 11] = -1.0  # a row whose largest magnitude is negative
    v, s = O.e4m3_rows(W)
    assert np.array_equal(O.e4m3_round(v), v)
    assert s[5] == 1.0 and not v[5].any()
    for n in range(64):
        if n == 5:
            continue
        k = np.argmax(np.abs(W[n]))
        assert abs(v[n, k]) == 448.0 and np.sign(v[n, k]) == np.sign(W[n, k])
    d = O.e4m3_dequant_rows(W)
    t = np.abs(W) / s[:, None]
    normal = t >= 2.0 ** -6
    assert np.all(np.abs(d - W)[normal] <= 2.0 ** -4 * np.abs(W)[normal] * (1 + 1e-12))
    assert np.all((np.abs(d - W) / s[:, None])[~normal] <= 2.0 ** -10 * (1 + 1e-12))


def test_input_scale_and_idempotence():
    assert O.input_scale((-8.0, 8.0, -1, 1)) == 56.0
    assert O.input_scale((-2.0, 4.0, -1, 1)) == 112.0
    x = np.random.default_rng(5).uniform(-8, 8, 5000)
    q = O.quantize_input(x, 56.0)
    assert np.array_equal(O.quantize_input(q, 56.0), q)
    assert np.max(np.abs(q)) <= 8.0
    assert np.all(np.abs(q - x) <= 2.0 ** -4 * np.abs(x) + 2.0 ** -10 / 56.0)


def test_fp8_clip_lin_is_the_exact_product_on_grid_inputs():
    """x on the input grid (code / q) and W rows of grid values times s: the
    quantisations are identities, so the result is the exact rational sum of
    code products times s / q."""
    r = np.random.default_rng(9)
    g = _grid()
    q = 56.0
    b = (-8.0, 8.0, -np.inf, np.inf)
    cx = r.choice(g, size=(3, 40))
    cw = r.choice(g, size=(5, 40))
    cw[:, 0] = 448.0  # every row's largest magnitude is 448, so s is exactly the row factor
    s = np.array([2.0 ** -9, 0.01, 1.0, 3.0, 2.0 ** 5])
    x = cx / q
    W = cw * s[:, None]
    got = O.clip_lin(x, O.e4m3_dequant_rows(W), b, fp8=True)
    for i in range(3):
        for n in range(5):
            acc = sum(Fraction(float(cx[i, k])) * Fraction(float(cw[n, k])) for k in range(40))
            want = acc * Fraction(float(O.e4m3_rows(W)[1][n])) / Fraction(q)
            assert abs(got[i, n] - float(want)) <= 1e-12 * max(1.0, abs(float(want)))


def test_fp8_weights_touch_only_the_e4m3_projections():
    import synth
    W = synth.model_weights("pr1", n_layers=1)
    F = O.fp8_weights(W)
    assert F["fp8"] and F["stem"] is W["stem"] and F["head"] is W["head"]
    for k, v in W["layers"][0].items():
        if k in O.FP8_MATRICES:
            vals, s = O.e4m3_rows(v)
            assert np.array_equal(F["layers"][0][k], vals * s[:, None])
            assert not np.array_equal(F["layers"][0][k], v)
        else:
            assert F["layers"][0][k] is v


def test_decode_matches_torch_bit_patterns():
    codes = np.arange(256, dtype=np.uint8)
    t = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    d = O.e4m3_decode(codes)
    assert np.array_equal(np.isnan(d), np.isnan(t)) and np.isnan(d).sum() == 2
    ok = ~np.isnan(t)
    assert np.array_equal(d[ok], t[ok])
    # encode . decode is the identity on the grid
    assert np.array_equal(O.e4m3_round(d[ok]), d[ok])


def test_linear_e4m3_against_integer_arithmetic():
    """Codes scaled by 2^9 are integers: the accumulator is an exact integer
    sum, checked with Python integers."""
    r = np.random.default_rng(21)
    finite = np.array([c for c in range(256) if c & 127 != 127], np.uint8)
    x = r.choice(finite, size=(4, 256))
    w = r.choice(finite, size=(3, 256))
    cs = np.array([1.0, 0.5, 2.0 ** -10])
    got = O.linear_e4m3(x, w, cs, -np.inf, np.inf)
    xi = np.rint(O.e4m3_decode(x) * 512).astype(np.int64)
    wi = np.rint(O.e4m3_decode(w) * 512).astype(np.int64)
    for i in range(4):
        for n in range(3):
            acc = sum(int(a) * int(b) for a, b in zip(xi[i], wi[n]))
            assert got[i, n] == float(Fraction(acc, 512 * 512) * Fraction(cs[n]))
    s = O.linear_e4m3(x, w, cs, -8.0, 8.0, silu_q=(-8.0, 8.0, 56.0))
    assert np.array_equal(O.e4m3_round(s), s) and np.max(np.abs(s)) <= 448.0


def test_rounding_is_odd_and_monotone():
    x = np.sort(np.random.default_rng(4).uniform(-500, 500, 100_000))
    r = O.e4m3_round(x)
    assert np.all(np.diff(r) >= 0)
    assert np.array_equal(O.e4m3_round(-x), -r)
