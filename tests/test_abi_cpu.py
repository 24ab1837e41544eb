"""The C-ABI library without a GPU: it loads, exports every symbol the header
declares, and its host-side logic (sizes, argument checks) behaves."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

from oracle import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ae():
    from log_mel_front_b200 import build
    build.build()
    import log_mel_front_b200 as m
    return m


def _header_symbols():
    src = open(os.path.join(ROOT, "include", "ae.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ae_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_symbol(ae):
    syms = _header_symbols()
    assert len(syms) >= 15
    lib = ctypes.CDLL(ae.LIB_PATH)
    for s in syms:
        assert hasattr(lib, s), s
    assert sorted(ae.EXPORTS) == syms


def test_sizes_match_the_page_table(ae):
    for line in open(os.path.join(ROOT, "tests", "golden", "token_counts.txt")):
        if line.strip() and not line.startswith("#"):
            n, f, t = map(int, line.split())
            assert ae.ae_num_frames(n) == f and ae.ae_num_tokens(n) == t, n


def test_sizes_match_the_oracle_on_random_lengths(ae):
    rng = np.random.default_rng(0)
    for n in list(range(0, 800)) + [int(x) for x in rng.integers(0, 700000, 2000)] + [-5]:
        assert ae.ae_num_frames(n) == O.num_frames(max(n, 0))
        assert ae.ae_num_tokens(n) == O.num_tokens(max(n, 0))


def test_workspace_sizes_are_monotone(ae):
    a = ae.ae_workspace_size(None, 1, 99, 25)
    b = ae.ae_workspace_size(None, 64, 64 * 2999, 64 * 750)
    assert 0 < a < b
    assert a % 256 == 0 and b % 256 == 0


def test_refusals_before_any_device_work(ae):
    # bad offsets are refused on the host, before the library touches CUDA
    with pytest.raises(ae.AEError) as e:
        ae.ae_logmel(0, [0, 100, 50], 0, 0, 1 << 20, stream=0)
    assert e.value.status == ae.AE_EINVAL and "non-decreasing" in str(e.value)
    with pytest.raises(ae.AEError) as e:
        ae.ae_logmel(0, [5, 100], 0, 0, 1 << 20, stream=0)
    assert e.value.status == ae.AE_EINVAL
    with pytest.raises(ae.AEError) as e:
        ae.ae_logmel(0, [0, 16000], 0, 0, 1 << 20, stream=0)   # null device pointers
    assert e.value.status == ae.AE_EINVAL
    with pytest.raises(ae.AEError) as e:
        ae.ae_local_attention(0, 0, 0, 1024, 1, 0, 0, 1.0, 50.0, [0, 10], 0, 1024, 0, 0, stream=0)
    assert e.value.status == ae.AE_EINVAL
    # an empty batch is legal and does nothing
    ae.ae_logmel(0, [0], 0, 0, 0, stream=0)
    # the bounded-wait self-test and the e4m3 projection check their arguments first
    for limit in (0, 1000001):
        with pytest.raises(ae.AEError) as e:
            ae.ae_selftest_bounded_wait(limit, stream=0)
        assert e.value.status == ae.AE_EINVAL
    for M, N, K in ((4, 256, 100), (4, 200, 128), (-1, 256, 128), (4, 256, 131072)):
        with pytest.raises(ae.AEError) as e:
            ae.ae_linear_e4m3(0, 0, 0, M, N, K, -8.0, 8.0, 0, stream=0)
        assert e.value.status == ae.AE_EINVAL
    ae.ae_linear_e4m3(0, 0, 0, 0, 256, 128, -8.0, 8.0, 0, stream=0)  # M = 0: nothing to do
    # the second front-end: unsupported shapes, bad offsets, over-wide bands
    for kw in (dict(n_fft=256), dict(hop=161), dict(win_length=600), dict(n_mels=129), dict(log_floor=0.0)):
        with pytest.raises(ae.AEError) as e:
            ae.ae_lfm_logmel(ae.lfm_config(**kw), 0, [0, 100], 0, 0, 1 << 20, stream=0)
        assert e.value.status == ae.AE_EUNSUPPORTED
    with pytest.raises(ae.AEError) as e:
        ae.ae_lfm_logmel(ae.lfm_config(), 0, [0, 100, 50], 0, 0, 1 << 20, stream=0)
    assert e.value.status == ae.AE_EINVAL
    with pytest.raises(ae.AEError) as e:  # 8 bands over 257 bins: far more than 16 bins a band
        ae.ae_lfm_logmel(ae.lfm_config(n_mels=8), 0, [0, 100], 0, 0, 1 << 20, stream=0)
    assert e.value.status == ae.AE_EUNSUPPORTED
    ae.ae_lfm_logmel(ae.lfm_config(), 0, [0, 0], 0, 0, 0, stream=0)  # no frames: nothing to do
    assert [ae.ae_lfm_num_frames(ae.lfm_config(), n) for n in (0, 1, 160, 48123)] == [0, 1, 2, 301]


def test_attention_tables_closed_form(ae):
    rng = np.random.default_rng(1)
    relk = (0.02 * rng.standard_normal((1024, 1024))).astype(np.float32)
    pds = (0.1 * rng.standard_normal(128)).astype(np.float32)
    R, qs, ks = ae.ae_attention_tables(relk, pds)
    assert abs(ks - math.log2(1 + math.e)) < 1e-6
    assert np.allclose(qs, O.q_scale_of(128) * O.softplus(pds), rtol=1e-6)
    assert np.allclose(R, O.relative_keys(relk, 12, 1024), rtol=1e-5, atol=1e-6)


def test_second_frontend_constants_in_sync_with_the_oracle(ae):
    """The library's default configuration of the second front-end equals the
    oracle's reading of the page's constants, field by field (the page names
    them without values, so both sides must take the same reading), and the
    two agree on frame counts."""
    from oracle import lfm as L
    c = ae.lfm_config()
    d = L.DEFAULTS
    assert (c.sample_rate, c.n_fft, c.win_length, c.hop, c.n_mels) == \
        (d["sample_rate"], d["n_fft"], d["win_length"], d["hop"], d["n_mels"])
    for f in ("preemph", "log_floor", "var_eps"):
        assert getattr(c, f) == np.float32(d[f]), f
    for n in (0, 1, 159, 160, 161, 16000, 480000, 480001):
        assert ae.ae_lfm_num_frames(c, n) == L.num_frames(n, d["hop"]), n


def test_second_frontend_refuses_a_zero_variance_epsilon(ae):
    """var_eps must be positive: with 0, a band whose frames are all equal (a
    silent clip) would be normalised by 0 / 0. The refusal is a host check
    (no GPU needed): the size helpers report the configuration invalid."""
    c = ae.lfm_config()
    assert ae.ae_lfm_num_frames(c, 16000) > 0
    c.var_eps = 0.0
    assert ae.ae_lfm_num_frames(c, 16000) == -1
    assert ae.ae_lfm_workspace_size(c, 4) == 0


def test_partition_refusals(ae):
    import numpy as np
    for off, parts in (([0, 100, 50], 2), ([0, 10], 0), ([0, 10], 70000), ([5, 10], 2)):
        with pytest.raises(ae.AEError) as e:
            ae.ae_partition_clips(np.array(off, np.int64), parts)
        assert e.value.status == ae.AE_EINVAL
