"""GPU parity of the LFM2A Conformer encoder (ae_lenc_*, include/ae.h) with its
float64 oracle (oracle/lfm_encoder.py), through the C ABI.

Inputs: spectrograms from the second front-end's oracle (the LFM2A log-mel,
normalised per band) of seeded noise-and-tone clips, and seeded random
weights (synth.lfm_encoder_weights; the matrices hold bf16 values, so both
sides multiply by the same numbers). The stem, one block and the whole body
are compared element by element at the library's bf16 bounds (max rel err
2e-2, cosine 0.999); clip lengths cover one token, the 128-row query and key
block edges and a ragged mix; the attention is per clip, so packing must not
change a clip's rows (bit for bit on the GPU)."""
import numpy as np
import pytest

import synth
from oracle import lfm as LF
from oracle import lfm_encoder as E
from tests.helpers import assert_bf16, dev, offsets, workspace

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import log_mel_front_b200 as ae  # noqa: E402


def _sync():
    torch.cuda.synchronize()
    assert ae.ae_device_status() == ae.AE_OK


def _mels(lengths, seed=31):
    out = []
    for i, n in enumerate(lengths):
        wave = synth.noise_tones_clip(n, seed, i)
        out.append(LF.features(wave).astype(np.float32))
    return out


@pytest.fixture(scope="module")
def w2():
    return synth.lfm_encoder_weights(n_layers=2)


@pytest.fixture(scope="module")
def m2(w2):
    m = ae.LencModel(w2)
    yield m
    m.close()


def _gpu_stem(m, mels):
    frames = [x.shape[0] for x in mels]
    toks = [ae.ae_lenc_num_tokens(f) for f in frames]
    off = offsets(frames)
    d_mel = dev(np.concatenate(mels)) if sum(frames) else torch.zeros(1, device="cuda")
    d_x = torch.full((max(sum(toks), 1), 512), float("nan"), device="cuda")
    ws = workspace(m.workspace_size(off))
    ae.ae_lenc_stem(m, d_mel, off, d_x, ws, ws.numel())
    _sync()
    return d_x[:sum(toks)].cpu().numpy(), toks


def _gpu_encode(m, mels, hidden=2048):
    frames = [x.shape[0] for x in mels]
    toks = [ae.ae_lenc_num_tokens(f) for f in frames]
    off = offsets(frames)
    d_mel = dev(np.concatenate(mels)) if sum(frames) else torch.zeros(1, device="cuda")
    d_out = torch.full((sum(toks) + 1, hidden), float("nan"), device="cuda")   # one sentinel row
    ws = workspace(m.workspace_size(off))
    ae.ae_lenc_encode(m, d_mel, off, d_out, ws, ws.numel())
    _sync()
    g = d_out.cpu().numpy()
    assert np.all(np.isnan(g[-1])), "rows written beyond the batch's token count"
    return g[:-1], toks


def test_token_counts_follow_the_stem():
    for F in (0, 1, 2, 7, 8, 9, 17, 3001):
        assert ae.ae_lenc_num_tokens(F) == E.stem_len(F)


def test_stem_matches_oracle(m2, w2):
    mels = _mels([16000, 2000, 47000])
    g, toks = _gpu_stem(m2, mels)
    o = np.concatenate([E.stem(x.astype(np.float64), w2) for x in mels])
    assert g.shape == o.shape == (sum(toks), 512)
    assert_bf16(g, o, "LFM2A stem")


def test_stem_work_item_edges(m2, w2):
    """The first stem kernel takes runs of 16 rows of its output per work item:
    clips of 1, 2, 63, 64, 65, 128 and 129 frames put the last run's edge on,
    before and after a multiple of 16 rows (and one clip is a single run)."""
    lens = [100, 160, 9920, 10080, 10240, 20320, 20480]
    mels = _mels(lens, seed=43)
    assert [x.shape[0] for x in mels] == [1, 2, 63, 64, 65, 128, 129]
    g, toks = _gpu_stem(m2, mels)
    o = np.concatenate([E.stem(x.astype(np.float64), w2) for x in mels])
    assert g.shape == o.shape == (sum(toks), 512)
    assert_bf16(g, o, "LFM2A stem at work-item edges")


def test_stem_mel_not_16_byte_aligned(m2):
    """With a mel base 4 bytes off a 16-byte boundary the first stem kernel
    stages its rows 4 bytes at a time instead of 16: the same rows."""
    mels = _mels([16000, 2000, 10240], seed=44)
    frames = [x.shape[0] for x in mels]
    toks = [ae.ae_lenc_num_tokens(f) for f in frames]
    off = offsets(frames)
    flat = np.concatenate(mels)
    outs = []
    for shift in (0, 1):
        base = torch.zeros(flat.size + 8, device="cuda")
        base[shift:shift + flat.size] = dev(flat.ravel())
        d_x = torch.full((sum(toks), 512), float("nan"), device="cuda")
        ws = workspace(m2.workspace_size(off))
        ae.ae_lenc_stem(m2, base[shift:shift + flat.size], off, d_x, ws, ws.numel())
        _sync()
        outs.append(d_x.cpu().numpy())
    assert np.all(np.isfinite(outs[0]))
    assert np.array_equal(outs[0], outs[1])


@pytest.mark.parametrize("toks", [[1], [5, 128, 129, 3], [300, 7, 256]])
def test_block_matches_oracle(m2, w2, toks):
    """One block from the same float32 input: the attention runs over whole clips
    (T = 1, clips ending on and just past a 128-row block, a ragged mix)."""
    rng = np.random.default_rng(sum(toks))
    x = rng.standard_normal((sum(toks), 512)).astype(np.float32)
    off = offsets(toks)
    d_x = dev(x)
    ws = workspace(m2.block_workspace_size(off))
    ae.ae_lenc_block(m2, 1, d_x, off, ws, ws.numel())
    _sync()
    g = d_x.cpu().numpy()
    o = []
    for i, t in enumerate(toks):
        xi = x[off[i]:off[i + 1]].astype(np.float64)
        o.append(E.block(xi, w2["layers"][1], E.relative_pos_emb(t, 512), w2["cfg"]))
    assert_bf16(g, np.concatenate(o), f"LFM2A block, clips of {toks} tokens")


def test_encode_matches_oracle_full_depth():
    """The whole body, 17 blocks and the adapter, on clips of 4 s and 9.5 s."""
    w = synth.lfm_encoder_weights()
    m = ae.LencModel(w)
    try:
        mels = _mels([64000, 152000], seed=37)
        g, toks = _gpu_encode(m, mels)
    finally:
        m.close()
    off = offsets(toks)
    assert np.all(np.isfinite(g))
    for i, x in enumerate(mels):
        o = E.encode(x.astype(np.float64), w)
        assert o.shape == (toks[i], 2048)
        assert_bf16(g[off[i]:off[i + 1]], o, f"LFM2A encode, clip {i} ({toks[i]} tokens, 17 blocks)")


def test_encode_edges_and_packing(m2, w2):
    """Clips with no tokens, one token and a ragged mix; each clip's rows equal
    the oracle's and equal those of the clip encoded alone, bit for bit."""
    lens = [100, 0, 16000, 2500, 33000]
    mels = [np.zeros((0, 128), np.float32) if n == 0 else x for n, x in zip(lens, _mels([max(n, 1) for n in lens]))]
    g, toks = _gpu_encode(m2, mels)
    off = offsets(toks)
    for i, x in enumerate(mels):
        o = E.encode(x.astype(np.float64), w2)
        assert g[off[i]:off[i + 1]].shape == o.shape
        if toks[i]:
            assert_bf16(g[off[i]:off[i + 1]], o, f"LFM2A encode, {toks[i]} tokens")
            alone, _ = _gpu_encode(m2, [x])
            assert np.array_equal(alone, g[off[i]:off[i + 1]])


def test_packed_batch_matches_single_clips(m2, w2):
    """Eight clips of 10-30 s packed into one call (2,376 tokens): every clip's
    rows equal the clip encoded alone, bit for bit, and two of them match the
    oracle."""
    lens = [480000] * 3 + [320000, 160000, 240000, 400000, 480000]
    mels = _mels(lens, seed=41)
    g, toks = _gpu_encode(m2, mels)
    assert sum(toks) >= 2048 and len(toks) >= 2
    off = offsets(toks)
    for i, x in enumerate(mels):
        alone, _ = _gpu_encode(m2, [x])
        assert np.array_equal(alone, g[off[i]:off[i + 1]]), f"clip {i} differs from the clip alone"
    for i in (3, 4):
        o = E.encode(mels[i].astype(np.float64), w2)
        assert_bf16(g[off[i]:off[i + 1]], o, f"LFM2A encode in a split batch, clip {i} ({toks[i]} tokens)")


def test_other_sizes_in_one_process():
    """Models of other sizes one after another in one process: conv module
    widths 4 (even: one tap of padding on the left, two on the right), 33 (the
    widest taken) and 1, with smaller FFN and adapter widths. The widths other
    than 9 take the generic depthwise kernel, whose shared memory grows with
    the width; the narrow model runs first."""
    lens = [64000, 2500, 20480]
    mels = _mels(lens, seed=47)
    for k, (n_ff, ad_ff, hidden) in ((4, (256, 512, 768)), (33, (512, 256, 512)), (1, (768, 1024, 256))):
        shape = dict(synth.LENC_SHAPE, n_layers=2, conv_k=k, n_ff=n_ff, adapter_ff=ad_ff, llm_hidden=hidden)
        w = synth.lfm_encoder_weights(shape=shape, seed=5100 + k)
        m = ae.LencModel(w)
        try:
            g, toks = _gpu_encode(m, mels, hidden=hidden)
        finally:
            m.close()
        off = offsets(toks)
        for i, x in enumerate(mels):
            o = E.encode(x.astype(np.float64), w)
            assert o.shape == (toks[i], hidden)
            assert_bf16(g[off[i]:off[i + 1]], o, f"LFM2A encode, conv_k {k}, n_ff {n_ff}, clip {i} ({toks[i]} tokens)")


def test_refusals(m2):
    off = offsets([16])
    with pytest.raises(ae.AEError) as e:
        ae.ae_lenc_encode(m2, torch.zeros(16 * 128, device="cuda"), off, torch.zeros((2, 2048), device="cuda"),
                          workspace(256), 16)
    assert e.value.status == ae.AE_EWORKSPACE
    with pytest.raises(ae.AEError) as e:
        ae.ae_lenc_block(m2, 2, torch.zeros((1, 512), device="cuda"), offsets([1]), workspace(1 << 20), 1 << 20)
    assert e.value.status == ae.AE_EINVAL
    with pytest.raises(ae.AEError) as e:   # more than 4096 rows after the stem
        big = 8 * 4096 + 1
        ae.ae_lenc_encode(m2, torch.zeros(1, device="cuda"), offsets([big]), torch.zeros(1, device="cuda"),
                          workspace(256), 256)
    assert e.value.status == ae.AE_EUNSUPPORTED
    _sync()
