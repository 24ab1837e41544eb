"""Parity of the CUDA library (through its C ABI) with the float64 oracle.

Every case runs the library on seeded synthetic inputs from ``synth`` and
compares it element by element with the oracle on the same inputs, within
the tolerances of ``helpers``. Full-size workloads run in the launch
configuration the bench times; where the oracle cannot finish the whole
batch in seconds, it checks a seeded sample of clips (every clip's output
depends on that clip alone) or of tokens.
"""
import math

import numpy as np
import pytest

import synth
from oracle import oracle as O
from tests.helpers import (LOGMEL_ABS, assert_bf16, assert_f32, assert_logmel, dev, offsets, rel_err, cosine,
                           workspace)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import log_mel_front_b200 as ae  # noqa: E402


def _sync():
    torch.cuda.synchronize()
    assert ae.ae_device_status() == ae.AE_OK


# ------------------------------------------------------------------ fixtures

@pytest.fixture(scope="module")
def w_pr1():
    return synth.model_weights("pr1")


@pytest.fixture(scope="module")
def m_pr1(w_pr1):
    m = ae.Model(w_pr1, ae.AE_F32)
    yield m
    m.close()


@pytest.fixture(scope="module")
def w_tower():
    return synth.model_weights("tower")


@pytest.fixture(scope="module")
def m_tower(w_tower):
    m = ae.Model(w_tower, ae.AE_BF16)
    yield m
    m.close()


def gpu_logmel(clips):
    flat, off = synth.pack(clips)
    frames = sum(O.num_frames(len(c)) for c in clips)
    d_wave = dev(flat if len(flat) else np.zeros(1, np.float32))
    d_mel = torch.full((max(frames, 1), 128), float("nan"), device="cuda")
    nb = ae.ae_workspace_size(None, len(clips), frames, 0)
    ws = workspace(nb)
    ae.ae_logmel(d_wave, off, d_mel, ws, ws.numel())
    _sync()
    return d_mel[:frames].cpu().numpy()


def gpu_encode(model, clips, embed_dim=512):
    flat, off = synth.pack(clips)
    frames = sum(O.num_frames(len(c)) for c in clips)
    toks = sum(O.num_tokens(len(c)) for c in clips)
    d_wave = dev(flat)
    d_out = torch.full((toks + 1, embed_dim), float("nan"), device="cuda")   # one sentinel row
    nb = model.workspace_size(len(clips), frames, toks)
    ws = workspace(nb)
    ae.ae_encode(model, d_wave, off, d_out, ws, ws.numel())
    _sync()
    g = d_out.cpu().numpy()
    assert np.all(np.isnan(g[toks])), "rows written beyond the batch's token count"
    return g[:toks], offsets([O.num_tokens(len(c)) for c in clips])


# ------------------------------------------------------------------ log-mel

def test_logmel_pr1_clip():
    wave = synth.pr1_wave()
    g = gpu_logmel([wave])
    o = O.log_mel(wave)
    assert g.shape == (99, 128)
    assert_logmel(g, o, "log-mel pr1")


def test_logmel_edge_lengths_packed():
    rng = np.random.default_rng(7)
    lens = [0, 100, 160, 161, 321, 480, 1000, 16000, 72825, 1234, 480001]
    clips = [(0.3 * rng.standard_normal(n)).astype(np.float32) for n in lens]
    clips[7] = np.zeros(16000, np.float32)  # silence
    g = gpu_logmel(clips)
    frames = [O.num_frames(n) for n in lens]
    assert g.shape[0] == sum(frames)
    off = offsets(frames)
    for i, c in enumerate(clips):
        o = O.log_mel(c)
        gi = g[off[i]:off[i + 1]]
        assert gi.shape == o.shape
        if len(o):
            assert_logmel(gi, o, f"log-mel clip of {lens[i]} samples")
    sil = g[off[7]:off[8]]
    assert np.max(np.abs(sil - math.log(1e-3))) < 1e-6


def test_logmel_same_clip_at_every_sample_alignment():
    # the staging copies 16 bytes at a time where a clip starts on a 16-byte
    # boundary and 4 bytes at a time elsewhere: the same clip placed at the four
    # offsets mod 4 (one-sample spacer clips between) gives the same rows
    rng = np.random.default_rng(11)
    c = (0.3 * rng.standard_normal(7776)).astype(np.float32)
    one = np.array([0.25], np.float32)
    g = gpu_logmel([c, one, c, one, c, one, c])
    n, n1 = O.num_frames(len(c)), O.num_frames(1)
    starts = [k * (n + n1) for k in range(4)]
    for s0 in starts[1:]:
        assert np.array_equal(g[s0:s0 + n], g[:n])
    assert_logmel(g[:n], O.log_mel(c), "log-mel 7776-sample clip")


def test_logmel_tone_band():
    t = np.arange(16000) / 16000
    wave = (0.5 * np.sin(2 * np.pi * 1000.0 * t)).astype(np.float32)
    g = gpu_logmel([wave])
    best = int(np.argmax(g[g.shape[0] // 2]))
    m = 2595 * np.log10(1 + 8000 / 700) * (best + 1) / 129
    assert abs(700 * (10 ** (m / 2595) - 1) - 1000.0) < 60.0


def test_logmel_frontend_workload_full():
    clips = synth.waves("frontend")
    g = gpu_logmel(clips)
    assert g.shape == (64 * 2999, 128)
    for i, c in enumerate(clips):
        o = O.log_mel(c)
        assert_logmel(g[i * 2999:(i + 1) * 2999], o, f"log-mel frontend clip {i}")


# ------------------------------------------------------------------ stem

def _stem_case(model, W, clips, bf16):
    mels = [O.log_mel(c) for c in clips]
    frames = [m.shape[0] for m in mels]
    toks = [O.num_tokens(len(c)) for c in clips]
    T = sum(toks)
    d_mel = dev(np.concatenate(mels).astype(np.float32))
    d_h = torch.full((max(T, 1), 1024), float("nan"), device="cuda")
    ws = workspace(model.workspace_size(len(clips), sum(frames), T))
    ae.ae_subsample(model, d_mel, offsets(frames), d_h, ws, ws.numel())
    _sync()
    g = d_h[:T].cpu().numpy()
    # the oracle starts from the same float32 mel the GPU got
    o = np.concatenate([O.subsample(m.astype(np.float32).astype(np.float64), W["stem"]) for m in mels])
    return g, o


def test_subsample_f32_pr1(m_pr1, w_pr1):
    g, o = _stem_case(m_pr1, w_pr1, [synth.pr1_wave()], False)
    assert g.shape == (25, 1024)
    assert_f32(g, o, "subsample f32")


def test_subsample_bf16_ragged(m_tower, w_tower):
    rng = np.random.default_rng(3)
    clips = [(0.3 * rng.standard_normal(n)).astype(np.float32) for n in (16000, 161, 5000, 33333)]
    g, o = _stem_case(m_tower, w_tower, clips, True)
    assert_bf16(g, o, "subsample bf16")


def test_subsample_bf16_mel_not_16_byte_aligned(m_tower, w_tower):
    """d_mel 4 bytes past a 16-byte boundary (allowed by ae_subsample): the
    tensor-core conv0 stages its mel rows with 4-byte copies instead of
    16-byte ones; same rows as the aligned call, bit for bit, and the oracle's."""
    rng = np.random.default_rng(5)
    clips = [(0.3 * rng.standard_normal(n)).astype(np.float32) for n in (16000, 7000, 48000)]
    mels = [O.log_mel(c) for c in clips]
    frames = [m.shape[0] for m in mels]
    T = sum(O.num_tokens(len(c)) for c in clips)
    flat = np.concatenate(mels).astype(np.float32)
    base = torch.zeros(flat.size + 4, device="cuda")
    base[1:1 + flat.size] = torch.from_numpy(flat.ravel()).cuda()
    d_mis = base[1:1 + flat.size]
    assert d_mis.data_ptr() % 16 == 4
    ws = workspace(m_tower.workspace_size(len(clips), sum(frames), T))
    outs = []
    for d_mel in (dev(flat), d_mis):
        d_h = torch.full((T, 1024), float("nan"), device="cuda")
        ae.ae_subsample(m_tower, d_mel, offsets(frames), d_h, ws, ws.numel())
        _sync()
        outs.append(d_h.cpu().numpy())
    assert np.array_equal(outs[0], outs[1])
    o = np.concatenate([O.subsample(m.astype(np.float32).astype(np.float64), w_tower["stem"]) for m in mels])
    assert_bf16(outs[1], o, "subsample bf16, unaligned mel")


# ------------------------------------------------------------------ one layer

def _layer_case(model, W, layer, h, toks):
    T = sum(toks)
    d_h = dev(h.astype(np.float32))
    ws = workspace(model.workspace_size(len(toks), 0, T))
    ae.ae_conformer_layer(model, layer, d_h, offsets(toks), ws, ws.numel())
    _sync()
    g = d_h.cpu().numpy()
    o = O.conformer_layer(h.astype(np.float32).astype(np.float64), O.positions(toks), W["layers"][layer],
                          W["bounds"][layer], W["shape"])
    return g, o


def test_layer_f32_pr1(m_pr1, w_pr1):
    mel = O.log_mel(synth.pr1_wave())
    h = O.subsample(mel, w_pr1["stem"])
    g, o = _layer_case(m_pr1, w_pr1, 0, h, [25])
    assert_f32(g, o, "layer f32")


def test_layer_f32_ragged(m_pr1, w_pr1):
    rng = np.random.default_rng(11)
    toks = [1, 12, 13, 130, 3]
    h = rng.standard_normal((sum(toks), 1024)) * 1.5
    g, o = _layer_case(m_pr1, w_pr1, 0, h, toks)
    assert_f32(g, o, "layer f32 ragged")


def test_layer_bf16_ragged(m_tower, w_tower):
    rng = np.random.default_rng(12)
    toks = [5, 130, 300, 1, 11]
    h = rng.standard_normal((sum(toks), 1024))
    for layer in (0, 11):
        g, o = _layer_case(m_tower, w_tower, layer, h, toks)
        assert_bf16(g, o, f"layer {layer} bf16")


# ------------------------------------------------------------------ whole forward

def test_encode_pr1_f32(m_pr1, w_pr1):
    g, _ = gpu_encode(m_pr1, [synth.pr1_wave()])
    o = O.encode([synth.pr1_wave()], w_pr1)[0]
    assert g.shape == (25, 512)
    assert_f32(g, o, "encode pr1")


def _trace_case(model, W, clips):
    """ae_encode_trace on clips; returns the GPU stages and the oracle's trace."""
    flat, off = synth.pack(clips)
    frames = sum(O.num_frames(len(c)) for c in clips)
    toks = sum(O.num_tokens(len(c)) for c in clips)
    H, nl = W["shape"]["hidden"], len(W["layers"])
    d_wave = dev(flat)
    d_out = torch.full((toks, W["shape"]["embed_dim"]), float("nan"), device="cuda")
    d_mel = torch.full((frames, 128), float("nan"), device="cuda")
    d_tr = torch.full((nl + 1, toks, H), float("nan"), device="cuda")
    ws = workspace(model.workspace_size(len(clips), frames, toks))
    ae.ae_encode_trace(model, d_wave, off, d_out, d_mel, d_tr, ws, ws.numel())
    _sync()
    g = (d_mel.cpu().numpy(), d_tr.cpu().numpy(), d_out.cpu().numpy())
    # without trace buffers the call is ae_encode: the same rows, bit for bit
    d_out2 = torch.full_like(d_out, float("nan"))
    ae.ae_encode_trace(model, d_wave, off, d_out2, None, None, ws, ws.numel())
    _sync()
    assert np.array_equal(d_out2.cpu().numpy(), g[2])
    o, tr = O.encode(clips, W, trace=True)
    return g, (np.concatenate(tr["mels"]), tr["subsample"], tr["layers"], np.concatenate(o))


def test_encode_trace_stages_f32(m_pr1, w_pr1):
    """The per-stage dump (encode_mels' trace): log-mel rows, the residual
    stream after in_proj and after the layer, and the output of two packed
    clips, each against the oracle's trace of the same call."""
    wave = synth.pr1_wave()
    (mel, tr, out), (o_mel, o_sub, o_layers, o_out) = _trace_case(m_pr1, w_pr1, [wave, wave[:9000]])
    assert_logmel(mel, o_mel, "trace: log-mel")
    assert_f32(tr[0], o_sub, "trace: after in_proj")
    for li, ol in enumerate(o_layers):
        assert_f32(tr[li + 1], ol, f"trace: after layer {li}")
    assert_f32(out, o_out, "trace: output")


def test_encode_trace_stages_bf16_tower(m_tower, w_tower):
    """The same dump through all 12 bf16 layers of the tower model, two clips."""
    clips = [c[:24000] for c in synth.waves("tower")[:2]]
    (mel, tr, out), (o_mel, o_sub, o_layers, o_out) = _trace_case(m_tower, w_tower, clips)
    assert len(o_layers) == 12 and tr.shape[0] == 13
    assert_logmel(mel, o_mel, "trace: log-mel")
    assert_bf16(tr[0], o_sub, "trace: after in_proj")
    for li, ol in enumerate(o_layers):
        assert_bf16(tr[li + 1], ol, f"trace: after layer {li}")
    assert_bf16(out, o_out, "trace: output")


def test_encode_tower_full_batch_sampled_clips(m_tower, w_tower):
    clips = synth.waves("tower")
    g, off = gpu_encode(m_tower, clips)
    assert g.shape == (16 * 750, 512)
    assert np.all(np.isfinite(g))
    # every clip (about 3 s of oracle time each)
    for i in range(16):
        o = O.encode([clips[i]], w_tower)[0]
        assert_bf16(g[off[i]:off[i + 1]], o, f"tower clip {i}")


def test_encode_ragged_full_batch_sampled_clips(m_tower, w_tower):
    lens = synth.clip_lengths("ragged")
    clips = synth.waves("ragged")
    g, off = gpu_encode(m_tower, clips)
    # every clip's row count is ae_num_tokens of its length (the library's own
    # count), equal to the page's formula, and the rows fill the output exactly
    assert [ae.ae_num_tokens(n) for n in lens] == [O.num_tokens(n) for n in lens]
    assert g.shape[0] == sum(O.num_tokens(n) for n in lens)
    assert np.all(np.isfinite(g))
    # 16 clips: the shortest, the longest and 14 more drawn with a fixed seed
    # (spread over the batch, so that a row count wrong anywhere before a
    # sampled clip would shift its rows and fail its comparison), the last one
    # of the batch among them
    order = np.argsort(lens)
    rng = np.random.default_rng(404)
    rest = [i for i in range(len(lens)) if i not in (int(order[0]), int(order[-1]), len(lens) - 1)]
    picks = [int(order[0]), int(order[-1]), len(lens) - 1] + sorted(rng.choice(rest, 13, replace=False).tolist())
    assert len(set(picks)) == 16
    for i in picks:
        o = O.encode([clips[i]], w_tower)[0]
        assert_bf16(g[off[i]:off[i + 1]], o, f"ragged clip {i} ({lens[i]} samples)")


def test_packing_is_bit_invariant_on_gpu(m_tower):
    rng = np.random.default_rng(21)
    clips = [(0.3 * rng.standard_normal(n)).astype(np.float32) for n in (20000, 161, 47000, 16000)]
    g, off = gpu_encode(m_tower, clips)
    for i in (0, 2):
        alone, _ = gpu_encode(m_tower, [clips[i]])
        assert np.array_equal(alone, g[off[i]:off[i + 1]]), i


def test_two_half_batches_on_two_streams_are_bit_identical(m_tower):
    """A batch of 4096+ tokens runs as two halves on two streams; with kernel
    timing on, ae_encode takes a single pass on one stream. The two results
    are bit for bit the same (every output row depends on its clip alone)."""
    rng = np.random.default_rng(17)
    lens = [480000] * 6 + [320000, 17, 240000, 1000]
    clips = [(0.3 * rng.standard_normal(n)).astype(np.float32) for n in lens]
    assert sum(O.num_tokens(len(c)) for c in clips) >= 4096
    split, _ = gpu_encode(m_tower, clips)
    ae.ae_profile_enable(True)
    try:
        single, _ = gpu_encode(m_tower, clips)
    finally:
        ae.ae_profile_enable(False)
    assert np.all(np.isfinite(split))
    assert np.array_equal(split, single)


def test_encode_host_async_two_streams_match_device_path(m_tower):
    """ae_encode_host_async on two streams with their own workspaces, four
    calls in flight: each output equals ae_encode's, bit for bit."""
    rng = np.random.default_rng(5)
    clips = [(0.3 * rng.standard_normal(n)).astype(np.float32) for n in (16000, 48000, 3000)]
    g, _ = gpu_encode(m_tower, clips)
    flat, soff = synth.pack(clips)
    h_wave = torch.from_numpy(flat).pin_memory()
    nb = ae.ae_encode_host_workspace_size(m_tower, soff)
    outs = [torch.full(g.shape, float("nan")).pin_memory() for _ in range(2)]
    wss = [workspace(nb) for _ in range(2)]
    streams = [torch.cuda.Stream() for _ in range(2)]
    for i in range(4):
        ae.ae_encode_host_async(m_tower, h_wave, soff, outs[i % 2], wss[i % 2], nb, streams[i % 2])
    _sync()
    for o in outs:
        assert np.array_equal(o.numpy(), g)


# ------------------------------------------------------------------ attention core

def _attn_oracle(q, k, v, pos, R, qd, cap=50.0):
    return O.local_attention_core(q.astype(np.float64), k.astype(np.float64), v.astype(np.float64), pos,
                                  R, qd, 8, 12, cap)


def test_attention_f32_small():
    p = synth.attention_params()
    rng = np.random.default_rng(4)
    toks = [3, 12, 140, 200]
    T = sum(toks)
    q, k, v = (rng.standard_normal((T, 1024)).astype(np.float32) for _ in range(3))
    R, qs, ks = ae.ae_attention_tables(p["relk"], p["pds"])
    out = torch.empty((T, 1024), device="cuda")
    ws = workspace(ae.ae_workspace_size(None, len(toks), 0, T))
    ae.ae_local_attention(dev(q), dev(k), dev(v), 1024, ae.AE_F32, dev(R), dev(qs), ks, 50.0, offsets(toks),
                          out, 1024, ws, ws.numel())
    _sync()
    Ro = O.relative_keys(p["relk"], 12, 1024)
    o = _attn_oracle(q, k, v, O.positions(toks), Ro, O.softplus(p["pds"]))
    assert_f32(out.cpu().numpy(), o, "attention f32")


def test_attention_microbench_full_size_sampled():
    p = synth.attention_params()
    S, T = synth.ATT_SEQS, synth.ATT_T
    R, qs, ks = ae.ae_attention_tables(p["relk"], p["pds"])
    q = torch.empty((S * T, 1024), dtype=torch.bfloat16, device="cuda")
    k, v = torch.empty_like(q), torch.empty_like(q)
    for s in range(S):
        qq, kk, vv = synth.attention_qkv(s)
        q[s * T:(s + 1) * T] = torch.from_numpy(qq).to(torch.bfloat16)
        k[s * T:(s + 1) * T] = torch.from_numpy(kk).to(torch.bfloat16)
        v[s * T:(s + 1) * T] = torch.from_numpy(vv).to(torch.bfloat16)
    out = torch.empty_like(q)
    toks = [T] * S
    ws = workspace(ae.ae_workspace_size(None, S, 0, S * T))
    ae.ae_local_attention(q, k, v, 1024, ae.AE_BF16, dev(R), dev(qs), ks, 50.0, offsets(toks), out, 1024, ws,
                          ws.numel())
    _sync()
    Ro = O.relative_keys(p["relk"], 12, 1024)
    qd = O.softplus(p["pds"])
    rng = np.random.default_rng(99)
    for s in (0, 13, 31):
        qq, kk, vv = synth.attention_qkv(s)
        idx = np.unique(np.concatenate([np.arange(0, 14), rng.integers(14, T, 50), [T - 1]]))
        got = out[s * T + idx].float().cpu().numpy()
        # each sampled token needs only its own window of 12 rows
        want = np.stack([_attn_oracle(qq[max(0, t - 11):t + 1], kk[max(0, t - 11):t + 1], vv[max(0, t - 11):t + 1],
                                      np.arange(max(0, t - 11), t + 1), Ro, qd)[-1] for t in idx])
        assert_bf16(got, want, f"attention seq {s}")


@pytest.mark.parametrize("toks", [[2, 3], [1, 3, 12, 13, 127, 1, 128, 129]])
def test_attention_bf16_edges_all_tokens(toks):
    """Every token of short and ragged batches, q/k/v as strided views of one
    [T][3072] buffer (the layout of the fused projection): clip starts inside a
    128-token tile, sequences shorter than the window, T below, at and just
    past a tile boundary."""
    p = synth.attention_params()
    rng = np.random.default_rng(len(toks))
    T = sum(toks)
    qkv = synth.round_to_bf16((2.0 * rng.standard_normal((T, 3072))).astype(np.float32))
    d = dev(qkv).to(torch.bfloat16)
    R, qs, ks = ae.ae_attention_tables(p["relk"], p["pds"])
    out = torch.full((T, 1024), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = workspace(ae.ae_workspace_size(None, len(toks), 0, T))
    ae.ae_local_attention(d[:, :1024], d[:, 1024:2048], d[:, 2048:], 3072, ae.AE_BF16, dev(R), dev(qs), ks, 50.0,
                          offsets(toks), out, 1024, ws, ws.numel())
    _sync()
    Ro = O.relative_keys(p["relk"], 12, 1024)
    o = _attn_oracle(qkv[:, :1024], qkv[:, 1024:2048], qkv[:, 2048:], O.positions(toks), Ro, O.softplus(p["pds"]))
    assert_bf16(out.float().cpu().numpy(), o, f"attention bf16, {T} tokens in {len(toks)} clips")


def test_attention_bf16_output_stride_not_32_byte_aligned():
    """An output row stride of 1032 elements (16-byte but not 32-byte multiples):
    rows leave as 16-byte pieces instead of 32-byte sectors; the same values as
    the dense output, bit for bit, and the oracle's."""
    p = synth.attention_params()
    rng = np.random.default_rng(77)
    toks = [300, 5, 200]
    T = sum(toks)
    qkv = synth.round_to_bf16((2.0 * rng.standard_normal((T, 3072))).astype(np.float32))
    d = dev(qkv).to(torch.bfloat16)
    R, qs, ks = ae.ae_attention_tables(p["relk"], p["pds"])
    ws = workspace(ae.ae_workspace_size(None, len(toks), 0, T))
    outs = []
    for ld in (1024, 1032):
        buf = torch.full((T, ld), float("nan"), dtype=torch.bfloat16, device="cuda")
        ae.ae_local_attention(d[:, :1024], d[:, 1024:2048], d[:, 2048:], 3072, ae.AE_BF16, dev(R), dev(qs), ks, 50.0,
                              offsets(toks), buf, ld, ws, ws.numel())
        _sync()
        g = buf.float().cpu().numpy()
        if ld > 1024:
            assert np.all(np.isnan(g[:, 1024:])), "columns past the row written"
        outs.append(g[:, :1024])
    assert np.array_equal(outs[0], outs[1])
    Ro = O.relative_keys(p["relk"], 12, 1024)
    o = _attn_oracle(qkv[:, :1024], qkv[:, 1024:2048], qkv[:, 2048:], O.positions(toks), Ro, O.softplus(p["pds"]))
    assert_bf16(outs[1], o, "attention bf16, output stride 1032")


# ------------------------------------------------------------------ refusals (host checks, nothing enqueued)

def test_refusals(m_tower):
    clips = [np.zeros(16000, np.float32)]
    flat, off = synth.pack(clips)
    d_wave = dev(flat)
    out = torch.empty((25, 512), device="cuda")
    need = m_tower.workspace_size(1, 99, 25)
    ws = workspace(need)
    with pytest.raises(ae.AEError) as e:
        ae.ae_encode(m_tower, d_wave, off, out, ws, need - 1)
    assert e.value.status == ae.AE_EWORKSPACE
    with pytest.raises(ae.AEError) as e:
        ae.ae_encode(m_tower, d_wave, np.array([0, 100, 50]), out, ws, need)
    assert e.value.status == ae.AE_EINVAL
    with pytest.raises(ae.AEError) as e:
        ae.ae_conformer_layer(m_tower, 12, out, [0, 25], ws, need)
    assert e.value.status == ae.AE_EINVAL
    with pytest.raises(ae.AEError) as e:
        ae.ae_encode(m_tower, None, off, out, ws, need)
    assert e.value.status == ae.AE_EINVAL
    # the rejected calls wrote nothing
    _sync()


def test_model_refuses_other_shapes(w_pr1):
    import copy
    w = copy.deepcopy(w_pr1)
    w["shape"]["heads"] = 4
    with pytest.raises(ae.AEError) as e:
        ae.Model(w, ae.AE_F32)
    assert e.value.status == ae.AE_EUNSUPPORTED
    w = copy.deepcopy(w_pr1)
    w["bounds"][0]["k"] = (-4.0, 4.0, -8.0, 8.0)
    with pytest.raises(ae.AEError) as e:
        ae.Model(w, ae.AE_F32)
    assert e.value.status == ae.AE_EUNSUPPORTED
