"""ctypes binding of libae.so (include/ae.h): argument marshalling only.

Every function keeps the C name. Device buffers are passed as torch CUDA
tensors (or raw integer addresses); offsets as int64 sequences; streams as
torch.cuda.Stream (or a raw handle, None = the current torch stream). No
computation happens here: each call goes straight to the library, and a
missing library raises at import.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libae.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m log_mel_front_b200.build` "
        "(there is no fallback implementation)")
lib = C.CDLL(LIB_PATH)

AE_OK, AE_EINVAL, AE_EUNSUPPORTED, AE_EWORKSPACE, AE_ECUDA, AE_ENOMEM, AE_EDEVICE = range(7)
AE_F32, AE_BF16, AE_FP8 = 0, 1, 2
AE_LIN_BF16, AE_LIN_SILU_E4M3 = 0, 1
STATUS_NAMES = {0: "AE_OK", 1: "AE_EINVAL", 2: "AE_EUNSUPPORTED", 3: "AE_EWORKSPACE", 4: "AE_ECUDA",
                5: "AE_ENOMEM", 6: "AE_EDEVICE"}

_fp = C.POINTER(C.c_float)
_i64p = C.POINTER(C.c_int64)


class ae_lfm_config(C.Structure):
    _fields_ = [("sample_rate", C.c_int32), ("n_fft", C.c_int32), ("win_length", C.c_int32), ("hop", C.c_int32),
                ("n_mels", C.c_int32), ("preemph", C.c_float), ("log_floor", C.c_float), ("var_eps", C.c_float)]


class ae_config(C.Structure):
    _fields_ = [(n, C.c_int32) for n in ("n_mels", "c0", "c1", "hidden", "heads", "ffn", "left", "kernel",
                                        "out_dim", "embed_dim", "n_layers")] + \
               [("softcap", C.c_float), ("residual_weight", C.c_float)]


class ae_clip(C.Structure):
    _fields_ = [("lo_in", C.c_float), ("hi_in", C.c_float), ("lo_out", C.c_float), ("hi_out", C.c_float)]


LAYER_PTRS = ("ff1_pre", "ff1_w1", "ff1_w2", "ff1_post", "ff2_pre", "ff2_w1", "ff2_w2", "ff2_post",
              "norm_pre_attn", "norm_post_attn", "norm_out", "q", "k", "v", "post", "per_dim_scale",
              "relative_k", "lc_pre", "lc_start", "lc_dw", "lc_norm", "lc_end")
LAYER_CLIPS = ("clip_ff1_w1", "clip_ff1_w2", "clip_q", "clip_k", "clip_v", "clip_post", "clip_lc_start",
               "clip_lc_end", "clip_ff2_w1", "clip_ff2_w2")


class ae_host_layer(C.Structure):
    _fields_ = [(n, _fp) for n in LAYER_PTRS] + [(n, ae_clip) for n in LAYER_CLIPS]


class ae_host_weights(C.Structure):
    _fields_ = [("conv0", _fp), ("ln0", _fp), ("conv1", _fp), ("ln1", _fp), ("in_proj", _fp),
                ("layers", C.POINTER(ae_host_layer)), ("out_proj", _fp), ("out_bias", _fp), ("embed", _fp)]


_vp, _sz, _st, _i32 = C.c_void_p, C.c_size_t, C.c_int, C.c_int


def _sig(name, res, *args):
    f = getattr(lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_sig("ae_num_frames", C.c_int64, C.c_int64)
_sig("ae_num_tokens", C.c_int64, C.c_int64)
_sig("ae_partition_clips", _st, _i64p, _i32, _i32, C.POINTER(C.c_int32), _i64p)
_sig("ae_model_create", _st, C.POINTER(ae_config), C.POINTER(ae_host_weights), _i32, C.POINTER(_vp))
_sig("ae_model_destroy", None, _vp)
_sig("ae_workspace_size", _sz, _vp, C.c_int64, C.c_int64, C.c_int64)
_sig("ae_logmel", _st, _vp, _i64p, _i32, _vp, _vp, _sz, _vp)
_sig("ae_subsample", _st, _vp, _vp, _i64p, _i32, _vp, _vp, _sz, _vp)
_sig("ae_conformer_layer", _st, _vp, _i32, _vp, _i64p, _i32, _vp, _sz, _vp)
_sig("ae_encode", _st, _vp, _vp, _i64p, _i32, _vp, _vp, _sz, _vp)
_sig("ae_encode_trace", _st, _vp, _vp, _i64p, _i32, _vp, _vp, _vp, _vp, _sz, _vp)
_sig("ae_encode_host_workspace_size", _sz, _vp, _i64p, _i32)
_sig("ae_encode_host", _st, _vp, _vp, _i64p, _i32, _vp, _vp, _sz, _vp)
_sig("ae_encode_host_async", _st, _vp, _vp, _i64p, _i32, _vp, _vp, _sz, _vp)
_sig("ae_attention_tables", _st, _fp, _fp, _i32, _i32, _i32, _fp, _fp, _fp)
_sig("ae_local_attention", _st, _vp, _vp, _vp, C.c_int64, _i32, _vp, _vp, C.c_float, C.c_float, _i64p, _i32,
     _vp, C.c_int64, _vp, _sz, _vp)
_sig("ae_last_error", C.c_char_p)
_sig("ae_device_status", _st)
_sig("ae_version", C.c_char_p)
_sig("ae_logmel_noalloc", _st, _vp, _i64p, _i32, _vp, _vp)
_sig("ae_resample_len", C.c_int64, C.c_int64, C.c_int32, C.c_int32)
_sig("ae_resample_workspace_size", _sz, _i64p, _i32, C.c_int32, C.c_int32, _i32)
_sig("ae_resample", _st, _vp, _i32, C.c_int64, _i64p, _i32, C.c_int32, C.c_int32, _vp, _vp, _sz, _vp)
_sig("ae_linear_e4m3", _st, _vp, _vp, _vp, C.c_int64, C.c_int32, C.c_int32, C.c_float, C.c_float, _i32, C.c_float,
     C.c_float, C.c_float, _vp, _vp)
_sig("ae_selftest_bounded_wait", _st, C.c_uint32, _i32, _vp)
_sig("ae_launch_count", C.c_uint64)
_sig("ae_lfm_default_config", None, C.POINTER(ae_lfm_config))
_sig("ae_lfm_num_frames", C.c_int64, C.POINTER(ae_lfm_config), C.c_int64)
_sig("ae_lfm_workspace_size", _sz, C.POINTER(ae_lfm_config), _i32)
_sig("ae_lfm_logmel", _st, C.POINTER(ae_lfm_config), _vp, _i64p, _i32, _vp, _vp, _sz, _vp)
_sig("ae_profile_enable", _st, _i32)
_sig("ae_profile_read", _st, C.POINTER(C.c_double), _i64p, C.POINTER(C.c_double), C.POINTER(C.c_double), _i64p)

# every symbol include/ae.h declares
EXPORTS = ("ae_num_frames", "ae_num_tokens", "ae_model_create", "ae_model_destroy", "ae_workspace_size",
           "ae_logmel", "ae_subsample", "ae_conformer_layer", "ae_encode", "ae_encode_trace",
           "ae_encode_host_workspace_size",
           "ae_encode_host", "ae_encode_host_async", "ae_attention_tables", "ae_local_attention", "ae_last_error",
           "ae_device_status", "ae_version", "ae_profile_enable", "ae_profile_read", "ae_logmel_noalloc",
           "ae_resample_len", "ae_resample_workspace_size", "ae_resample", "ae_linear_e4m3",
           "ae_selftest_bounded_wait", "ae_lfm_default_config", "ae_lfm_num_frames", "ae_lfm_workspace_size",
           "ae_lfm_logmel", "ae_launch_count", "ae_partition_clips", "ae_lenc_default_config", "ae_lenc_num_tokens",
           "ae_lenc_create", "ae_lenc_destroy", "ae_lenc_workspace_size", "ae_lenc_block_workspace_size",
           "ae_lenc_stem", "ae_lenc_block", "ae_lenc_encode")

KERNEL_CLASSES = ("tables", "logmel", "conv0", "conv1", "gemm", "attention", "lconv", "rowop", "resample",
                  "gemm_fp8", "lfm", "lenc_gemm", "lenc_attention", "lenc_row")


class AEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.ae_last_error().decode(errors="replace")
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")


def _check(st: int, where: str):
    if st != AE_OK:
        raise AEError(st, where)


def _ptr(x) -> int | None:
    """Device or host address of a tensor / array / int (None stays NULL)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    raise TypeError(type(x))


def _stream(s) -> int | None:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _off(off) -> tuple[np.ndarray, C.POINTER(C.c_int64)]:
    a = np.ascontiguousarray(np.asarray(off, dtype=np.int64))
    return a, a.ctypes.data_as(_i64p)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


# ------------------------------------------------------------------ calls

def ae_num_frames(n: int) -> int:
    return lib.ae_num_frames(int(n))


def ae_num_tokens(n: int) -> int:
    return lib.ae_num_tokens(int(n))


def ae_partition_clips(sample_off, n_parts: int) -> tuple[np.ndarray, np.ndarray]:
    """(part of each clip int32 [n_clips], tokens of each part int64 [n_parts])."""
    a, p = _off(sample_off)
    n = len(a) - 1
    part = np.zeros(max(n, 0), np.int32)
    tok = np.zeros(max(int(n_parts), 1), np.int64)
    _check(lib.ae_partition_clips(p, n, int(n_parts), part.ctypes.data_as(C.POINTER(C.c_int32)),
                                  tok.ctypes.data_as(_i64p)), "ae_partition_clips")
    return part, tok[:int(n_parts)]


def ae_workspace_size(model, n_clips: int, total_frames: int, total_tokens: int) -> int:
    return lib.ae_workspace_size(model.handle if model is not None else None, n_clips, total_frames, total_tokens)


def ae_logmel(d_wave, sample_off, d_mel, d_ws, ws_bytes: int, stream=None):
    a, p = _off(sample_off)
    _check(lib.ae_logmel(_ptr(d_wave), p, len(a) - 1, _ptr(d_mel), _ptr(d_ws), ws_bytes, _stream(stream)),
           "ae_logmel")


def ae_logmel_noalloc(d_wave, sample_off, d_mel, stream=None):
    """ae_logmel without a workspace: for callers that must not allocate device
    memory (the clip tables live in a fixed array inside the library)."""
    a, p = _off(sample_off)
    _check(lib.ae_logmel_noalloc(_ptr(d_wave), p, len(a) - 1, _ptr(d_mel), _stream(stream)), "ae_logmel_noalloc")


def ae_subsample(model, d_mel, frame_off, d_h, d_ws, ws_bytes: int, stream=None):
    a, p = _off(frame_off)
    _check(lib.ae_subsample(model.handle, _ptr(d_mel), p, len(a) - 1, _ptr(d_h), _ptr(d_ws), ws_bytes,
                            _stream(stream)), "ae_subsample")


def ae_conformer_layer(model, layer: int, d_h, tok_off, d_ws, ws_bytes: int, stream=None):
    a, p = _off(tok_off)
    _check(lib.ae_conformer_layer(model.handle, layer, _ptr(d_h), p, len(a) - 1, _ptr(d_ws), ws_bytes,
                                  _stream(stream)), "ae_conformer_layer")


def ae_encode(model, d_wave, sample_off, d_out, d_ws, ws_bytes: int, stream=None):
    a, p = _off(sample_off)
    _check(lib.ae_encode(model.handle, _ptr(d_wave), p, len(a) - 1, _ptr(d_out), _ptr(d_ws), ws_bytes,
                         _stream(stream)), "ae_encode")


def ae_encode_trace(model, d_wave, sample_off, d_out, d_mel, d_trace, d_ws, ws_bytes: int, stream=None):
    a, p = _off(sample_off)
    _check(lib.ae_encode_trace(model.handle, _ptr(d_wave), p, len(a) - 1, _ptr(d_out), _ptr(d_mel), _ptr(d_trace),
                               _ptr(d_ws), ws_bytes, _stream(stream)), "ae_encode_trace")


def ae_encode_host_workspace_size(model, sample_off) -> int:
    a, p = _off(sample_off)
    return lib.ae_encode_host_workspace_size(model.handle, p, len(a) - 1)


def ae_encode_host(model, h_wave, sample_off, h_out, d_ws, ws_bytes: int, stream=None):
    a, p = _off(sample_off)
    _check(lib.ae_encode_host(model.handle, _ptr(h_wave), p, len(a) - 1, _ptr(h_out), _ptr(d_ws), ws_bytes,
                              _stream(stream)), "ae_encode_host")


def ae_encode_host_async(model, h_wave, sample_off, h_out, d_ws, ws_bytes: int, stream=None):
    """Enqueues ae_encode_host on `stream` without waiting; the buffers belong
    to the call until the stream has passed it."""
    a, p = _off(sample_off)
    _check(lib.ae_encode_host_async(model.handle, _ptr(h_wave), p, len(a) - 1, _ptr(h_out), _ptr(d_ws), ws_bytes,
                                    _stream(stream)), "ae_encode_host_async")


def ae_attention_tables(relative_k, per_dim_scale, hidden: int = 1024, heads: int = 8, left: int = 12):
    rk, pd = _f32(relative_k), _f32(per_dim_scale)
    R = np.zeros((left, hidden), np.float32)
    qs = np.zeros(hidden // heads, np.float32)
    ks = C.c_float(0.0)
    _check(lib.ae_attention_tables(rk.ctypes.data_as(_fp), pd.ctypes.data_as(_fp), hidden, heads, left,
                                   R.ctypes.data_as(_fp), qs.ctypes.data_as(_fp), C.byref(ks)),
           "ae_attention_tables")
    return R, qs, ks.value


def ae_local_attention(d_q, d_k, d_v, ld_qkv: int, dtype: int, d_R, d_qscale, k_scale: float, softcap: float,
                       tok_off, d_out, ld_out: int, d_ws, ws_bytes: int, stream=None):
    a, p = _off(tok_off)
    _check(lib.ae_local_attention(_ptr(d_q), _ptr(d_k), _ptr(d_v), ld_qkv, dtype, _ptr(d_R), _ptr(d_qscale),
                                  k_scale, softcap, p, len(a) - 1, _ptr(d_out), ld_out, _ptr(d_ws), ws_bytes,
                                  _stream(stream)), "ae_local_attention")


def ae_linear_e4m3(d_x, d_w, d_cs, M: int, N: int, K: int, lo: float, hi: float, d_y, out: int = AE_LIN_BF16,
                   lo2: float = float("-inf"), hi2: float = float("inf"), q_out: float = 1.0, stream=None):
    _check(lib.ae_linear_e4m3(_ptr(d_x), _ptr(d_w), _ptr(d_cs), M, N, K, lo, hi, out, lo2, hi2, q_out, _ptr(d_y),
                              _stream(stream)), "ae_linear_e4m3")


def ae_device_status() -> int:
    return lib.ae_device_status()


def ae_launch_count() -> int:
    """Kernels the library has launched since it was loaded."""
    return int(lib.ae_launch_count())


def lfm_config(**kw) -> "ae_lfm_config":
    """The library's defaults (ae_lfm_default_config) with the given fields replaced."""
    c = ae_lfm_config()
    lib.ae_lfm_default_config(C.byref(c))
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def ae_lfm_num_frames(cfg, n_samples: int) -> int:
    return lib.ae_lfm_num_frames(C.byref(cfg), int(n_samples))


def ae_lfm_workspace_size(cfg, n_clips: int) -> int:
    return lib.ae_lfm_workspace_size(C.byref(cfg), int(n_clips))


def ae_lfm_logmel(cfg, d_wave, sample_off, d_out, d_ws, ws_bytes: int, stream=None):
    a, p = _off(sample_off)
    _check(lib.ae_lfm_logmel(C.byref(cfg), _ptr(d_wave), p, len(a) - 1, _ptr(d_out), _ptr(d_ws), ws_bytes,
                             _stream(stream)), "ae_lfm_logmel")


def ae_selftest_bounded_wait(limit_us: int, arrive: bool = False, stream=None):
    _check(lib.ae_selftest_bounded_wait(int(limit_us), 1 if arrive else 0, _stream(stream)),
           "ae_selftest_bounded_wait")


def ae_version() -> str:
    return lib.ae_version().decode()


def ae_profile_enable(on: bool = True):
    _check(lib.ae_profile_enable(1 if on else 0), "ae_profile_enable")


def ae_resample_len(n_samples: int, rate_in: int, rate_out: int = 16000) -> int:
    return lib.ae_resample_len(int(n_samples), int(rate_in), int(rate_out))


def ae_resample_workspace_size(sample_off, rate_in: int, rate_out: int = 16000, channels: int = 1) -> int:
    a, p = _off(sample_off)
    return lib.ae_resample_workspace_size(p, len(a) - 1, int(rate_in), int(rate_out), int(channels))


def ae_resample(d_x, channels: int, ch_stride: int, sample_off, rate_in: int, rate_out: int, d_y, d_ws,
                ws_bytes: int, stream=None):
    a, p = _off(sample_off)
    _check(lib.ae_resample(_ptr(d_x), int(channels), int(ch_stride), p, len(a) - 1, int(rate_in), int(rate_out),
                           _ptr(d_y), _ptr(d_ws), ws_bytes, _stream(stream)), "ae_resample")


def ae_profile_read() -> dict:
    """{class: {"ms", "launches", "flops", "bytes"}} since the last read, and "dropped"."""
    n = len(KERNEL_CLASSES)
    ms, fl, by = (C.c_double * n)(), (C.c_double * n)(), (C.c_double * n)()
    la = (C.c_int64 * n)()
    dr = C.c_int64(0)
    _check(lib.ae_profile_read(ms, la, fl, by, C.byref(dr)), "ae_profile_read")
    out = {k: {"ms": ms[i], "launches": la[i], "flops": fl[i], "bytes": by[i]} for i, k in enumerate(KERNEL_CLASSES)}
    out["dropped"] = dr.value
    return out


# ------------------------------------------------------------------ model

class Model:
    """An ae_model built from a weight dict in the checkpoint's layout
    (``synth.model_weights`` produces one): host arrays in, device model out."""

    def __init__(self, weights: dict, dtype: int = AE_BF16):
        s = weights["shape"]
        cfg = ae_config(n_mels=s["n_mels"], c0=s["c0"], c1=s["c1"], hidden=s["hidden"], heads=s["heads"],
                        ffn=s["ffn"], left=s["left"], kernel=s["kernel"], out_dim=s["out_dim"],
                        embed_dim=s["embed_dim"], n_layers=len(weights["layers"]), softcap=s["softcap"],
                        residual_weight=s["residual_weight"])
        keep = []

        def fp(a):
            a = _f32(a)
            keep.append(a)
            return a.ctypes.data_as(_fp)

        st, hd = weights["stem"], weights["head"]
        L = len(weights["layers"])
        layers = (ae_host_layer * max(L, 1))()
        names = {"ff1_pre": "ff1.pre", "ff1_w1": "ff1.w1", "ff1_w2": "ff1.w2", "ff1_post": "ff1.post",
                 "ff2_pre": "ff2.pre", "ff2_w1": "ff2.w1", "ff2_w2": "ff2.w2", "ff2_post": "ff2.post",
                 "per_dim_scale": "pds", "relative_k": "relk"}
        for i, (ly, bd) in enumerate(zip(weights["layers"], weights["bounds"])):
            for f in LAYER_PTRS:
                setattr(layers[i], f, fp(ly[names.get(f, f)]))
            for f in LAYER_CLIPS:
                key = f[5:].replace("ff1_", "ff1.").replace("ff2_", "ff2.")
                setattr(layers[i], f, ae_clip(*[float(v) for v in bd[key]]))
        w = ae_host_weights(conv0=fp(st["conv0"]), ln0=fp(st["ln0"]), conv1=fp(st["conv1"]), ln1=fp(st["ln1"]),
                            in_proj=fp(st["in_proj"]), layers=layers, out_proj=fp(hd["out_proj"]),
                            out_bias=fp(hd["out_bias"]), embed=fp(hd["embed"]))
        h = C.c_void_p()
        _check(lib.ae_model_create(C.byref(cfg), C.byref(w), dtype, C.byref(h)), "ae_model_create")
        self.handle = h.value
        self.dtype = dtype
        self.shape = dict(s)
        self.n_layers = L

    def workspace_size(self, n_clips: int, total_frames: int, total_tokens: int) -> int:
        return lib.ae_workspace_size(self.handle, n_clips, total_frames, total_tokens)

    def close(self):
        if getattr(self, "handle", None):
            lib.ae_model_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ------------------------------------------------------------------ LFM2A Conformer encoder

class ae_lenc_config(C.Structure):
    _fields_ = [(n, C.c_int32) for n in ("n_mels", "n_embd", "n_head", "n_layers", "n_ff", "conv_k", "stem_ch",
                                        "adapter_ff", "llm_hidden")] + [("eps", C.c_float)]


LENC_BLOCK_FIELDS = ("ffn1_norm_w", "ffn1_norm_b", "ffn1_up_w", "ffn1_up_b", "ffn1_down_w", "ffn1_down_b",
                     "ln1_w", "ln1_b", "q_w", "q_b", "k_w", "k_b", "v_w", "v_b", "o_w", "o_b",
                     "linear_pos_w", "pos_bias_u", "pos_bias_v",
                     "norm_conv_w", "norm_conv_b", "pw1_w", "pw1_b", "dw_w", "dw_b", "conv_norm_w", "conv_norm_b",
                     "pw2_w", "pw2_b",
                     "ffn2_norm_w", "ffn2_norm_b", "ffn2_up_w", "ffn2_up_b", "ffn2_down_w", "ffn2_down_b",
                     "ln2_w", "ln2_b")


def _lenc_key(field: str) -> str:
    """The weight-dict key (synth.lfm_encoder_weights) of a block field."""
    if field.startswith(("ffn1_", "ffn2_")):
        return field[:4] + "." + field[5:]
    if field[:2] in ("q_", "k_", "v_", "o_") and len(field) == 3:
        return "attn_" + field
    if field in ("pw1_w", "pw1_b", "dw_w", "dw_b", "pw2_w", "pw2_b"):
        return "conv_" + field
    return field


class ae_lenc_host_block(C.Structure):
    _fields_ = [(n, _fp) for n in LENC_BLOCK_FIELDS]


class ae_lenc_host_weights(C.Structure):
    _fields_ = [("stem_w", _fp * 5), ("stem_b", _fp * 5), ("pre_w", _fp), ("pre_b", _fp),
                ("blocks", C.POINTER(ae_lenc_host_block)),
                ("ad_norm_w", _fp), ("ad_norm_b", _fp), ("ad_up_w", _fp), ("ad_up_b", _fp),
                ("ad_down_w", _fp), ("ad_down_b", _fp)]


_sig("ae_lenc_default_config", None, C.POINTER(ae_lenc_config))
_sig("ae_lenc_num_tokens", C.c_int64, C.c_int64)
_sig("ae_lenc_create", _st, C.POINTER(ae_lenc_config), C.POINTER(ae_lenc_host_weights), C.POINTER(_vp))
_sig("ae_lenc_destroy", None, _vp)
_sig("ae_lenc_workspace_size", _sz, _vp, _i64p, _i32)
_sig("ae_lenc_block_workspace_size", _sz, _vp, _i64p, _i32)
_sig("ae_lenc_stem", _st, _vp, _vp, _i64p, _i32, _vp, _vp, _sz, _vp)
_sig("ae_lenc_block", _st, _vp, _i32, _vp, _i64p, _i32, _vp, _sz, _vp)
_sig("ae_lenc_encode", _st, _vp, _vp, _i64p, _i32, _vp, _vp, _sz, _vp)


def lenc_config(**kw) -> "ae_lenc_config":
    """The library's defaults (ae_lenc_default_config) with the given fields replaced."""
    c = ae_lenc_config()
    lib.ae_lenc_default_config(C.byref(c))
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def ae_lenc_num_tokens(n_frames: int) -> int:
    return lib.ae_lenc_num_tokens(int(n_frames))


class LencModel:
    """An ae_lenc built from a weight dict in the page's layouts
    (``synth.lfm_encoder_weights`` produces one)."""

    def __init__(self, W: dict):
        s = W["cfg"]
        cfg = lenc_config(**{k: s[k] for k in ("n_mels", "n_embd", "n_head", "n_layers", "n_ff", "conv_k", "stem_ch",
                                               "adapter_ff", "llm_hidden", "eps")})
        keep = []

        def fp(a):
            a = _f32(a)
            keep.append(a)
            return a.ctypes.data_as(_fp)

        L = len(W["layers"])
        blocks = (ae_lenc_host_block * max(L, 1))()
        for i, ly in enumerate(W["layers"]):
            for f in LENC_BLOCK_FIELDS:
                setattr(blocks[i], f, fp(ly[_lenc_key(f)]))
        w = ae_lenc_host_weights()
        for i in range(5):
            w.stem_w[i] = fp(W[f"stem{i}.w"])
            w.stem_b[i] = fp(W[f"stem{i}.b"])
        w.pre_w, w.pre_b = fp(W["pre_w"]), fp(W["pre_b"])
        w.blocks = blocks
        for k in ("ad_norm_w", "ad_norm_b", "ad_up_w", "ad_up_b", "ad_down_w", "ad_down_b"):
            setattr(w, k, fp(W[k]))
        h = C.c_void_p()
        _check(lib.ae_lenc_create(C.byref(cfg), C.byref(w), C.byref(h)), "ae_lenc_create")
        self.handle = h.value
        self.cfg = dict(s)

    def workspace_size(self, frame_off) -> int:
        a, p = _off(frame_off)
        return lib.ae_lenc_workspace_size(self.handle, p, len(a) - 1)

    def block_workspace_size(self, tok_off) -> int:
        a, p = _off(tok_off)
        return lib.ae_lenc_block_workspace_size(self.handle, p, len(a) - 1)

    def close(self):
        if getattr(self, "handle", None):
            lib.ae_lenc_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def ae_lenc_stem(model, d_mel, frame_off, d_x, d_ws, ws_bytes: int, stream=None):
    a, p = _off(frame_off)
    _check(lib.ae_lenc_stem(model.handle, _ptr(d_mel), p, len(a) - 1, _ptr(d_x), _ptr(d_ws), ws_bytes,
                            _stream(stream)), "ae_lenc_stem")


def ae_lenc_block(model, layer: int, d_x, tok_off, d_ws, ws_bytes: int, stream=None):
    a, p = _off(tok_off)
    _check(lib.ae_lenc_block(model.handle, int(layer), _ptr(d_x), p, len(a) - 1, _ptr(d_ws), ws_bytes,
                             _stream(stream)), "ae_lenc_block")


def ae_lenc_encode(model, d_mel, frame_off, d_out, d_ws, ws_bytes: int, stream=None):
    a, p = _off(frame_off)
    _check(lib.ae_lenc_encode(model.handle, _ptr(d_mel), p, len(a) - 1, _ptr(d_out), _ptr(d_ws), ws_bytes,
                              _stream(stream)), "ae_lenc_encode")
