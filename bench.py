#!/usr/bin/env python
"""Throughput of the B200 audio-encoder forward.

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--workload ragged|tower|tower_fp8|frontend|lfm_frontend|lfm_encoder|lfm_ragged|attention|resample]
    python bench.py --impl reference ...      # the CPU oracle on the same workload (bounded sample)

A step is one ae_encode over one batch (default: the ragged batch, 256 clips
of 1-30 s packed without padding, the 12-layer tower plus the embedding
head, bf16 tensor-core projections), inputs resident in device memory. K
steps are timed with CUDA events on the launching stream after W warm-up
steps, L2 flushed (256 MiB written) between steps, outside the events.

With N > 1 ranks (torchrun, or `--gpus N`, which re-launches itself under
torchrun), the clip workloads run a global batch of N times the workload's
clips, split over the ranks by ae_partition_clips (greedy token balance; the
model is replicated, and the data path has no collective): weak scaling. The
step time is the max over ranks; the value counts the whole global batch. The
attention and resampling workloads run one replica per rank.

One JSON line on rank 0: the metric, the end-to-end figure through
ae_encode_host_async (host buffers, copies inside the timed region), the
roofline of the dominant kernel class from the library's per-launch event
timing, the clocks seen during the timed region, and the oracle's CPU
baseline.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "audio seconds encoded/sec (soft tokens/sec) on 1 B200; % HBM / % tensor peak"
UNIT = "audio-s/s"
L2_FLUSH_BYTES = 256 << 20


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------ clocks

# DRAM traffic of the dominant kernel comes from a committed ncu summary
# (dram__bytes_read.sum + dram__bytes_write.sum per launch over one step). The
# summary records the sha256 of the kernel's sources at capture time; once they
# differ the figure no longer describes the kernel and is reported as null.
_GEMM_SRC = ("log_mel_front_b200/csrc/gemm.cu", "log_mel_front_b200/csrc/common.cuh")
TRAFFIC_PROFILES = {
    ("gemm", "tower"): ("profiles/gemm_tc_tower_dram.md", _GEMM_SRC),
    ("gemm_fp8", "tower_fp8"): ("profiles/gemm_e4m3_tower_dram.md", _GEMM_SRC),
    ("gemm", "ragged"): ("profiles/gemm_tc_ragged_dram.md", _GEMM_SRC),
}


def sources_sha256(paths) -> str:
    import hashlib
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def captured_traffic(kind: str, workload: str):
    """(bytes per launch, note) from the committed capture of this kernel class
    on this workload, or (None, why)."""
    if (kind, workload) not in TRAFFIC_PROFILES:
        return None, "no capture for this kernel on this workload"
    path, srcs = TRAFFIC_PROFILES[(kind, workload)]
    vals = {}
    try:
        with open(os.path.join(ROOT, path)) as f:
            for line in f:
                if ":" in line and line.split(":", 1)[0].strip() in ("traffic_bytes_per_launch", "source_sha256"):
                    k, v = line.split(":", 1)
                    vals[k.strip()] = v.strip().strip("`")
    except OSError:
        return None, "capture summary missing"
    if "traffic_bytes_per_launch" not in vals or "source_sha256" not in vals:
        return None, "capture summary incomplete"
    if vals["source_sha256"] != sources_sha256(srcs):
        return None, "kernel sources changed since the capture"
    return float(vals["traffic_bytes_per_launch"]), path


class Clocks:
    """nvidia-smi sampled every 100 ms during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        time.sleep(0.3)
        if self.p:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()

    def summary(self):
        self.f.flush()
        rows = []
        for line in open(self.f.name):
            c = [x.strip() for x in line.split(",")]
            if len(c) < 10:
                continue
            try:
                rows.append((float(c[1]), float(c[2]), float(c[4]), c[6], c[7], c[8], c[9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        busy = [r for r in rows if r[2] >= 30] or rows
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in busy for n, v in zip(names, r[3:]) if v.lower().startswith("active")})
        return {"sm_mhz": float(np.median([r[0] for r in busy])), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(busy)}


def tensor_peak_kind(clocks: dict) -> tuple[bool, str]:
    """Which measured bf16 peak a projection timed in this run is held to: the
    burst figure (cuBLAS in a short burst at the maximum clock) when the SM
    clock under load stayed within 10% of its maximum, else the sustained one
    (a seconds-long loop under the power cap, near 1.35 GHz)."""
    mhz, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    if mhz and mx and mhz >= 0.9 * mx:
        return True, "burst"
    return False, "sustained"


# ------------------------------------------------------------------ workloads

def workload_desc(name: str, info: dict) -> dict:
    base = {"tower": "16 clips x 30 s, 12 Conformer layers + embedding head, bf16 weights, f32 accumulation",
            "tower_fp8": "16 clips x 30 s, 12 Conformer layers + embedding head; FFN W1/W2, q/k/v and lc_start "
                         "on e4m3 operands (per-row weight scales, input scale from the ClipLin clamp), the other "
                         "projections bf16; f32 accumulation",
            "ragged": "256 clips of 1-30 s (uniform whole samples), packed, 12 layers + head, bf16",
            "frontend": "log-mel front-end only, 64 clips x 30 s, f32",
            "lfm_frontend": "second (LFM2A) log-mel front-end: pre-emphasis, centre padding, power spectrum, Slaney "
                            "bank, per-band normalisation; 64 clips x 30 s, f32",
            "lfm_encoder": "LFM2A encoder from PCM: the second log-mel front-end, the 5-layer conv stem, 17 "
                           "Conformer blocks with Transformer-XL attention and the erf-GELU adapter to 2048; 16 "
                           "clips x 30 s (376 tokens each), bf16 weights, f32 accumulation",
            "lfm_ragged": "LFM2A encoder from PCM (second log-mel front-end, stem, 17 blocks, adapter) on the "
                          "ragged batch: 256 clips of 1-30 s, packed, bf16 weights, f32 accumulation",
            "attention": "local-attention core only, 32 x 8192 tokens, 8 heads x 128, bf16 q/k/v",
            "resample": "mixdown + Kaiser-sinc resampling to 16 kHz, 64 stereo clips x 30 s at 44.1 kHz, f32"}[name]
    d = {"workload": f"{name}: {base}", "l2": "flushed between steps (256 MiB write)",
         "model": "gemma4_audio tower shape (random init)"}
    d.update(info)
    return d


ENCODE_WORKLOADS = ("tower", "tower_fp8", "ragged")
LFM_ENCODER_WORKLOADS = ("lfm_encoder", "lfm_ragged")
CLIP_WORKLOADS = ENCODE_WORKLOADS + ("frontend", "lfm_frontend") + LFM_ENCODER_WORKLOADS


def rank_clips(lengths, world: int, rank: int, partition) -> list[int]:
    """Global indices (ascending) of the clips this rank encodes: `partition`
    (ae_partition_clips) splits the global batch by greedy token balance; every
    rank computes the same split from the lengths alone."""
    off = np.zeros(len(lengths) + 1, np.int64)
    off[1:] = np.cumsum(lengths)
    part, _ = partition(off, world)
    return [i for i in range(len(lengths)) if part[i] == rank]


def audio_seconds(lengths) -> float:
    """Audio the encoder reads from clips of these lengths (30 s cap)."""
    return sum(min(int(n), synth.MAX_SAMPLES) for n in lengths) / synth.SAMPLE_RATE


def data_of(name: str) -> str:
    """The synthetic batch a workload runs on (the e4m3 tower runs the tower's,
    the second front-end the first one's)."""
    return {"tower_fp8": "tower", "lfm_frontend": "frontend", "lfm_encoder": "tower", "lfm_ragged": "ragged"}.get(
        name, name)


class Ours:
    def __init__(self, name: str, rank: int = 0, world: int = 1):
        import torch
        import log_mel_front_b200 as ae
        self.ae, self.torch, self.name = ae, torch, name
        self.stream = torch.cuda.current_stream()
        self.job_audio_s = None
        if name in CLIP_WORKLOADS:
            lens_all = synth.global_lengths(data_of(name), world)
            self.mine = rank_clips(lens_all, world, rank, ae.ae_partition_clips)
            self.lens = [lens_all[i] for i in self.mine]
            self.job_clips, self.job_audio_s = len(lens_all), audio_seconds(lens_all)
            self.job_tokens = sum(ae.ae_num_tokens(n) for n in lens_all)
            if name in LFM_ENCODER_WORKLOADS:  # the LFM2A encoder's own rows: its stem leaves 12.5 per second
                cfg = ae.lfm_config()
                self.job_tokens = sum(ae.ae_lenc_num_tokens(ae.ae_lfm_num_frames(cfg, n)) for n in lens_all)
            clips = synth.global_waves(data_of(name), lens_all, self.mine)
            flat, self.off = synth.pack(clips)
            self.h_wave = torch.from_numpy(flat).pin_memory()
            self.d_wave = self.h_wave.cuda()
            self.frames = sum(ae.ae_num_frames(n) for n in self.lens)
            self.tokens = sum(ae.ae_num_tokens(n) for n in self.lens)
            self.audio_s = audio_seconds(self.lens)
        if name in ENCODE_WORKLOADS:
            self.model = ae.Model(synth.model_weights(data_of(name)), ae.AE_FP8 if name == "tower_fp8" else ae.AE_BF16)
            self.ws_bytes = self.model.workspace_size(len(self.lens), self.frames, self.tokens)
            self.d_out = torch.empty((self.tokens, 512), device="cuda")
            self.h_out = torch.empty((self.tokens, 512)).pin_memory()
            self.ws_host_bytes = ae.ae_encode_host_workspace_size(self.model, self.off)
            self.ws = torch.empty(max(self.ws_bytes, self.ws_host_bytes), dtype=torch.uint8, device="cuda")
            self.dominant = "gemm_fp8" if name == "tower_fp8" else "gemm"
        elif name in LFM_ENCODER_WORKLOADS:
            self.cfg = ae.lfm_config()
            self.lfm_frames = [ae.ae_lfm_num_frames(self.cfg, n) for n in self.lens]
            self.frames = sum(self.lfm_frames)
            self.lfm_ws_bytes = ae.ae_lfm_workspace_size(self.cfg, len(self.lens))
            self.lfm_ws = torch.empty(self.lfm_ws_bytes, dtype=torch.uint8, device="cuda")
            self.d_mel = torch.empty((self.frames, 128), device="cuda")
            self.enc = ae.LencModel(synth.lfm_encoder_weights())
            self.frame_off = np.concatenate([[0], np.cumsum(self.lfm_frames)]).astype(np.int64)
            self.tokens = sum(ae.ae_lenc_num_tokens(f) for f in self.lfm_frames)
            self.ws_bytes = self.enc.workspace_size(self.frame_off)
            self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")
            self.d_out = torch.empty((self.tokens, 2048), device="cuda")
            self.h_out = torch.empty((self.tokens, 2048)).pin_memory()
            self.dominant = "lenc_gemm"
        elif name == "lfm_frontend":
            self.cfg = ae.lfm_config()
            self.frames = sum(ae.ae_lfm_num_frames(self.cfg, n) for n in self.lens)
            self.ws_bytes = ae.ae_lfm_workspace_size(self.cfg, len(self.lens))
            self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")
            self.d_mel = torch.empty((self.frames, self.cfg.n_mels), device="cuda")
            self.h_mel = torch.empty((self.frames, self.cfg.n_mels)).pin_memory()
            self.dominant = "lfm"
        elif name == "frontend":
            self.ws_bytes = ae.ae_workspace_size(None, len(self.lens), self.frames, 0)
            self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")
            self.d_mel = torch.empty((self.frames, 128), device="cuda")
            self.h_mel = torch.empty((self.frames, 128)).pin_memory()
            self.dominant = "logmel"
        elif name == "resample":
            n = synth.RS_RATE * synth.RS_SECONDS
            self.lens = [n] * synth.RS_CLIPS
            self.off = np.arange(synth.RS_CLIPS + 1, dtype=np.int64) * n
            planes = np.empty((2, synth.RS_CLIPS * n), np.float32)
            for k in range(synth.RS_CLIPS):
                ch = synth.resample_clip(k)
                planes[0, k * n:(k + 1) * n] = ch[0]
                planes[1, k * n:(k + 1) * n] = ch[1]
            self.h_x = torch.from_numpy(planes).pin_memory()
            self.d_x = self.h_x.cuda()
            self.n_out = sum(ae.ae_resample_len(v, synth.RS_RATE) for v in self.lens)
            self.d_y = torch.empty(self.n_out, device="cuda")
            self.h_y = torch.empty(self.n_out).pin_memory()
            self.ws_bytes = ae.ae_resample_workspace_size(self.off, synth.RS_RATE, 16000, 2)
            self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")
            self.tokens = self.n_out
            self.audio_s = synth.RS_CLIPS * float(synth.RS_SECONDS)
            self.dominant = "resample"
        elif name == "attention":
            S, T = synth.ATT_SEQS, synth.ATT_T
            p = synth.attention_params()
            R, qs, self.ks = ae.ae_attention_tables(p["relk"], p["pds"])
            self.R, self.qs = torch.from_numpy(R).cuda(), torch.from_numpy(qs).cuda()
            g = torch.Generator(device="cuda").manual_seed(4)
            self.q, self.k, self.v = (torch.randn((S * T, 1024), generator=g, device="cuda").to(torch.bfloat16)
                                      for _ in range(3))
            self.o = torch.empty_like(self.q)
            self.tok_off = np.arange(S + 1, dtype=np.int64) * T
            self.tokens = S * T
            self.audio_s = self.tokens / 25.0
            self.ws_bytes = ae.ae_workspace_size(None, S, 0, self.tokens)
            self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")
            self.dominant = "attention"
        self.flush = torch.empty(L2_FLUSH_BYTES // 4, device="cuda")

    def step(self):
        ae = self.ae
        if self.name in ENCODE_WORKLOADS:
            ae.ae_encode(self.model, self.d_wave, self.off, self.d_out, self.ws, self.ws_bytes, self.stream)
        elif self.name == "frontend":
            ae.ae_logmel(self.d_wave, self.off, self.d_mel, self.ws, self.ws_bytes, self.stream)
        elif self.name == "lfm_frontend":
            ae.ae_lfm_logmel(self.cfg, self.d_wave, self.off, self.d_mel, self.ws, self.ws_bytes, self.stream)
        elif self.name in LFM_ENCODER_WORKLOADS:
            ae.ae_lfm_logmel(self.cfg, self.d_wave, self.off, self.d_mel, self.lfm_ws, self.lfm_ws_bytes, self.stream)
            ae.ae_lenc_encode(self.enc, self.d_mel, self.frame_off, self.d_out, self.ws, self.ws_bytes, self.stream)
        elif self.name == "resample":
            ae.ae_resample(self.d_x, 2, self.d_x.shape[1], self.off, synth.RS_RATE, 16000, self.d_y, self.ws,
                           self.ws_bytes, self.stream)
        else:
            ae.ae_local_attention(self.q, self.k, self.v, 1024, ae.AE_BF16, self.R, self.qs, self.ks, 50.0,
                                  self.tok_off, self.o, 1024, self.ws, self.ws_bytes, self.stream)

    def step_e2e(self):
        """One step through the host-buffer path; returns (h2d bytes, d2h bytes)."""
        ae, torch = self.ae, self.torch
        if self.name in ENCODE_WORKLOADS:
            ae.ae_encode_host(self.model, self.h_wave, self.off, self.h_out, self.ws, self.ws.numel(), self.stream)
            return self.h_wave.numel() * 4, self.h_out.numel() * 4
        if self.name in ("frontend", "lfm_frontend"):
            self.d_wave.copy_(self.h_wave, non_blocking=True)
            self.step()
            self.h_mel.copy_(self.d_mel, non_blocking=True)
            self.stream.synchronize()
            return self.h_wave.numel() * 4, self.h_mel.numel() * 4
        if self.name in LFM_ENCODER_WORKLOADS:
            self.d_wave.copy_(self.h_wave, non_blocking=True)
            self.step()
            self.h_out.copy_(self.d_out, non_blocking=True)
            self.stream.synchronize()
            return self.h_wave.numel() * 4, self.h_out.numel() * 4
        if self.name == "resample":
            self.d_x.copy_(self.h_x, non_blocking=True)
            self.step()
            self.h_y.copy_(self.d_y, non_blocking=True)
            self.stream.synchronize()
            return self.h_x.numel() * 4, self.h_y.numel() * 4
        return 0, 0

    def e2e_pipelined(self, k: int) -> float:
        """k steps through ae_encode_host_async on two streams, each with its own
        workspace and pinned output buffer, so one step's host copies overlap the
        other's kernels; returns the device time of all k steps in ms (events on
        the first stream, after it has joined the second)."""
        ae, torch = self.ae, self.torch
        if not hasattr(self, "ws2"):
            self.ws2 = torch.empty_like(self.ws)
            self.h_out2 = torch.empty_like(self.h_out).pin_memory()
            self.stream2 = torch.cuda.Stream()
        slots = [(self.stream, self.ws, self.h_out), (self.stream2, self.ws2, self.h_out2)]
        torch.cuda.synchronize()
        a, b, j = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a.record(self.stream)
        self.stream2.wait_event(a)
        for i in range(k):
            s, ws, out = slots[i % 2]
            ae.ae_encode_host_async(self.model, self.h_wave, self.off, out, ws, ws.numel(), s)
        j.record(self.stream2)
        self.stream.wait_event(j)
        b.record(self.stream)
        b.synchronize()
        return a.elapsed_time(b)

    def timed(self, k: int, fn):
        torch = self.torch
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(k)]
        for a, b in ev:
            self.flush.zero_()
            a.record(self.stream)
            fn()
            b.record(self.stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in ev)


class OracleRun:
    """The oracle as it stands, timed on the host cores on a bounded sample of
    the workload (inputs prepared outside the timing)."""

    def __init__(self, name: str):
        from oracle import oracle as O
        self.O, self.name = O, name
        try:
            from threadpoolctl import threadpool_info
            self.threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
        except Exception:
            self.threads = os.cpu_count() or 1
        if name in ENCODE_WORKLOADS:
            self.W = synth.model_weights(data_of(name))
            if name == "tower_fp8":
                self.W = O.fp8_weights(self.W)
            self.lens = synth.clip_lengths(data_of(name))
            self.next = 0
        elif name == "resample":
            from oracle import resample as RS
            self.RS = RS
            self.next = 0
        elif name in LFM_ENCODER_WORKLOADS:
            self.next = 0
        elif name == "attention":
            p = synth.attention_params()
            q, k, v = synth.attention_qkv(0, T=2048)
            self.qkv = [x.astype(np.float64) for x in (q, k, v)]
            self.R = O.relative_keys(p["relk"], 12, 1024)
            self.qd = O.softplus(p["pds"])

    def step(self):
        """One bounded unit of work; returns (seconds, audio seconds, description)."""
        O = self.O
        if self.name in ENCODE_WORKLOADS:
            i = self.next % len(self.lens)
            self.next += 1
            c = synth.waves(data_of(self.name), [i])[0]
            t0 = time.perf_counter()
            O.encode([c], self.W)
            dt = time.perf_counter() - t0
            return dt, min(len(c), synth.MAX_SAMPLES) / synth.SAMPLE_RATE, f"clip {i} of the {self.name} workload"
        if self.name == "frontend":
            c = synth.waves(self.name, [0])[0]
            t0 = time.perf_counter()
            O.log_mel(c)
            return time.perf_counter() - t0, 30.0, "clip 0 of the frontend workload (log-mel)"
        if self.name == "lfm_frontend":
            from oracle import lfm as LF
            c = synth.waves("frontend", [0])[0]
            t0 = time.perf_counter()
            LF.features(c)
            return time.perf_counter() - t0, 30.0, "clip 0 of the frontend workload (second front-end)"
        if self.name in LFM_ENCODER_WORKLOADS:
            from oracle import lfm as LF
            from oracle import lfm_encoder as LE
            if not hasattr(self, "lenc_w"):
                self.lenc_w = synth.lfm_encoder_weights()
            data = data_of(self.name)
            i = self.next % len(synth.clip_lengths(data))
            self.next += 1
            c = synth.waves(data, [i])[0]
            t0 = time.perf_counter()
            LE.encode(LF.features(c), self.lenc_w)
            return (time.perf_counter() - t0, min(len(c), synth.MAX_SAMPLES) / synth.SAMPLE_RATE,
                    f"clip {i} of the {data} workload through the LFM2A front-end and encoder")
        if self.name == "resample":
            i = self.next % synth.RS_CLIPS
            self.next += 1
            ch = synth.resample_clip(i)
            t0 = time.perf_counter()
            self.RS.to_mono_16k(ch, synth.RS_RATE)
            return time.perf_counter() - t0, float(synth.RS_SECONDS), f"stereo clip {i} of the resample workload"
        t0 = time.perf_counter()
        O.local_attention_core(*self.qkv, np.arange(2048), self.R, self.qd, 8, 12, 50.0)
        return time.perf_counter() - t0, 2048 / 25.0, "2048 tokens of one attention sequence"


def oracle_baseline(name: str, budget_s: float = 20.0):
    """(audio-s/s, sample description, threads) of the oracle within about budget_s."""
    r = OracleRun(name)
    t = a = 0.0
    n = 0
    while n == 0 or t < budget_s:
        dt, au, _ = r.step()
        t, a, n = t + dt, a + au, n + 1
        if data_of(name) == "tower" and n >= 16:
            break
    return a / t, f"{n} unit(s) of the {name} workload through the f64 oracle ({a:.1f} s of audio)", r.threads


# ------------------------------------------------------------------ arms

def max_over_ranks(value: float, dist, device: str = "cuda") -> float:
    """The largest value over all ranks (every rank gets it); the value itself
    for a single process. The multi-GPU timings are reported this way."""
    if not dist:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: int, dist, device: str = "cuda") -> int:
    """The sum over all ranks (every rank gets it); the value itself for a
    single process. The whole job's kernel launches are counted this way."""
    if not dist:
        return int(value)
    import torch
    t = torch.tensor([int(value)], dtype=torch.int64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return int(t.item())


def whole_job_value(audio_s_per_replica: float, world: int, ms_total: float, steps: int) -> float:
    """Audio seconds per second of the whole job: every rank runs one replica of
    the batch per step (weak scaling), timed as the slowest rank."""
    return audio_s_per_replica * world / (ms_total / steps / 1e3)


def run_ours(args, rank, world, dist):
    import torch
    ours = Ours(args.workload, rank, world)
    ae = ours.ae
    for _ in range(args.warmup):
        ours.step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    with Clocks(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                else int(os.environ.get("LOCAL_RANK", 0))) as clk:
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        n0 = ae.ae_launch_count()
        ms_local = ours.timed(args.steps, ours.step)
        launches_timed = ae.ae_launch_count() - n0  # this library's kernels inside the timed steps
        ms = max_over_ranks(ms_local, dist)
        launches_timed = sum_over_ranks(launches_timed, dist)
        if dist:
            dist.barrier()
    clocks = clk.summary()
    # per-kernel-class timing over a replica of the timed region (events around every launch)
    ae.ae_profile_enable(True)
    ae.ae_profile_read()
    # at most 40 steps: the library keeps 16384 launch records
    prof_steps = min(args.steps, 40)
    ms_prof = ours.timed(prof_steps, ours.step)
    prof = ae.ae_profile_read()
    ae.ae_profile_enable(False)
    # end to end through the host-buffer entry point
    h2d = d2h = 0
    ms_e2e = None
    if args.workload in ENCODE_WORKLOADS:
        ours.e2e_pipelined(2)
        ms_e2e = ours.e2e_pipelined(args.steps)
        h2d, d2h = ours.h_wave.numel() * 4, ours.h_out.numel() * 4
    elif args.workload != "attention":
        ours.step_e2e()
        torch.cuda.synchronize()
        sizes = []

        def e2e():
            sizes.append(ours.step_e2e())
        ms_e2e = ours.timed(args.steps, e2e)
        h2d, d2h = sizes[0]
    if ms_e2e is not None:
        ms_e2e = max_over_ranks(ms_e2e, dist)
    h2d, d2h = sum_over_ranks(h2d, dist), sum_over_ranks(d2h, dist)
    if rank != 0:
        return None
    pk = peaks()
    per_step = ms / args.steps
    if ours.job_audio_s is not None:   # a partitioned global batch
        audio = ours.job_audio_s
        value = audio / (ms / args.steps / 1e3)
        job_tokens = ours.job_tokens
    else:                              # one replica per rank
        audio = ours.audio_s * world
        value = whole_job_value(ours.audio_s, world, ms, args.steps)
        job_tokens = ours.tokens * world
    dom = prof[ours.dominant]
    burst, kind = tensor_peak_kind(clocks)
    if ours.dominant in ("gemm", "gemm_fp8", "lenc_gemm"):
        # e4m3 dense rate = the measured bf16 figure x the nominal ratio 4.5 / 2.25 PFLOP/s
        mult = 2.0 if ours.dominant == "gemm_fp8" else 1.0
        achieved = dom["flops"] / (dom["ms"] / 1e3) / 1e12
        pb, ps = mult * pk["bf16_tflops"], mult * pk["bf16_tflops_sustained"]
        peak = round(pb if burst else ps, 1)
        roof = {"bound": "tensor", "unit": "TFLOP/s",
                "peak_kind": ("e4m3 = 2 x " if mult == 2.0 else "") + f"bf16 {kind} (" + pk["source"] + ")" +
                             ("; nominal ratio 4.5 / 2.25 PFLOP/s" if mult == 2.0 else ""),
                "frac_vs_burst": round(achieved / pb, 4), "frac_vs_sustained": round(achieved / ps, 4)}
    elif ours.dominant == "resample":
        # the FIR is plain FP32 multiply-add: 148 SMs x 128 FP32 lanes x 2 flop at the max SM clock
        sm_mhz = (clocks.get("sm_max_mhz") or 1965.0)
        achieved = dom["flops"] / (dom["ms"] / 1e3) / 1e12
        peak = round(148 * 128 * 2 * sm_mhz * 1e6 / 1e12, 2)
        roof = {"bound": "alu", "unit": "TFLOP/s",
                "peak_kind": f"FP32 FMA from unit counts: 148 SMs x 128 lanes x 2 flop x {sm_mhz:.0f} MHz",
                "note": "achieved counts the FIR's algorithmic flops (2 per tap); at 44.1 kHz the FIR runs as "
                        "tensor-core products of bf16-split inputs and taps (k_rs_fir_tc), so the fraction "
                        "compares it with what the float32 FMA pipe could do"}
    else:
        achieved = dom["bytes"] / (dom["ms"] / 1e3) / 1e9
        peak = pk["hbm_gbs"]
        roof = {"bound": "hbm", "unit": "GB/s", "peak_kind": "HBM copy (" + pk["source"] + ")"}
    traffic, traffic_src = captured_traffic(ours.dominant, args.workload)
    roof.update({"kernel": {"gemm": "k_gemm_tc (all projections)", "logmel": "k_logmel",
                            "lfm": "k_lfm_spec + k_lfm_norm",
                            "lenc_gemm": "k_gemm_tc (the LFM2A encoder's projections)",
                            "gemm_fp8": "k_gemm_tc<e4m3> (FFN W1/W2, q/k/v, lc_start)",
                            "attention": "k_attention_tc",
                            "resample": "k_rs_fir_tc (with its tap matrix and mixdown)"}[ours.dominant],
                 "achieved": round(achieved, 2), "peak": peak, "frac": round(achieved / peak, 4),
                 "traffic": None if traffic is None else round(traffic), "traffic_source": traffic_src,
                 "algorithmic_bytes_per_launch": round(dom["bytes"] / max(dom["launches"], 1)),
                 "launches_per_step": dom["launches"] / prof_steps,
                 "share_of_step": round(dom["ms"] / max(ms_prof, 1e-9), 4)})
    classes = {k: {"ms_per_step": round(v["ms"] / prof_steps, 4), "launches_per_step": v["launches"] / prof_steps,
                   **({"tflops": round(v["flops"] / (v["ms"] / 1e3) / 1e12, 1)} if v["flops"] and v["ms"] else {}),
                   **({"gbs": round(v["bytes"] / (v["ms"] / 1e3) / 1e9, 1)} if v["bytes"] and v["ms"] else {})}
               for k, v in prof.items() if k != "dropped" and v["launches"]}
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": {"frontend": "f32", "lfm_frontend": "f32", "resample": "f32", "lfm_encoder": "bf16", "lfm_ragged": "bf16",
                  "tower_fp8": "e4m3+bf16"}.get(args.workload, "bf16"),
        "data": "synthetic",
        "config": workload_desc(args.workload, (({
            "clips": ours.job_clips, "tokens": ours.job_tokens, "audio_seconds": round(ours.job_audio_s, 3),
            "clips_rank0": len(ours.lens), "tokens_rank0": ours.tokens,
            "parallelism": (f"dp{world}: a global batch of {world} x the workload's clips split by "
                            "ae_partition_clips (greedy token balance), model replicated, no data-path collective")
            if world > 1 else "1 GPU"} if ours.job_audio_s is not None else {
            "clips": len(getattr(ours, "lens", [])) or synth.ATT_SEQS,
            ("output_samples_per_replica" if args.workload == "resample" else "tokens_per_replica"): ours.tokens,
            "audio_seconds_per_replica": round(ours.audio_s, 3), "parallelism": f"replicas x{world}"}) | {
            ("output_samples_per_s" if args.workload == "resample" else "soft_tokens_per_s"):
                round(job_tokens / (per_step / 1e3), 1)})),
        "e2e": None if ms_e2e is None else {
            "value": round(audio / (ms_e2e / args.steps / 1e3), 2), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "api": {"tower": "ae_encode_host_async, two streams (copies of one step overlap the kernels of the other)",
                    "tower_fp8": "ae_encode_host_async, two streams (copies of one step overlap the kernels of the "
                                 "other)",
                    "ragged": "ae_encode_host_async, two streams (copies of one step overlap the kernels of the other)",
                    "frontend": "ae_logmel + copies", "lfm_frontend": "ae_lfm_logmel + copies",
                    "lfm_encoder": "ae_lfm_logmel + ae_lenc_encode + copies",
                    "lfm_ragged": "ae_lfm_logmel + ae_lenc_encode + copies",
                    "resample": "ae_resample + copies"}[args.workload]},
        "gpu_launches": int(launches_timed),
        "roofline": roof,
        "kernel_classes": classes,
        "profiled_ms_per_step": round(ms_prof / prof_steps, 4),
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        v, sample, threads = oracle_baseline(args.workload)
        line["cpu_baseline"] = {"value": round(v, 4), "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": sample}
    return line


def run_reference(args):
    """The base contract's reference arm: the oracle on the host cores, one
    bounded unit of the workload per step (a 30 s clip for the tower)."""
    r = OracleRun(args.workload)
    for _ in range(args.warmup):
        r.step()
    t = a = 0.0
    desc = ""
    for _ in range(args.steps):
        dt, au, desc = r.step()
        t, a = t + dt, a + au
    v = a / t
    return {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * t / args.steps, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_desc(args.workload, {"parallelism": "cpu"}),
            "cpu_baseline": {"value": round(v, 4), "unit": UNIT, "cores": r.threads, "kind": "oracle",
                             "sample": f"one unit per step, e.g. {desc}"},
            "e2e": {"value": round(v, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=("tower", "tower_fp8", "ragged", "frontend", "lfm_frontend", "lfm_encoder",
                                           "lfm_ragged",
                                           "attention", "resample"),
                    default="ragged")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: re-launch this command under torchrun
        import socket
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
               "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
        sys.exit(subprocess.call(cmd))
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    if args.gpus > 1 and world != args.gpus:
        sys.exit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}: launch one rank per GPU")
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    import torch
    dist = None
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        line = run_ours(args, rank, world, dist)
    finally:
        if dist:
            dist.barrier()
            dist.destroy_process_group()
    if rank == 0 and line:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
