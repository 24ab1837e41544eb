/*
 * ae.h -- C ABI of the B200 (sm_100a) audio-encoder forward: 16 kHz waveform
 * -> log-mel -> two-conv subsampling stem -> Conformer layers with causal
 * local attention -> 512-d embedding rows.
 *
 * The operations are those of the gemma4_audio tower as the docs.rs page of
 * cortiq-engine 0.8.49, egemma2_audio.rs, states them (module doc items 1-5,
 * and the functions named beside each call below). Three adjacent parts sit
 * beside it: the channel mixdown and resampling to 16 kHz that precede the
 * front-end (ae_resample), an 8-bit (e4m3) variant of the tower's projections
 * (AE_FP8, ae_linear_e4m3), and the LFM2A encoder's log-mel front-end
 * (ae_lfm_logmel).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Pointers named d_* are CUDA device pointers; h_* are host pointers.
 * - The caller owns every buffer, the workspace and the stream. The library
 *   owns only an ae_model (weights and load-time tables) until
 *   ae_model_destroy.
 * - Clips are packed back to back without padding. A batch of n_clips clips
 *   is described by host int64 offsets [n_clips + 1], non-decreasing,
 *   starting at 0 (samples, frames or tokens depending on the call).
 * - In the tower's calls, clips longer than 480000 samples are cut to their
 *   first 480000 samples (the feature extractor's 30 s truncation), and a
 *   clip of 160 samples or fewer has no frames and no tokens; it is legal and
 *   produces no rows. The resampler and the LFM2A front-end take clips of any
 *   length.
 * - Calls are stream-ordered: they enqueue work on `stream` and return
 *   without waiting for it, except ae_encode_host, which waits. They never
 *   allocate device memory; all scratch space comes from the caller's
 *   workspace (d_ws, ws_bytes), whose size ae_workspace_size (or the
 *   resampler's and the LFM2A front-end's own *_workspace_size) returns. Two
 *   calls that share a workspace must be ordered on one stream.
 * - Every argument is checked on the host before anything is enqueued: null
 *   pointers, a workspace below the required size, offsets that are not
 *   monotone, sizes whose indices would not fit the kernels' 32-bit
 *   arithmetic, and configurations the compiled kernels do not implement.
 *   A refused call returns an error status, writes nothing and enqueues
 *   nothing; ae_last_error() then names the offending argument.
 * - AE_ECUDA reports a CUDA launch or API failure seen by the host when the
 *   work was enqueued. Faults of kernels that already ran are reported by
 *   the CUDA runtime on the next synchronising call, as for any kernel.
 * - There is no CPU fallback: if no CUDA device is usable every compute
 *   call returns AE_ECUDA.
 */
#ifndef AE_H
#define AE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (NULL = the legacy default stream). */
typedef struct CUstream_st *ae_stream;

typedef enum {
  AE_OK = 0,
  AE_EINVAL = 1,        /* a bad argument (null pointer, bad offsets, bad layer index) */
  AE_EUNSUPPORTED = 2,  /* a configuration the compiled kernels do not implement */
  AE_EWORKSPACE = 3,    /* ws_bytes below ae_workspace_size */
  AE_ECUDA = 4,         /* a CUDA API or launch error */
  AE_ENOMEM = 5,        /* device memory for the model could not be allocated */
  AE_EDEVICE = 6        /* a kernel gave up a bounded wait (see ae_device_status) */
} ae_status;

/* Arithmetic of the tower. AE_F32: float32 weights, activations and
 * products (CUDA-core FMA). AE_BF16: bf16 weights and bf16 operands of
 * every projection on the tcgen05 tensor cores with float32 accumulation;
 * the residual stream, norms, attention and convolution arithmetic stay
 * float32. The front-end is float32 in all three.
 *
 * AE_FP8: AE_BF16 with 8-bit projections where the model bounds the input.
 * The page keeps a quantized pack's kernels as an option (egemma2_audio.rs,
 * AudioTower::load, CMF_EGEMMA2_LOWMEM); here the low-precision format is
 * OCP e4m3 on the tcgen05 kind::f8f6f4 path. The page gives no such format,
 * so this arithmetic is this library's, not the page's. FFN W1 and W2, q/k/v and
 * lc_start: each weight row n is stored as e4m3 codes of
 * W[n][k] / s_n, s_n = max_k |W[n][k]| / 448 (1 for an all-zero row),
 * rounded to nearest even from the float32 input in float64 arithmetic.
 * Each input is stored as e4m3 codes of x * q, q = 448 / max(|lo_in|,
 * |hi_in|) of the projection's input clamp, rounded to nearest even from
 * float32. The producing kernel writes them: the row passes for W1,
 * q/k/v and lc_start, and W1's SiLU epilogue for W2. The accumulator
 * column n is multiplied by s_n / q before the epilogue. These projections
 * need finite input bounds (AE_EUNSUPPORTED otherwise). post, lc_end,
 * in_proj, out_proj, embed and conv1 stay bf16. */
typedef enum { AE_F32 = 0, AE_BF16 = 1, AE_FP8 = 2 } ae_dtype;

/* Hyper-parameters of the tower (egemma2_audio.rs, AudioTower::load reads
 * them from audio_config). The kernels are compiled for the release shape:
 * n_mels 128, c0 128, c1 32, hidden 1024, heads 8 (head_dim 128), left 12
 * (attention_context_left 13 minus one), kernel 5; ffn, out_dim and
 * embed_dim must be multiples of 256; n_layers >= 0. Anything else is
 * refused with AE_EUNSUPPORTED. attention_context_right must be 0 in the
 * release and is not a parameter here. */
typedef struct {
  int32_t n_mels, c0, c1, hidden, heads, ffn, left, kernel, out_dim, embed_dim, n_layers;
  float softcap;          /* attention_logit_cap, 50 */
  float residual_weight;  /* FFN half-residual, 0.5 */
} ae_config;

/* Input and output bounds of one clippable projection (Gemma4ClippableLinear,
 * the page's ClipLin): y = clamp(clamp(x, lo_in, hi_in) W^T, lo_out, hi_out).
 * +-INFINITY means unbounded. */
typedef struct { float lo_in, hi_in, lo_out, hi_out; } ae_clip;

/* One Conformer layer's weights as host float32 arrays in the checkpoint's
 * layouts: matrices [out][in] row-major; norm weights [hidden];
 * per_dim_scale [head_dim]; lc_dw [hidden][kernel]. For AE_BF16 every
 * matrix is converted to bf16 by round-to-nearest-even at model creation;
 * for AE_FP8 the e4m3 projections are quantised as described at ae_dtype
 * and the other matrices converted to bf16.
 * q, k and v must share their input bounds (they read the same normalised
 * activations through one fused projection). */
typedef struct {
  const float *ff1_pre, *ff1_w1, *ff1_w2, *ff1_post;
  const float *ff2_pre, *ff2_w1, *ff2_w2, *ff2_post;
  const float *norm_pre_attn, *norm_post_attn, *norm_out;
  const float *q, *k, *v, *post;
  const float *per_dim_scale, *relative_k;
  const float *lc_pre, *lc_start, *lc_dw, *lc_norm, *lc_end;
  ae_clip clip_ff1_w1, clip_ff1_w2, clip_q, clip_k, clip_v, clip_post;
  ae_clip clip_lc_start, clip_lc_end, clip_ff2_w1, clip_ff2_w2;
} ae_host_layer;

/* Stem and head weights (host float32): conv0 [c0][1][3][3], ln0 [c0],
 * conv1 [c1][c0][3][3], ln1 [c1], in_proj [hidden][c1 * n_mels/4],
 * out_proj [out_dim][hidden], out_bias [out_dim], embed [embed_dim][out_dim],
 * layers [n_layers]. */
typedef struct {
  const float *conv0, *ln0, *conv1, *ln1, *in_proj;
  const ae_host_layer *layers;
  const float *out_proj, *out_bias, *embed;
} ae_host_weights;

typedef struct ae_model ae_model;

/* --- sizes (egemma2_audio.rs, num_frames / num_tokens) --------------------- */

/* Mel frames of a clip of n samples: 0 if min(n, 480000) <= 160, else
 * ceil((min(n, 480000) - 160) / 160). Negative n gives 0. */
int64_t ae_num_frames(int64_t n_samples);

/* Soft tokens of a clip of n samples: ceil(ceil(frames / 2) / 2). */
int64_t ae_num_tokens(int64_t n_samples);

/* --- data-parallel partition of a batch ------------------------------------ */

/* Assigns the clips of a batch to n_parts devices (or streams) for
 * data-parallel encoding. Every clip's output rows depend on that clip alone
 * (egemma2_audio.rs, encode_locked: the stem runs per clip, attention spans
 * min(pos + 1, 12) rows of the clip and the depthwise conv stops at its
 * start), so the parts need no exchange, only the model on every device.
 * Greedy token balance: clips in decreasing order of soft tokens
 * (ae_num_tokens of their length; equal counts by lower clip index) each go
 * to the part holding the fewest tokens so far (equal totals by lower part
 * index). The largest part's total then exceeds the smallest one's by at
 * most one clip's tokens (750 at most). Deterministic: every caller that
 * passes the same lengths gets the same assignment, so ranks can compute it
 * independently.
 * h_sample_off: host int64 [n_clips + 1] sample offsets, as for ae_encode.
 * h_part: host int32 [n_clips], receives each clip's part in [0, n_parts).
 * h_tokens: host int64 [n_parts] or NULL, receives each part's token total.
 * n_parts in [1, 65536]. Host only: no device is touched and nothing is
 * enqueued; AE_EINVAL for bad offsets, counts or null pointers. */
ae_status ae_partition_clips(const int64_t *h_sample_off, int n_clips, int n_parts, int32_t *h_part,
                             int64_t *h_tokens);

/* --- model ----------------------------------------------------------------- */

/* Validates cfg and the weight pointers, converts and uploads the weights
 * to the current CUDA device, and computes the load-time tables of each
 * layer (AudioTower::load): softplus(per_dim_scale) with torch's threshold
 * of 20, and the relative keys R = pe relative_k^T of distances
 * 0..left-1 from the sinusoids [sin(d inv) | cos(d inv)],
 * inv_i = exp(-i ln(1e4) / (hidden/2 - 1)), all in float64 on the host and
 * stored as float32. Synchronous. On failure *out is NULL. */
ae_status ae_model_create(const ae_config *cfg, const ae_host_weights *w, ae_dtype dtype,
                          ae_model **out);
void ae_model_destroy(ae_model *m);

/* Bytes of workspace that any call below needs for a batch of n_clips clips
 * holding total_frames mel frames and total_tokens soft tokens in all. With
 * m == NULL: the workspace of ae_logmel and ae_local_attention. */
size_t ae_workspace_size(const ae_model *m, int64_t n_clips, int64_t total_frames,
                         int64_t total_tokens);

/* --- the hot path ------------------------------------------------------------ */

/* Log-mel features (MelFrontend::log_mel): per frame i of each clip,
 * x_j = wave[160 i + j - 160] (0 before the clip) times the periodic Hann
 * window 0.5 - 0.5 cos(2 pi j / 320), j < 320, zero-padded to 512; |rfft|;
 * 128 HTK mel bands over 0-8 kHz without normalisation; ln(mel + 0.001).
 * d_wave: float32 [h_sample_off[n_clips]]. d_mel: float32 [sum frames][128],
 * clip after clip. Workspace: ae_workspace_size(NULL, ...). */
ae_status ae_logmel(const float *d_wave, const int64_t *h_sample_off, int n_clips, float *d_mel,
                    void *d_ws, size_t ws_bytes, ae_stream stream);

/* Subsampling stem plus input projection (AudioTower::subsample and
 * input_proj_linear), per clip: 3x3 stride-2 conv 1 -> c0 with zero pad 1,
 * bias-free LayerNorm over channels (eps 1e-6), ReLU; 3x3 stride-2 conv
 * c0 -> c1, LayerNorm, ReLU; flatten frequency-major (f * c1 + c); times
 * in_proj^T (no bias, no clamp). d_mel: float32 [h_frame_off[n_clips]][128].
 * d_h: float32 [sum tokens][hidden], the residual stream entering layer 0,
 * 16-byte aligned (the projection writes it with TMA stores; AE_EINVAL
 * otherwise). */
ae_status ae_subsample(const ae_model *m, const float *d_mel, const int64_t *h_frame_off,
                       int n_clips, float *d_h, void *d_ws, size_t ws_bytes, ae_stream stream);

/* One Conformer layer in place on the float32 residual stream d_h
 * [h_tok_off[n_clips]][hidden] (the loop body of encode_locked):
 * FFN1 (h += rw * rms_post(W2 silu(W1 rms_pre(h)))), local attention
 * (h += rms_post_attn(post(attn(q, k, v of rms_pre_attn(h))))), where a
 * token sees itself and the left-1 tokens before it in its own clip,
 * q * log2(e)/sqrt(head_dim) * softplus(per_dim_scale), k * log2(1+e),
 * logits q.k + q.R[d] capped by softcap * tanh(z / softcap) and a
 * natural-exp softmax; light conv (h += lc_end(silu(rms(dwconv(glu(
 * lc_start(rms(h)))))))) with a causal depthwise conv that does not reach
 * before the clip start; FFN2; h = rms_norm_out(h). Every ClipLin clamps
 * its input and output. */
ae_status ae_conformer_layer(const ae_model *m, int layer, float *d_h, const int64_t *h_tok_off,
                             int n_clips, void *d_ws, size_t ws_bytes, ae_stream stream);

/* The whole forward (AudioTower::soft_tokens for one packed batch):
 * log-mel, stem, in_proj, every layer, then out_proj + bias, a weightless
 * RMS norm and embed. d_wave: float32 [h_sample_off[n_clips]]. d_out:
 * float32 [sum tokens][embed_dim], clip after clip, 16-byte aligned (the
 * projection writes it with TMA stores; AE_EINVAL otherwise). A batch of 4096
 * to 32768 tokens in two or more clips runs as two half-batches, the second on
 * a stream the model owns, forked from and joined back into `stream` (the
 * rows are those of one pass; larger batches fill the GPU in one pass). */
ae_status ae_encode(const ae_model *m, const float *d_wave, const int64_t *h_sample_off,
                    int n_clips, float *d_out, void *d_ws, size_t ws_bytes, ae_stream stream);

/* ae_encode with per-stage copies, the `trace` of AudioTower::encode_mels
 * (egemma2_audio.rs: the subsampling output, every layer's output and the
 * tower output, all packed), for stage-by-stage comparison. One pass on
 * `stream` (no half-batch split). d_mel (nullable): float32 [sum frames][128],
 * the log-mel rows. d_trace (nullable): float32 [n_layers + 1][sum tokens]
 * [hidden]: slot 0 the residual stream after in_proj, slot l + 1 after layer
 * l. d_out, the workspace and the errors are those of ae_encode; the copies
 * are device-to-device, asynchronous on `stream`. */
ae_status ae_encode_trace(const ae_model *m, const float *d_wave, const int64_t *h_sample_off, int n_clips,
                          float *d_out, float *d_mel, float *d_trace, void *d_ws, size_t ws_bytes,
                          ae_stream stream);

/* ae_encode from host memory to host memory: copies h_wave into the
 * workspace, runs ae_encode, copies the rows back to h_out and waits for
 * the stream. Pinned host buffers make the copies asynchronous DMA. The
 * workspace must hold ae_workspace_size(...) plus the wave and output
 * bytes, rounded up to 256 each: see ae_encode_host_workspace_size. */
size_t ae_encode_host_workspace_size(const ae_model *m, const int64_t *h_sample_off, int n_clips);
ae_status ae_encode_host(const ae_model *m, const float *h_wave, const int64_t *h_sample_off,
                         int n_clips, float *h_out, void *d_ws, size_t ws_bytes, ae_stream stream);

/* ae_encode_host without the final wait: the copies and kernels are only
 * enqueued on `stream`. h_wave, h_out and d_ws belong to the call until the
 * stream has reached this point (synchronize it, or wait on an event recorded
 * after the call). Calls on different streams with their own workspaces and
 * output buffers overlap one batch's copies with another's kernels; each call
 * runs its batch as one pass on its stream (ae_encode and ae_encode_host split
 * a batch of 4096 to 32768 tokens in two halves on two streams instead). */
ae_status ae_encode_host_async(const ae_model *m, const float *h_wave, const int64_t *h_sample_off,
                               int n_clips, float *h_out, void *d_ws, size_t ws_bytes, ae_stream stream);

/* --- the attention core alone ------------------------------------------------ */

/* Load-time tables of one attention layer on the host in float64, stored
 * float32: h_R [left][hidden] = rows 0..left-1 of pe relative_k^T, and
 * h_qscale [hidden/heads] = log2(e)/sqrt(head_dim) * softplus(per_dim_scale).
 * *k_scale = log2(1 + e). */
ae_status ae_attention_tables(const float *h_relative_k, const float *h_per_dim_scale, int hidden,
                              int heads, int left, float *h_R, float *h_qscale, float *k_scale);

/* The attention core of the page's `attention` on clamped projections:
 * o_t = sum_{d <= min(pos_t, left-1)} softmax_d(cap tanh((q_t s) . (k_scale
 * k_{t-d}) + (q_t s) . R[d]) / cap)) v_{t-d} per head, s = d_qscale.
 * d_q/d_k/d_v: [total_tokens][hidden] rows with a stride of ld_qkv
 * elements, bf16 (dtype AE_BF16) or float32 (AE_F32); d_out the same type,
 * [total_tokens][ld_out]. d_R: float32 [left][hidden]; d_qscale: float32
 * [head_dim]. Requires hidden 1024, heads 8, left 12. Token offsets per
 * sequence h_tok_off [n_clips + 1]. Workspace: ae_workspace_size(NULL, ...). */
ae_status ae_local_attention(const void *d_q, const void *d_k, const void *d_v, int64_t ld_qkv,
                             ae_dtype dtype, const float *d_R, const float *d_qscale,
                             float k_scale, float softcap, const int64_t *h_tok_off, int n_clips,
                             void *d_out, int64_t ld_out, void *d_ws, size_t ws_bytes,
                             ae_stream stream);

/* --- one e4m3 projection alone ------------------------------------------------- */

/* Output of ae_linear_e4m3. */
typedef enum { AE_LIN_BF16 = 0, AE_LIN_SILU_E4M3 = 1 } ae_lin_out;

/* The projection kernel of AE_FP8 models on its own (tcgen05 kind::f8f6f4,
 * CTA pairs): acc[m][n] = sum_k x[m][k] w[n][k] in float32 over e4m3
 * operands, then per output column n the factor cs[n] (the weight row's scale
 * over the input's code scale), then:
 *   AE_LIN_BF16:      y [M][N] bf16 = clamp(acc cs, lo, hi)
 *   AE_LIN_SILU_E4M3: y [M][N] e4m3 codes of
 *                     clamp(silu(clamp(acc cs, lo, hi)), lo2, hi2) * q_out
 *                     (nearest even, magnitudes beyond 448 saturated)
 * (the epilogues of q/k/v and FFN W2, and of FFN W1, which writes W2's input).
 * d_x [M][K] and d_w [N][K]: e4m3 codes (OCP E4M3: sign, 4 exponent bits with
 * bias 7, 3 mantissa bits; the patterns 0x7F and 0xFF are NaN), row-major,
 * device memory, 16-byte aligned; d_cs [N] float32, 16-byte aligned; d_y
 * 32-byte aligned. K a positive multiple of 128 up to 65536, N a positive
 * multiple of 256 up to 65536, 0 <= M < 2^31. The caller owns every buffer;
 * nothing is allocated. Arguments are checked before anything is enqueued
 * (AE_EINVAL); launch errors give AE_ECUDA. Asynchronous on `stream`. */
ae_status ae_linear_e4m3(const void *d_x, const void *d_w, const float *d_cs, int64_t M, int32_t N, int32_t K,
                         float lo, float hi, ae_lin_out out, float lo2, float hi2, float q_out, void *d_y,
                         ae_stream stream);

/* --- log-mel without a caller workspace ---------------------------------------- */

/* ae_logmel for callers that cannot allocate device memory at all: code that
 * runs where the allocator must not be entered (a real-time audio callback,
 * an inference host whose device memory belongs entirely to its own pool
 * allocator, a plugin that is handed only its input and output buffers). It
 * computes exactly what ae_logmel computes, but keeps its only scratch data,
 * the per-call clip tables, in a fixed array inside the library (128 KiB in
 * the device memory of every GPU that loads the library, held until the
 * process exits) instead of a workspace. The pages have no counterpart: the
 * reference front-end runs on the host.
 *
 * d_wave, h_sample_off, n_clips, d_mel and stream mean what they mean for
 * ae_logmel. At most 4000 clips per call; more is refused with AE_EINVAL
 * before anything is enqueued. The call calls no cudaMalloc or cudaFree.
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture. The address is kept per device with the CUDA
 * context it belongs to: after cudaDeviceReset (a new context) the next call
 * looks it up again, and that call, too, must come before any capture. Every call uses the same array and rewrites the
 * part it reads, so calls that may overlap on the GPU (on different streams,
 * or from several host threads) race with each other: order them on one
 * stream. */
ae_status ae_logmel_noalloc(const float *d_wave, const int64_t *h_sample_off, int n_clips, float *d_mel,
                            ae_stream stream);

/* --- second log-mel front-end (LFM2A) ------------------------------------------- */

/* The front-end of the LFM2A audio encoder as the page of its GPU port lays it
 * out (log_mel_spectrogram_gpu: stft_frames, power_spec, mel_project,
 * mel_norm): frames of n_fft samples every hop samples with n_fft / 2 samples
 * of zero padding per side (1 + N / hop frames for N > 0 samples, none for
 * N = 0); pre-emphasis y[n] = x[n] - preemph x[n-1] on the clip (x[-1] = 0);
 * a periodic Hann window of win_length samples centred in the n_fft-wide
 * frame; the power spectrum |X_k|^2, k = 0 .. n_fft / 2; a Slaney mel
 * filterbank (librosa's default: Slaney scale, points evenly spaced from 0 to
 * sample_rate / 2, triangles scaled by 2 / (f_{b+2} - f_b)); ln(max(mel,
 * log_floor)); then per band (v - mean) / sqrt(var + var_eps) with the mean
 * and biased variance of the first ceil(N / hop) frames (those whose centre
 * lies in the clip) and zeros for the rest. The page names these constants
 * but gives no values; ae_lfm_default_config fills in the ones this library
 * takes (16 kHz, n_fft 512, window 400, hop 160, 128 bands, pre-emphasis
 * 0.97, floor 2^-24, variance epsilon 1e-5). */
typedef struct {
  int32_t sample_rate, n_fft, win_length, hop, n_mels;
  float preemph, log_floor, var_eps;
} ae_lfm_config;

void ae_lfm_default_config(ae_lfm_config *cfg);

/* Frames of a clip of n samples: 1 + n / hop for n > 0, else 0 (-1 for an
 * invalid cfg). */
int64_t ae_lfm_num_frames(const ae_lfm_config *cfg, int64_t n_samples);

/* Workspace bytes of ae_lfm_logmel for n_clips clips (0 for an invalid cfg). */
size_t ae_lfm_workspace_size(const ae_lfm_config *cfg, int n_clips);

/* d_wave: packed float32 clips (device), clip i = [h_sample_off[i],
 * h_sample_off[i+1]); d_out: [total frames][n_mels] float32, time-major,
 * clips back to back (16-byte aligned). Supported: n_fft 512; win_length and
 * hop even, 2 <= win_length <= 512, 2 <= hop <= 320; 1 <= n_mels <= 128 with
 * at most 32 nonzero bins per band; sample_rate in [1000, 1000000];
 * log_floor > 0, var_eps > 0 (a silent band would divide 0 by 0), all finite (AE_EINVAL or AE_EUNSUPPORTED
 * otherwise, before anything is enqueued). At most 2^31 - 1 frames in all.
 * Asynchronous on `stream`; no allocation. */
ae_status ae_lfm_logmel(const ae_lfm_config *cfg, const float *d_wave, const int64_t *h_sample_off, int n_clips,
                        float *d_out, void *d_ws, size_t ws_bytes, ae_stream stream);

/* --- LFM2A Conformer encoder ---------------------------------------------------- */

/* The Conformer body of the LFM2A audio encoder as the page of its GPU port
 * runs it (cera 0.5.3, audio_encoder_gpu.rs: encode_audio_gpu, macaron_ffn,
 * conv_stem_gpu with STEM_LAYER_MODES / STEM_RELU_AFTER, and the ops of the
 * AudioEncoderGpuOps trait), from a log-mel spectrogram such as
 * ae_lfm_logmel's:
 *   stem: 3x3 stride-2 conv 1 -> C (+bias, ReLU), depthwise 3x3 stride 2
 *   (+bias), pointwise C -> C (+bias, ReLU), depthwise 3x3 stride 2 (+bias),
 *   pointwise C -> C (+bias, ReLU), all with zero padding 1 per side; the
 *   (channel, time, freq) result flattened to (time, channel * freq) and
 *   pre_encode_out (+bias) to n_embd;
 *   n_layers blocks, each: x += 0.5 FFN(LN(x)) with FFN = down(silu(up(.)
 *   + b) ) + b; a = LN(x); q, k, v = linear + bias; p = pos_emb W_pos^T (no
 *   bias); x += o(attn) + b_o, where attn is Transformer-XL attention,
 *   softmax_j(((q_i + u) . k_j + (q_i + v) . p_{i-j}) / sqrt(head_dim)) v_j
 *   over the keys of the clip; conv module: g = GLU(pw1(LN(x)) + b) (first
 *   half times sigmoid of the second), a depthwise conv over time of k taps
 *   (pad (k - 1) / 2 left, the rest right, within the clip) + bias, a
 *   per-channel affine, SiLU, x += pw2(.) + b; x += 0.5 FFN2(LN(x)); x =
 *   LN(x);
 *   adapter: out = down(gelu_erf(up(LN(x)) + b)) + b (erf-form GELU).
 * LayerNorms use the biased variance and their weight and bias. pos_emb has
 * 2 t - 1 rows for relative positions t - 1 .. -(t - 1), row p holding
 * sin(p w_i), cos(p w_i) in columns 2i, 2i + 1, w_i = 10000^(-2i / n_embd);
 * the page shows neither this table nor the attention's relative shift, so
 * both are this library's reading of them. Projections run as bf16 tcgen05
 * GEMMs with float32 accumulation; the residual stream, norms and softmax are
 * float32. The kernels are compiled for n_mels 128, n_embd 512, n_head 8
 * (head_dim 64), stem channels 256; n_ff, adapter_ff and llm_hidden multiples
 * of 256; 1 <= conv_k <= 33; n_layers >= 0; at most 4096 rows after the stem
 * per clip (AE_EUNSUPPORTED otherwise). */
typedef struct {
  int32_t n_mels, n_embd, n_head, n_layers, n_ff, conv_k, stem_ch, adapter_ff, llm_hidden;
  float eps;  /* LayerNorm epsilon */
} ae_lenc_config;

/* One block's weights, host float32, matrices [out][in] row-major: the FFN's
 * up [n_ff][n_embd] and down [n_embd][n_ff], q/k/v/o and pw2 [n_embd][n_embd],
 * linear_pos [n_embd][n_embd], pw1 [2 n_embd][n_embd], dw [conv_k][n_embd]
 * (taps first); every vector [n_embd] except up_b [n_ff] and pw1_b
 * [2 n_embd]. norm_conv_* is the conv module's LayerNorm, conv_norm_* its
 * per-channel affine. */
typedef struct {
  const float *ffn1_norm_w, *ffn1_norm_b, *ffn1_up_w, *ffn1_up_b, *ffn1_down_w, *ffn1_down_b;
  const float *ln1_w, *ln1_b;
  const float *q_w, *q_b, *k_w, *k_b, *v_w, *v_b, *o_w, *o_b;
  const float *linear_pos_w, *pos_bias_u, *pos_bias_v;
  const float *norm_conv_w, *norm_conv_b, *pw1_w, *pw1_b, *dw_w, *dw_b, *conv_norm_w, *conv_norm_b, *pw2_w, *pw2_b;
  const float *ffn2_norm_w, *ffn2_norm_b, *ffn2_up_w, *ffn2_up_b, *ffn2_down_w, *ffn2_down_b;
  const float *ln2_w, *ln2_b;
} ae_lenc_host_block;

/* Stem weights [C][1][3][3] (layers 0, 1, 3) and [C][C] (layers 2, 4) with
 * biases [C]; pre_encode_out [n_embd][C * n_mels / 8] with columns in the
 * page's (channel, freq) order, bias [n_embd]; blocks [n_layers]; adapter
 * LayerNorm [n_embd], up [adapter_ff][n_embd] + [adapter_ff], down
 * [llm_hidden][adapter_ff] + [llm_hidden]. */
typedef struct {
  const float *stem_w[5], *stem_b[5];
  const float *pre_w, *pre_b;
  const ae_lenc_host_block *blocks;
  const float *ad_norm_w, *ad_norm_b, *ad_up_w, *ad_up_b, *ad_down_w, *ad_down_b;
} ae_lenc_host_weights;

typedef struct ae_lenc ae_lenc;

/* The sizes the page names without values, as this library reads them: 128
 * mels, n_embd 512, 8 heads, 17 layers, n_ff 2048, conv_k 9, 256 stem
 * channels, adapter_ff 2048, llm_hidden 2048, eps 1e-5. */
void ae_lenc_default_config(ae_lenc_config *cfg);

/* Rows after the stem for a clip of n_frames mel frames: three times
 * ceil(n / 2) (0 for n_frames <= 0). */
int64_t ae_lenc_num_tokens(int64_t n_frames);

/* Validates cfg and the pointers, converts the matrices to bf16 and uploads
 * everything to the current device. Synchronous; *out is NULL on failure. */
ae_status ae_lenc_create(const ae_lenc_config *cfg, const ae_lenc_host_weights *w, ae_lenc **out);
void ae_lenc_destroy(ae_lenc *m);

/* Workspace bytes of ae_lenc_stem / ae_lenc_encode for clips with these mel
 * frame offsets, and of ae_lenc_block for these token offsets (0 for invalid
 * offsets). */
size_t ae_lenc_workspace_size(const ae_lenc *m, const int64_t *h_frame_off, int n_clips);
size_t ae_lenc_block_workspace_size(const ae_lenc *m, const int64_t *h_tok_off, int n_clips);

/* The stem and pre_encode_out per clip: d_mel float32 [h_frame_off[n]][128]
 * -> d_x float32 [sum tokens][n_embd] (16-byte aligned). */
ae_status ae_lenc_stem(const ae_lenc *m, const float *d_mel, const int64_t *h_frame_off, int n_clips, float *d_x,
                       void *d_ws, size_t ws_bytes, ae_stream stream);

/* Block `layer` in place on d_x float32 [h_tok_off[n]][n_embd] (16-byte
 * aligned); attention within each clip. */
ae_status ae_lenc_block(const ae_lenc *m, int layer, float *d_x, const int64_t *h_tok_off, int n_clips,
                        void *d_ws, size_t ws_bytes, ae_stream stream);

/* The whole body: stem, every block, adapter. d_out float32 [sum tokens]
 * [llm_hidden], clip after clip (16-byte aligned). A clip with no tokens gives
 * no rows. Asynchronous on `stream`; nothing is allocated. */
ae_status ae_lenc_encode(const ae_lenc *m, const float *d_mel, const int64_t *h_frame_off, int n_clips,
                         float *d_out, void *d_ws, size_t ws_bytes, ae_stream stream);

/* --- input conditioning: mixdown and resampling -------------------------------- */

/* Output length of ae_resample for one clip of n_samples at rate_in:
 * n_samples when the rates are equal or n_samples is 0, else
 * ceil(p * n_samples / o) with o = rate_in / g, p = rate_out / g, g their
 * gcd (egemma2_audio.rs, resample_hq: the length of its output). -1 for
 * a negative count or a rate outside 1 .. 1000000. */
int64_t ae_resample_len(int64_t n_samples, int32_t rate_in, int32_t rate_out);

/* Workspace bytes ae_resample needs for these clips, rates and channel
 * count (0 for invalid arguments): clip tables, the per-phase taps
 * (rate_out / g rows) and, for more than one channel, the mixed-down input. */
size_t ae_resample_workspace_size(const int64_t *h_sample_off, int n_clips, int32_t rate_in, int32_t rate_out,
                                  int channels);

/* Channel mixdown and band-limited resampling, per clip (egemma2_audio.rs,
 * to_mono_16k and resample_hq):
 *   mono[i] = (x_0[i] + x_1[i] + ... + x_{C-1}[i]) / C, float32 adds in
 *   channel order and a float32 division (one channel passes unchanged);
 *   y[n] = sum over inputs m with |t| < 64 of mono[m] c sinc(t)
 *          I0(12.8 sqrt(1 - (t/64)^2)) / I0(12.8),
 *   t = (m - n o / p) c, c = 0.958 min(o, p) / o, inputs outside the clip 0,
 * for n < ae_resample_len(N, rate_in, rate_out). The taps are evaluated in
 * float64. Where a row of N = 16 p / gcd(p, 16) outputs (the taps repeat
 * from one row to the next) holds at most 160 and its window at most 4096
 * inputs (44.1, 48, 32, 24, 96 and 8 kHz among the common rates), the sums
 * run on the tensor cores: inputs and taps each split into two bf16 parts
 * (v = hi + lo to about 2^-18), the four products of the parts accumulated
 * in float32. Other rates apply the taps in float32 with float32
 * accumulation in two interleaved partial sums. Either way, against the
 * float64 definition the error stays below (L / 2 + 2) 2^-24 x 2.7 x
 * max |mono| with L = 2 ceil(64 / c) + 3 (2.7 bounds the taps' absolute
 * sum): 3e-5 x max |mono| from 48 kHz, 6e-5 from 96 kHz. Equal rates copy
 * mono.
 * d_x: float32, channel ch of the packed clips at d_x + ch * ch_stride
 * (ch_stride >= h_sample_off[n_clips] when channels > 1), clip k at
 * [h_sample_off[k], h_sample_off[k+1]) in every channel. channels 1 .. 64.
 * d_y: float32, clip k's outputs at the sum of the lengths of clips 0..k-1.
 * Workspace: ae_resample_workspace_size(...), 256-byte aligned. Caller owns
 * every buffer; nothing is allocated; the call is asynchronous on stream.
 * Rates whose reduced output rate p makes the tap table exceed 2^26 entries
 * are refused with AE_EUNSUPPORTED. Co-prime rates (large o) are computed
 * from global memory, correctly but more slowly. */
ae_status ae_resample(const float *d_x, int channels, int64_t ch_stride, const int64_t *h_sample_off, int n_clips,
                      int32_t rate_in, int32_t rate_out, float *d_y, void *d_ws, size_t ws_bytes,
                      ae_stream stream);

/* --- kernel timing ------------------------------------------------------------ */

/* Classes of the kernels the calls launch. */
typedef enum {
  AE_K_TABLES = 0,   /* per-call clip tables and token positions */
  AE_K_LOGMEL = 1,   /* fused log-mel front-end */
  AE_K_CONV0 = 2,    /* stem conv0 + LayerNorm + ReLU */
  AE_K_CONV1 = 3,    /* stem conv1 + LayerNorm + ReLU (implicit GEMM) */
  AE_K_GEMM = 4,     /* the f32 and bf16 projections (tcgen05 for AE_BF16, AE_FP8) */
  AE_K_ATTENTION = 5,
  AE_K_LCONV = 6,    /* depthwise conv + RMS norm + SiLU */
  AE_K_ROWOP = 7,    /* residual / RMS-norm row passes */
  AE_K_RESAMPLE = 8, /* mixdown, resampler taps and FIR */
  AE_K_GEMM_FP8 = 9, /* the e4m3 projections of AE_FP8 (tcgen05 kind::f8f6f4) */
  AE_K_LFM = 10,     /* the second log-mel front-end (spectrum, bands, normalisation) */
  AE_K_LENC_GEMM = 11,      /* the LFM2A encoder's projections (tcgen05, bf16) */
  AE_K_LENC_ATTENTION = 12, /* its Transformer-XL attention */
  AE_K_LENC_ROW = 13,       /* its stem convolutions, LayerNorms, conv-module middle, position table */
  AE_K_COUNT = 14
} ae_kernel_class;

/* Kernel timing for measurement (the analogue of the page's
 * CMF_EGEMMA2_PROF split). While enabled, every call records a CUDA event
 * pair on its stream around each kernel it launches, together with the
 * launch's algorithmic work: flops for the projections and conv1 (2 M N K),
 * bytes that must cross DRAM for the others (inputs read once, outputs
 * written once). Enabling allocates the event pool (up to 16384 launches
 * between reads); the calls themselves still allocate nothing. Not
 * thread-safe: enable, call and read from one thread. */
ae_status ae_profile_enable(int on);

/* Synchronises the device, then returns per class (arrays of AE_K_COUNT)
 * the summed event milliseconds, launch counts, flops and bytes since the
 * last read, and resets them. Any output pointer may be NULL. *dropped
 * (if not NULL) receives the launches not timed because the pool was full. */
ae_status ae_profile_read(double *ms, int64_t *launches, double *flops, double *bytes, int64_t *dropped);

/* --- diagnostics ------------------------------------------------------------- */

/* Number of kernels this library has launched since it was loaded (every call,
 * thread and device; launches the CUDA runtime refused are not counted). Read
 * it before and after a region to count the region's launches. */
uint64_t ae_launch_count(void);


/* Message of the last failed call on this thread ("" if none). */
const char *ae_last_error(void);

/* Synchronises the current device and reports whether a kernel of this
 * library gave up a bounded wait since the last call (AE_EDEVICE), or the
 * device reported an error (AE_ECUDA); clears the library's flag. */
ae_status ae_device_status(void);

/* Exercises the failure path of the kernels' bounded waits without a fault:
 * enqueues one CTA that waits, with the same bounded wait the kernels use,
 * on a shared-memory barrier that completes only if `arrive` is nonzero. If
 * it does not, the wait gives up after limit_us microseconds and records the
 * timeout, so that the next ae_device_status returns AE_EDEVICE (and clears
 * it) while the context stays usable. limit_us in [1, 1000000] (AE_EINVAL
 * otherwise). Asynchronous on `stream`. */
ae_status ae_selftest_bounded_wait(uint32_t limit_us, int arrive, ae_stream stream);

/* Version of the library, "major.minor.patch". */
const char *ae_version(void);

#ifdef __cplusplus
}
#endif
#endif /* AE_H */
