// Internal declarations of the audio-encoder library: the device-resident
// model, the workspace layout and the kernel launchers. Not part of the ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <type_traits>
#include <string>
#include <vector>

#include "../../include/ae.h"

namespace ae {

using bf16 = __nv_bfloat16;

// Shapes the kernels are compiled for (the release tower).
constexpr int kMels = 128;        // mel bands
constexpr int kFrame = 320;       // window
constexpr int kHop = 160;         // hop
constexpr int kFft = 512;         // FFT size
constexpr int kMaxSamples = 480000;
constexpr int kC0 = 128;          // conv0 channels
constexpr int kC1 = 32;           // conv1 channels
constexpr int kF1 = 64;           // frequency rows after conv0
constexpr int kF2 = 32;           // frequency rows after conv1
constexpr int kHidden = 1024;
constexpr int kHeads = 8;
constexpr int kHeadDim = 128;
constexpr int kLeft = 12;         // attention span (itself + 11 before)
constexpr int kKernel = 5;        // depthwise taps

// Output modes of the GEMM epilogue.
enum EpiMode : int {
  EPI_F32 = 0,        // v = clamp(acc + bias) -> float
  EPI_BF16 = 1,       // v = clamp(acc) -> act
  EPI_SILU = 2,       // v = clamp2(silu(clamp(acc))) -> act
  EPI_GLU = 3,        // columns (2c, 2c+1) -> clamp, a * sigmoid(b) -> act column c
  EPI_ADD_F32 = 4,    // out += clamp(acc): a float residual update, one add per element
  EPI_SILU_Q8 = 5,    // v = clamp2(silu(clamp(acc))) -> e4m3 code of v * q8 (the next projection's operand)
  EPI_BIAS_BF16 = 6,     // v = clamp(acc + bias) -> bf16
  EPI_BIAS_SILU = 7,     // v = silu(acc + bias) -> bf16
  EPI_BIAS_GLU = 8,      // columns (2c, 2c+1) + bias -> a * sigmoid(b) -> bf16 column c
  EPI_BIAS_GELU = 9,     // v = gelu_erf(acc + bias) -> bf16
  EPI_BIAS_ADD_F32 = 10, // out += alpha * (acc + bias): a float residual update
};

struct EpiArgs {
  void *out;          // output base
  int64_t ld;         // output row stride in elements
  const float *bias;  // [N] or null
  float lo, hi;       // first clamp
  float lo2, hi2;     // clamp after the activation (EPI_SILU, EPI_SILU_Q8)
  int clamp2;         // 0 when that clamp cannot bind (silu_clamp_binds)
  int seg_w;          // if > 0: columns [s*seg_w, (s+1)*seg_w) use seg_lo/hi[s] as the first clamp
  float seg_lo[3], seg_hi[3];
  const float *cs;    // e4m3 projections: [N] factor of each accumulator column (weight row scale / q8 of x)
  float q8;           // EPI_SILU_Q8: scale of the e4m3 output codes
  float alpha;        // EPI_BIAS_ADD_F32: weight of the update
};

// Device copy of one layer.
struct LayerDev {
  float *ff1_pre, *ff1_post, *ff2_pre, *ff2_post;
  float *norm_pre_attn, *norm_post_attn, *norm_out, *lc_pre, *lc_norm;
  float *lc_dw;               // [hidden][kernel]
  float *R;                   // [left][hidden]
  float *qscale;              // [head_dim]: q_scale * softplus(per_dim_scale)
  void *ff1_w1, *ff1_w2, *ff2_w1, *ff2_w2;
  void *qkv;                  // [3*hidden][hidden]: q, k, v rows stacked
  void *post, *lc_end;
  void *lc_start;             // [2*hidden][hidden], rows interleaved (a_0, b_0, a_1, b_1, ...)
  ae_clip c_ff1_w1, c_ff1_w2, c_ff2_w1, c_ff2_w2, c_q, c_k, c_v, c_post, c_lc_start, c_lc_end;
  // tensor maps of the weight operands (bf16 only)
  CUtensorMap tm_ff1_w1, tm_ff1_w2, tm_ff2_w1, tm_ff2_w2, tm_qkv, tm_post, tm_lc_start, tm_lc_end;
  // AE_FP8: FFN W1/W2, q/k/v and lc_start hold e4m3 codes (the maps above are
  // 8-bit maps then); cs_* are their accumulator column factors, q8_* the
  // scales of their e4m3 inputs (448 over the input clamp's larger bound)
  float *cs_ff1_w1, *cs_ff1_w2, *cs_ff2_w1, *cs_ff2_w2, *cs_qkv, *cs_lc_start;
  float q8_ff1_w1, q8_ff1_w2, q8_ff2_w1, q8_ff2_w2, q8_qkv, q8_lc_start;
};

}  // namespace ae

struct ae_model {
  ae_config cfg;
  ae_dtype dtype;
  int device;
  float k_scale;
  // stem
  float *conv0c;    // [c0][9] (taps minus their channel mean) x LayerNorm gain: the norm's mean is linear in the patch
  float *conv0cov;  // [9][9] channel covariance of the taps: LayerNorm variance = p^T C p
  void *conv0b;     // [c0][64] bf16: conv0c split as (hi, lo, hi, 0...) per row, the B operand of k_conv0_tc
  float *ln0, *ln1;
  void *conv1;      // [c1][9 * c0], k = (dt * 3 + df) * c0 + c
  void *in_proj;    // [hidden][1024]
  void *out_proj;   // [out_dim][hidden]
  float *out_bias;
  void *embed;      // [embed_dim][out_dim]
  CUtensorMap tm_conv1, tm_in_proj, tm_out_proj, tm_embed;
  std::vector<ae::LayerDev> layers;
  std::vector<void *> allocs;
  // ae_encode runs the two halves of a large batch on the caller's stream and
  // on a side stream (fork and join through events), so that the tail waves
  // of one half's kernels overlap the other's. Consecutive calls take the two
  // side streams in turn, so that calls pipelined on two caller streams do
  // not queue their second halves behind each other. The mutex keeps each
  // call's fork/join sequence whole.
  cudaStream_t side[2] = {nullptr, nullptr};
  cudaEvent_t fork[2] = {nullptr, nullptr}, join[2] = {nullptr, nullptr};
  int next_side = 0;
  std::mutex split_mu;
};

namespace ae {

// Per-call clip tables, computed on the host from the caller's offsets.
struct ClipTables {
  int n_clips = 0;
  int64_t total_samples = 0, total_frames = 0, total_tokens = 0, stem_rows = 0;
  int64_t mel_tiles = 0, conv1_tiles = 0;
  std::vector<int64_t> sample_off;  // [B+1]
  std::vector<int32_t> frame_off, tok_off, stem_off, mel_tile_off, conv1_tile_off;  // [B+1]
};

// Device view of the tables (inside the workspace).
struct ClipTablesDev {
  int n_clips;
  const int64_t *sample_off;
  const int32_t *frame_off, *tok_off, *stem_off, *mel_tile_off, *conv1_tile_off;
  const int32_t *pos;  // [total_tokens]
};

// Workspace carve-up. Every region is 256-byte aligned.
struct WsLayout {
  size_t tables = 0, pos = 0, mel = 0, y0 = 0, xs = 0, h = 0, a = 0, big = 0, y = 0, o = 0;
  size_t total = 0;
};

constexpr int kMelTile = 32;       // frames per log-mel work item
constexpr int kConv1TileTok = 4;   // tokens per conv1 tile (4 x 32 frequency rows = 128 GEMM rows)

WsLayout ws_layout(const ae_model *m, int64_t n_clips, int64_t frames, int64_t tokens, bool with_model);

// launchers (return cudaError_t of the launch)
cudaError_t launch_upload_tables(const ClipTables &t, void *ws, const WsLayout &L, ClipTablesDev *dev,
                                 bool with_pos, cudaStream_t s);
size_t tables_bytes(int64_t n_clips);
cudaError_t launch_logmel(const float *wave, float *mel, const ClipTablesDev &t, int64_t mel_tiles,
                          cudaStream_t s);
cudaError_t launch_conv0(const ae_model *m, const float *mel, void *y0, const ClipTablesDev &t,
                         int64_t stem_rows, cudaStream_t s);
cudaError_t launch_conv1(const ae_model *m, const void *y0, int64_t stem_rows, void *xs,
                         const ClipTablesDev &t, int64_t conv1_tiles, int64_t tokens, cudaStream_t s);

// y = epilogue(x W^T); x [M][K] act, W [N][K]. For bf16 the caller passes
// the weight's tensor map (or null to build one).
cudaError_t gemm(const ae_model *m, const void *x, int64_t M, int K, const void *w, const CUtensorMap *tmW,
                 int N, int mode, const EpiArgs &ep, cudaStream_t s);
// The same on e4m3 operands (tcgen05 kind::f8f6f4): x [M][K] codes, the
// weight's 8-bit tensor map; ep.cs scales the accumulator columns.
cudaError_t gemm_e4m3(const void *x, int64_t M, int K, const CUtensorMap &tmW, int N, int mode, const EpiArgs &ep,
                      cudaStream_t s);

// Row update of the residual stream (one warp per row of `width` floats):
//   if y:      h += s * (y_norm ? rms(y) * wy : y)   (y in the model's act type)
//   if w_out:  h = rms(h) * w_out
//   write h back if anything changed it
//   if a_out:  a = clamp(rms(h) * w_next, lo, hi)  (act type of the model;
//              e4m3 codes of a * a_q8 when a_q8 > 0)
struct RowArgs {
  float *h; const void *y; const float *wy; float s; int y_norm;
  const float *w_out;
  void *a_out; const float *w_next; int a_rms; float lo, hi; float a_q8;
  int width; int64_t rows;
};
cudaError_t launch_rowop(const ae_model *m, const RowArgs &r, cudaStream_t s);

// Light-conv middle: c = clamp(silu(rms(dwconv(gl)) * w_norm), lo, hi).
cudaError_t launch_lconv(const ae_model *m, const void *gl, const float *w_dw, const float *w_norm,
                         float lo, float hi, void *out, const int32_t *pos, int64_t T, cudaStream_t s);

// Attention core; q/k/v rows of `ld` elements; output clamped to [lo, hi].
cudaError_t launch_attention(bool is_bf16, const void *q, const void *k, const void *v, int64_t ld,
                             const float *R, const float *qscale, float k_scale, float cap, const int32_t *pos,
                             int64_t T, void *out, int64_t ld_out, float lo, float hi, cudaStream_t s);

// Tensor-map encoding (driver entry point looked up at run time).
bool make_tmap_2d_bf16(CUtensorMap *tm, const void *base, uint64_t inner, uint64_t outer,
                       uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer);
bool make_tmap_2d_u8(CUtensorMap *tm, const void *base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                     uint32_t box_inner, uint32_t box_outer);
bool make_tmap_stem_y0(CUtensorMap *tm, const void *y0, int64_t stem_rows);

// Kernels this library has launched (ae_launch_count), all threads and devices.
std::atomic<uint64_t> &launch_counter();

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device. The attribute belongs to the device, so `done` keeps one bit per
// device index (0..63) whose attribute is already set; the call is
// thread-safe (setting it twice is harmless). Devices above 63 set it on
// every call.
template <typename... KArgs>
inline cudaError_t smem_attr(void (*kernel)(KArgs...), size_t bytes, std::atomic<uint64_t> &done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t(1) << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// Launch on stream s; the arguments are converted to the kernel's parameter types.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                            Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
  if (e == cudaSuccess) launch_counter().fetch_add(1, std::memory_order_relaxed);
  return e;
}

// Resampler (resample.cu): the rates reduced to o (in) and p (out), the cut-off
// c in cycles per input sample, the window half-width 64 / c in input samples;
// outputs in units of U (4 or 8): NT unit types, D input samples between units of a
// type, W (padded W_pad) input offsets in a unit's window, the lowest offset
// over all types; and the FIR's tiling (Q units of each of TG types per tile,
// n_groups type groups, staged input span, tap rows staged or not, shared
// memory).
struct RsPlan {
  int U = 4;      // outputs per unit (4, or 8 in the persistent form when it fits)
  int parts = 2;  // warps sharing one item's offset window (persistent form)
  int o = 1, p = 1;
  double c = 0.0, half = 0.0;
  int NT = 1, D = 1, W = 0, W_pad = 0, lo_min = 0, Q = 32, TG = 1, n_groups = 1, span = 0;
  bool stage_coef = true;
  size_t smem = 0;
  bool pipe = false;     // the persistent, double-buffered FIR applies
  size_t smem_pipe = 0;  // its shared memory
  // tensor-core form: rows of tcN outputs (a multiple of p and of 16, at most
  // 160) sit tcD = tcN o / p inputs apart; a row reads the tcK inputs from
  // tcLo on (relative to its first output's position), tcK a multiple of 64
  bool tc = false;
  int tcN = 0, tcD = 0, tcLo = 0, tcK = 0;
};
int64_t rs_len(int64_t n, int rate_in, int rate_out);  // -1 for invalid arguments
cudaError_t launch_rs_btc(const RsPlan &pl, void *bmat, cudaStream_t s);
cudaError_t launch_rs_fir_tc(const RsPlan &pl, const float *mono, float *y, void *bmat, const int64_t *in_off,
                             const int64_t *out_off, const int32_t *tile_off, int n_clips, int n_tiles,
                             cudaStream_t s);
RsPlan rs_plan(int rate_in, int rate_out);
cudaError_t launch_rs_table(const RsPlan &pl, float *coef, int32_t *lo, cudaStream_t s);
cudaError_t launch_rs_mix(const float *x, int channels, int64_t ch_stride, int64_t n, float *mono, cudaStream_t s);
cudaError_t launch_rs_fir(const RsPlan &pl, const float *mono, float *y, const float *coef, const int32_t *lo,
                          const int64_t *in_off, const int64_t *out_off, const int32_t *tile_off, int n_clips,
                          int n_tiles, cudaStream_t s);
// Copies host words into device memory with kernel launches (the bytes travel
// as kernel parameters), so the call stays asynchronous and capturable.
cudaError_t launch_upload_bytes(const void *host, size_t bytes, void *dev, cudaStream_t s);

// Second log-mel front-end (lfm.cu): per-call tables in the workspace and the
// parameters the kernels read.
constexpr int kLfmMaxMels = 128;  // bands
constexpr int kLfmMaxBins = 32;   // nonzero bins per band
constexpr int kLfmTile = 32;      // frames per work item of the spectrum kernel
constexpr int kLfmWarps = 8;      // warps of the spectrum kernel's band phase
struct LfmTablesDev {
  int n_clips, n_tiles;              // tiles: kLfmTile frames of one clip
  const int64_t *sample_off;         // [B + 1]
  const int32_t *frame_off, *tile_off;  // [B + 1]
  const int32_t *eff;                // [B]: frames whose statistics count
  const int32_t *bank_lo, *bank_cnt, *bank_off;  // [n_mels]: first bin, bins, offset in bank_w
  const float *bank_w;               // [nnz]: the bands' weights, packed
  unsigned long long *moments;       // [B][kLfmMaxMels][2]: sum v, sum v^2 in 2^-24 units (zeroed per call)
};
struct LfmParams {
  int n_mels, hop, win_length;
  int nnz;          // packed weights
  int wave_floats;  // staged-sample buffer of the spectrum kernel (a multiple of 4)
  int vec16;        // 1: the waveform base is 16-byte aligned (16-byte staging copies)
  float preemph, log_floor, var_eps;
  int wband[kLfmWarps + 1];  // bands of each warp in the band phase
};
size_t lfm_smem_bytes(const LfmParams &prm);
cudaError_t launch_lfm(const float *wave, float *out, const LfmTablesDev &t, const LfmParams &prm, cudaStream_t s);

// LFM2A Conformer encoder (lenc.cu, lenc_attention.cu): the shape the kernels
// are compiled for, per-call clip tables in the workspace and the arguments
// of the LayerNorm pass.
constexpr int kLencMels = 128;    // mel bands in
constexpr int kLencEmbd = 512;    // model width
constexpr int kLencHeads = 8;     // heads of 64
constexpr int kLencStemCh = 256;  // stem channels
constexpr int kLencMaxTok = 4096; // rows after the stem per clip
constexpr int kLencMaxConvK = 33; // depthwise conv taps
constexpr int kLencStemRun = 16;  // rows after the first two stem convolutions per work item
struct LencTablesDev {
  int n_clips;
  const int32_t *frame_off;  // [B + 1] mel frames
  const int32_t *s2_off;     // [B + 1] rows after the first two stem convolutions
  const int32_t *tok_off;    // [B + 1] rows after the stem (tokens)
  const int32_t *qblk_off;   // [B + 1] 128-token query blocks
  const int32_t *s2item_off; // [B + 1] work items of kLencStemRun such rows (the first stem kernel)
};
struct LencLnArgs {
  float *x; int64_t rows; float eps;
  const float *w1, *b1; int write_x;
  const float *w2, *b2;  // optional second LayerNorm for the operand
  bf16 *a;               // optional bf16 operand out
};
cudaError_t launch_lenc_stem01(const float *mel, const void *w0b, const float *b0, const float *w1, const float *b1,
                               void *y2, const LencTablesDev &t, int64_t s2_items, cudaStream_t s);
cudaError_t launch_lenc_dw2(const void *y, const float *w, const float *b, void *out, const LencTablesDev &t,
                            int64_t tokens, cudaStream_t s);
cudaError_t launch_lenc_ln(const LencLnArgs &r, cudaStream_t s);
cudaError_t launch_lenc_dwconv(const void *g, const float *w, const float *db, const float *aw, const float *ab, int k,
                               void *out, const int32_t *tok_off, int n_clips, int64_t T, cudaStream_t s);
cudaError_t launch_lenc_relpos(void *pe, int t_max, cudaStream_t s);
cudaError_t launch_lenc_xlattn(const void *qkv, int64_t T, const void *ptab, int64_t p_rows, int64_t p_cols, int p_col,
                               const float *bias_u, const float *bias_v, const int32_t *tok_off,
                               const int32_t *qblk_off, int n_clips, int n_qblk, int t_max, void *out,
                               cudaStream_t s);
// bf16 GEMM for callers without an ae_model: y = epilogue(x W^T), x [M][K]
// bf16, W given by its tensor map ([N][K] bf16).
cudaError_t gemm_bf16(const void *x, int64_t M, int K, const CUtensorMap &tmW, int N, int mode, const EpiArgs &ep,
                      cudaStream_t s);

// Runs fn(ctx), which enqueues kernels on s, inside a kernel-timing record of
// class cls with its algorithmic flops and bytes (ae_profile_enable).
cudaError_t profiled(int cls, double flops, double bytes, cudaStream_t s, cudaError_t (*fn)(void *), void *ctx);
template <class F>
inline cudaError_t profiled_f(int cls, double flops, double bytes, cudaStream_t s, F &&f) {
  return profiled(cls, flops, bytes, s, [](void *c) { return (*static_cast<std::remove_reference_t<F> *>(c))(); },
                  &f);
}

unsigned *device_status_word();
cudaError_t launch_wait_probe(unsigned long long limit_ns, int arrive, cudaStream_t s);
unsigned read_and_clear_status();
cudaError_t launch_pos(int32_t *pos, const int32_t *tok_off, int n_clips, cudaStream_t s);
void set_error(const std::string &msg);

}  // namespace ae
