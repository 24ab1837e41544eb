// C ABI of the audio-encoder library: argument checks, model creation (weight
// conversion or e4m3 quantisation, load-time tables), workspace layout and the
// stream-ordered call sequences of the hot path and of the adjacent parts (the
// resampler, the second log-mel front-end, the standalone e4m3 projection).
// Every computation of a call runs in the kernels of this library; the host
// only validates, builds the per-call and load-time tables, lays out and
// launches.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "ae_internal.h"
#include "e4m3_host.h"
#include "lfm_host.h"

namespace ae {

static thread_local std::string g_last_error;
void set_error(const std::string &msg) { g_last_error = msg; }

std::atomic<uint64_t> &launch_counter() {
  static std::atomic<uint64_t> n{0};
  return n;
}

static size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

static int64_t frames_of_samples(int64_t n) {
  if (n < 0) n = 0;
  if (n > kMaxSamples) n = kMaxSamples;
  return n <= kHop ? 0 : (n - kHop + kHop - 1) / kHop;
}
static int64_t tokens_of_frames(int64_t f) { return ((f + 1) / 2 + 1) / 2; }

// Limits that keep every index the kernels form inside their integer types.
constexpr int64_t kMaxClips = 1 << 20;
constexpr int64_t kMaxTokens = 4000000;
constexpr int64_t kMaxFrames = 16000000;

enum OffKind { kSamples, kFrames, kTokens };

static ae_status fail(ae_status st, const std::string &msg) {
  set_error(msg);
  return st;
}

// ------------------------------------------------------------------ kernel timing

struct Profiler {
  bool on = false;
  size_t cap = 0, n = 0;
  int64_t dropped = 0;
  std::vector<cudaEvent_t> ev;  // 2 per record
  struct Rec {
    int cls;
    double flops, bytes;
  };
  std::vector<Rec> recs;
};
static Profiler g_prof;

// Runs f (which enqueues kernels on s) between two recorded events.
template <class F>
static cudaError_t timed(int cls, double flops, double bytes, cudaStream_t s, F &&f) {
  Profiler &P = g_prof;
  const bool rec = P.on && P.n < P.cap;
  if (P.on && !rec) ++P.dropped;
  if (rec) cudaEventRecord(P.ev[2 * P.n], s);
  const cudaError_t e = f();
  if (rec) {
    cudaEventRecord(P.ev[2 * P.n + 1], s);
    P.recs[P.n] = {cls, flops, bytes};
    ++P.n;
  }
  return e;
}

// The timing record for callers outside this file (the LFM2A encoder).
cudaError_t profiled(int cls, double flops, double bytes, cudaStream_t s, cudaError_t (*fn)(void *), void *ctx) {
  return timed(cls, flops, bytes, s, [&] { return fn(ctx); });
}

static size_t act_bytes(const ae_model *m) { return m->dtype == AE_F32 ? 4 : 2; }

// A projection with its algorithmic flops (2 M N K) and bytes (x, W, y once).
static cudaError_t gemm_t(const ae_model *m, const void *x, int64_t M, int K, const void *w, const CUtensorMap *tmW,
                          int N, int mode, const EpiArgs &ep, cudaStream_t s) {
  const double a = (double)act_bytes(m);
  const double out_cols = mode == EPI_GLU ? N / 2 : N;
  // EPI_ADD_F32 reads and writes the float32 residual
  const double out_b = mode == EPI_ADD_F32 ? 8.0 : mode == EPI_F32 ? 4.0 : a;
  const double bytes = a * ((double)M * K + (double)N * K) + out_b * (double)M * out_cols;
  return timed(AE_K_GEMM, 2.0 * (double)M * N * K, bytes, s, [&] { return gemm(m, x, M, K, w, tmW, N, mode, ep, s); });
}

// An e4m3 projection: 1-byte x and W, y in bf16 (or e4m3 codes for EPI_SILU_Q8).
static cudaError_t gemm8_t(const void *x, int64_t M, int K, const CUtensorMap &tmW, int N, int mode,
                           const EpiArgs &ep, cudaStream_t s) {
  const double out_cols = mode == EPI_GLU ? N / 2 : N;
  const double out_b = mode == EPI_SILU_Q8 ? 1.0 : 2.0;
  const double bytes = (double)M * K + (double)N * K + out_b * (double)M * out_cols;
  return timed(AE_K_GEMM_FP8, 2.0 * (double)M * N * K, bytes, s,
               [&] { return gemm_e4m3(x, M, K, tmW, N, mode, ep, s); });
}

static cudaError_t tables_t(const ClipTables &T, void *ws, const WsLayout &L, ClipTablesDev *td, bool pos,
                            cudaStream_t s) {
  return timed(AE_K_TABLES, 0.0, 0.0, s, [&] { return launch_upload_tables(T, ws, L, td, pos, s); });
}

static double samples_read(const ClipTables &T) {
  double n = 0.0;
  for (int c = 0; c < T.n_clips; ++c)
    n += (double)std::min<int64_t>(T.sample_off[c + 1] - T.sample_off[c], kMaxSamples);
  return n;
}

// log-mel: every sample read once (4 bytes), every frame's 128 floats written once
static cudaError_t logmel_t(const float *wave, float *mel, const ClipTablesDev &td, const ClipTables &T,
                            cudaStream_t s) {
  const double bytes = 4.0 * samples_read(T) + 512.0 * (double)T.total_frames;
  return timed(AE_K_LOGMEL, 0.0, bytes, s, [&] { return launch_logmel(wave, mel, td, T.mel_tiles, s); });
}

// conv0 reads the mel rows and writes every stem row (64 x 128 per row)
static cudaError_t conv0_t(const ae_model *m, const float *mel, void *y0, const ClipTablesDev &td,
                           const ClipTables &T, cudaStream_t s) {
  const double bytes = 512.0 * (double)T.total_frames + (double)act_bytes(m) * kF1 * kC0 * (double)T.stem_rows;
  const double flops = 2.0 * 9 * kC0 * kF1 * (double)T.stem_rows;
  return timed(AE_K_CONV0, flops, bytes, s, [&] { return launch_conv0(m, mel, y0, td, T.stem_rows, s); });
}

// conv1 as a GEMM: M = tokens x 32 frequency rows, N = 32, K = 9 x 128
static cudaError_t conv1_t(const ae_model *m, const void *y0, void *xs, const ClipTablesDev &td, const ClipTables &T,
                           cudaStream_t s) {
  const double M = (double)T.total_tokens * kF2;
  const double a = (double)act_bytes(m);
  const double bytes = a * kF1 * kC0 * (double)T.stem_rows + a * kHidden * (double)T.total_tokens;
  return timed(AE_K_CONV1, 2.0 * M * kC1 * 9 * kC0, bytes, s,
               [&] { return launch_conv1(m, y0, T.stem_rows, xs, td, T.conv1_tiles, T.total_tokens, s); });
}

static cudaError_t rowop_t(const ae_model *m, const RowArgs &r, cudaStream_t s) {
  const double W = r.width;
  const bool changed = r.y || r.w_out;
  double per_row = 4.0 * W * (1.0 + (changed ? 1.0 : 0.0));  // h read, written back if changed
  if (r.y) per_row += W * (double)act_bytes(m);
  if (r.a_out) per_row += W * (r.a_q8 > 0.f ? 1.0 : (double)act_bytes(m));
  return timed(AE_K_ROWOP, 0.0, per_row * (double)r.rows, s, [&] { return launch_rowop(m, r, s); });
}

static ae_status build_tables(const int64_t *off, int n, OffKind kind, ClipTables &T, const char *name) {
  if (n < 0) return fail(AE_EINVAL, "n_clips is negative");
  if (n > kMaxClips) return fail(AE_EINVAL, "n_clips above 1048576");
  if (!off) return fail(AE_EINVAL, std::string(name) + " is null");
  if (off[0] != 0) return fail(AE_EINVAL, std::string(name) + "[0] must be 0");
  T = ClipTables();
  T.n_clips = n;
  const size_t B1 = (size_t)n + 1;
  T.sample_off.assign(B1, 0);
  T.frame_off.assign(B1, 0);
  T.tok_off.assign(B1, 0);
  T.stem_off.assign(B1, 0);
  T.mel_tile_off.assign(B1, 0);
  T.conv1_tile_off.assign(B1, 0);
  int64_t fr = 0, tk = 0, st = 0, mt = 0, ct = 0;
  for (int c = 0; c < n; ++c) {
    const int64_t len = off[c + 1] - off[c];
    if (len < 0) return fail(AE_EINVAL, std::string(name) + " is not non-decreasing at clip " + std::to_string(c));
    const int64_t F = kind == kSamples ? frames_of_samples(len) : (kind == kFrames ? len : 0);
    if (kind == kFrames && F > frames_of_samples(kMaxSamples))
      return fail(AE_EINVAL, "clip " + std::to_string(c) + " has more than 2999 frames");
    const int64_t tok = kind == kTokens ? len : tokens_of_frames(F);
    fr += F;
    tk += tok;
    st += 2 * tok + 2;
    mt += (F + kMelTile - 1) / kMelTile;
    ct += (tok + kConv1TileTok - 1) / kConv1TileTok;
    if (fr > kMaxFrames || tk > kMaxTokens) return fail(AE_EINVAL, "batch too large for one call (frames or tokens)");
    T.sample_off[c + 1] = kind == kSamples ? off[c + 1] : 0;
    T.frame_off[c + 1] = (int32_t)fr;
    T.tok_off[c + 1] = (int32_t)tk;
    T.stem_off[c + 1] = (int32_t)st;
    T.mel_tile_off[c + 1] = (int32_t)mt;
    T.conv1_tile_off[c + 1] = (int32_t)ct;
  }
  T.total_samples = kind == kSamples ? off[n] : 0;
  T.total_frames = fr;
  T.total_tokens = tk;
  T.stem_rows = st;
  T.mel_tiles = mt;
  T.conv1_tiles = ct;
  return AE_OK;
}

// Workspace: [tables][pos][h][ union( stem: mel, y0, xs | layers: a, big, y, o ) ]
WsLayout ws_layout(const ae_model *m, int64_t n_clips, int64_t frames, int64_t tokens, bool with_model) {
  WsLayout L;
  size_t off = 0;
  L.tables = off;
  off += al256(tables_bytes(n_clips));
  L.pos = off;
  off += al256((size_t)tokens * 4);
  if (!with_model || !m) {
    L.total = off;
    return L;
  }
  const size_t act = m->dtype == AE_F32 ? 4 : 2;
  const int64_t H = m->cfg.hidden;
  L.h = off;
  off += al256((size_t)tokens * H * 4);
  const size_t u = off;
  size_t so = u;
  L.mel = so;
  so += al256((size_t)frames * kMels * 4);
  L.y0 = so;
  so += al256(act * (size_t)(2 * tokens + 2 * n_clips) * kF1 * kC0);
  L.xs = so;
  so += al256(act * (size_t)tokens * kHidden);
  size_t lo_ = u;
  const int64_t big_w = std::max<int64_t>({m->cfg.ffn, 3 * H, m->cfg.out_dim, 2 * H});
  const int64_t y_w = std::max<int64_t>(H, m->cfg.out_dim);
  L.a = lo_;
  lo_ += al256(act * (size_t)tokens * H);
  L.big = lo_;
  lo_ += al256(act * (size_t)tokens * big_w);
  L.y = lo_;
  lo_ += al256((size_t)tokens * y_w * 4);
  L.o = lo_;
  lo_ += al256(act * (size_t)tokens * H);
  L.total = std::max(so, lo_);
  return L;
}

// ------------------------------------------------------------------ host-side load-time tables

static double softplus_torch(double x) { return x > 20.0 ? x : std::log1p(std::exp(x)); }

static void attention_tables_host(const float *relk, const float *pds, int hidden, int heads, int left, float *R,
                                  float *qscale, float *k_scale) {
  const int n_ts = hidden / 2;
  const double incr = std::log(10000.0) / (double)(std::max(n_ts, 2) - 1);
  std::vector<double> inv(n_ts), pe(hidden);
  for (int i = 0; i < n_ts; ++i) inv[i] = std::exp(-(double)i * incr);
  for (int d = 0; d < left; ++d) {
    for (int i = 0; i < n_ts; ++i) {
      pe[i] = std::sin(d * inv[i]);
      pe[n_ts + i] = std::cos(d * inv[i]);
    }
    for (int j = 0; j < hidden; ++j) {
      const float *w = relk + (size_t)j * hidden;
      double acc = 0.0;
      for (int i = 0; i < hidden; ++i) acc += pe[i] * (double)w[i];
      R[(size_t)d * hidden + j] = (float)acc;
    }
  }
  const int hd = hidden / heads;
  const double qs = (1.0 / std::sqrt((double)hd)) / std::log(2.0);
  for (int j = 0; j < hd; ++j) qscale[j] = (float)(qs * softplus_torch((double)pds[j]));
  *k_scale = (float)(std::log(1.0 + std::exp(1.0)) / std::log(2.0));
}

static uint16_t f2bf(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return 0x7fc0;
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

struct Uploader {
  ae_model *m;
  bool ok = true;
  template <typename T> T *alloc(size_t n) {
    void *p = nullptr;
    if (!ok || cudaMalloc(&p, std::max<size_t>(n, 1) * sizeof(T)) != cudaSuccess) {
      ok = false;
      return nullptr;
    }
    m->allocs.push_back(p);
    return static_cast<T *>(p);
  }
  float *f32(const float *h, size_t n) {
    float *d = alloc<float>(n);
    if (d && cudaMemcpy(d, h, n * 4, cudaMemcpyHostToDevice) != cudaSuccess) ok = false;
    return d;
  }
  // matrix in the model's GEMM operand type
  void *mat(const std::vector<float> &h) {
    if (m->dtype == AE_F32) return f32(h.data(), h.size());
    std::vector<uint16_t> b(h.size());
    for (size_t i = 0; i < h.size(); ++i) b[i] = f2bf(h[i]);
    uint16_t *d = alloc<uint16_t>(b.size());
    if (d && cudaMemcpy(d, b.data(), b.size() * 2, cudaMemcpyHostToDevice) != cudaSuccess) ok = false;
    return d;
  }
  void *mat(const float *h, size_t n) { return mat(std::vector<float>(h, h + n)); }
  // e4m3 rows: row n as codes of W[n][k] / s_n, s_n = max_k |W[n][k]| / 448;
  // *cs gets s_n / q8 per row (the accumulator column factor)
  void *mat_e4m3(const std::vector<float> &h, size_t rows, size_t cols, float q8, float **cs) {
    std::vector<uint8_t> codes(rows * cols);
    std::vector<float> f(rows);
    for (size_t r = 0; r < rows; ++r) {
      double sn;
      e4m3_quantise_row(h.data() + r * cols, cols, codes.data() + r * cols, &sn);
      f[r] = (float)(sn / (double)q8);
    }
    *cs = f32(f.data(), f.size());
    uint8_t *d = alloc<uint8_t>(codes.size());
    if (d && cudaMemcpy(d, codes.data(), codes.size(), cudaMemcpyHostToDevice) != cudaSuccess) ok = false;
    return d;
  }
  void *mat_e4m3(const float *h, size_t rows, size_t cols, float q8, float **cs) {
    return mat_e4m3(std::vector<float>(h, h + rows * cols), rows, cols, q8, cs);
  }
};

// Scale of an e4m3 input clamped to [lo, hi]: 448 over the larger bound.
static float q8_of(const ae_clip &c) { return (float)(448.0 / std::max(std::fabs((double)c.lo_in), std::fabs((double)c.hi_in))); }
static bool q8_ok(const ae_clip &c) {
  const double b = std::max(std::fabs((double)c.lo_in), std::fabs((double)c.hi_in));
  return std::isfinite(b) && b > 0.0;
}

static bool bad_clip(const ae_clip &c) {
  return std::isnan(c.lo_in) || std::isnan(c.hi_in) || std::isnan(c.lo_out) || std::isnan(c.hi_out) ||
         c.lo_in > c.hi_in || c.lo_out > c.hi_out;
}

// ------------------------------------------------------------------ one layer

struct Bufs {
  float *h;
  void *a, *big, *o;
  float *y;
  const int32_t *pos;
};

static EpiArgs ep_of(void *out, int64_t ld, float lo, float hi) {
  EpiArgs e;
  std::memset(&e, 0, sizeof(e));
  e.out = out;
  e.ld = ld;
  e.lo = lo;
  e.hi = hi;
  e.lo2 = -INFINITY;
  e.hi2 = INFINITY;
  e.clamp2 = 1;
  return e;
}

// Whether clamp(silu(c), lo2, hi2) can differ from silu(c) for c in [lo, hi]:
// silu(c) = c sigmoid(c) is at least -0.2785 everywhere (its minimum, at
// c = -1.2785) and below max(c, 0), so bounds of at most -0.5 and at least
// max(hi, 0) cannot bind (the margin covers the kernels' approximations).
static int silu_clamp_binds(float hi, float lo2, float hi2) {
  return !(lo2 <= -0.5f && hi2 >= std::max(hi, 0.0f));
}

static RowArgs row_of(float *h, int width, int64_t rows) {
  RowArgs r;
  std::memset(&r, 0, sizeof(r));
  r.h = h;
  r.width = width;
  r.rows = rows;
  r.a_rms = 1;
  r.lo = -INFINITY;
  r.hi = INFINITY;
  return r;
}

#define AE_TRY(x)                            \
  do {                                       \
    cudaError_t e_ = (x);                    \
    if (e_ != cudaSuccess) return e_;        \
  } while (0)

// What the layer's last row pass should also write into b.a.
enum NextA { kNextNone, kNextLayer, kNextPlain };

static cudaError_t run_layer(const ae_model *m, int li, const Bufs &b, int64_t T, bool a_ready, NextA next,
                             cudaStream_t s) {
  const LayerDev &L = m->layers[li];
  const int H = m->cfg.hidden, F = m->cfg.ffn;
  const float rw = m->cfg.residual_weight;
  const size_t act = act_bytes(m);
  const bool tc = m->dtype != AE_F32;
  const bool f8 = m->dtype == AE_FP8;  // FFN W1/W2, q/k/v and lc_start on e4m3 operands
  // the projections whose outputs feed a row pass write them in the act type
  // (bf16 for the tensor-core models): the row pass is bound by its bytes
  const int y_mode = tc ? EPI_BF16 : EPI_F32;
  if (!a_ready) {
    RowArgs r = row_of(b.h, H, T);
    r.a_out = b.a;
    r.w_next = L.ff1_pre;
    r.lo = L.c_ff1_w1.lo_in;
    r.hi = L.c_ff1_w1.hi_in;
    r.a_q8 = f8 ? L.q8_ff1_w1 : 0.f;
    AE_TRY(rowop_t(m, r, s));
  }
  auto ffn = [&](void *w1, const CUtensorMap *t1, const ae_clip &c1, void *w2, const CUtensorMap *t2,
                 const ae_clip &c2, const float *cs1, const float *cs2, float q8_2) -> cudaError_t {
    EpiArgs e1 = ep_of(b.big, F, c1.lo_out, c1.hi_out);
    e1.lo2 = c2.lo_in;
    e1.hi2 = c2.hi_in;
    e1.clamp2 = silu_clamp_binds(c1.hi_out, c2.lo_in, c2.hi_in);
    EpiArgs e2 = ep_of(b.y, H, c2.lo_out, c2.hi_out);
    if (f8) {
      e1.cs = cs1;
      e1.q8 = q8_2;
      e2.cs = cs2;
      AE_TRY(gemm8_t(b.a, T, H, *t1, F, EPI_SILU_Q8, e1, s));
      return gemm8_t(b.big, T, F, *t2, H, EPI_BF16, e2, s);
    }
    AE_TRY(gemm_t(m, b.a, T, H, w1, tc ? t1 : nullptr, F, EPI_SILU, e1, s));
    return gemm_t(m, b.big, T, F, w2, tc ? t2 : nullptr, H, y_mode, e2, s);
  };
  // ---- FFN1
  AE_TRY(ffn(L.ff1_w1, &L.tm_ff1_w1, L.c_ff1_w1, L.ff1_w2, &L.tm_ff1_w2, L.c_ff1_w2, L.cs_ff1_w1, L.cs_ff1_w2,
             L.q8_ff1_w2));
  {
    RowArgs r = row_of(b.h, H, T);
    r.y = b.y; r.wy = L.ff1_post; r.s = rw; r.y_norm = 1;
    r.a_out = b.a; r.w_next = L.norm_pre_attn; r.lo = L.c_q.lo_in; r.hi = L.c_q.hi_in;
    r.a_q8 = f8 ? L.q8_qkv : 0.f;
    AE_TRY(rowop_t(m, r, s));
  }
  // ---- attention: fused q/k/v projection, core, post
  {
    EpiArgs e = ep_of(b.big, 3 * H, -INFINITY, INFINITY);
    e.seg_w = H;
    e.seg_lo[0] = L.c_q.lo_out; e.seg_hi[0] = L.c_q.hi_out;
    e.seg_lo[1] = L.c_k.lo_out; e.seg_hi[1] = L.c_k.hi_out;
    e.seg_lo[2] = L.c_v.lo_out; e.seg_hi[2] = L.c_v.hi_out;
    if (f8) {
      e.cs = L.cs_qkv;
      AE_TRY(gemm8_t(b.a, T, H, L.tm_qkv, 3 * H, EPI_BF16, e, s));
    } else {
      AE_TRY(gemm_t(m, b.a, T, H, L.qkv, tc ? &L.tm_qkv : nullptr, 3 * H, EPI_BF16, e, s));
    }
    const uint8_t *qkv = static_cast<const uint8_t *>(b.big);
    AE_TRY(timed(AE_K_ATTENTION, 0.0, (double)T * 4 * H * act, s, [&] {
      return launch_attention(tc, qkv, qkv + act * H, qkv + 2 * act * H, 3 * H, L.R, L.qscale, m->k_scale,
                              m->cfg.softcap, b.pos, T, b.o, H, L.c_post.lo_in, L.c_post.hi_in, s);
    }));
    AE_TRY(gemm_t(m, b.o, T, H, L.post, tc ? &L.tm_post : nullptr, H, y_mode,
                  ep_of(b.y, H, L.c_post.lo_out, L.c_post.hi_out), s));
    RowArgs r = row_of(b.h, H, T);
    r.y = b.y; r.wy = L.norm_post_attn; r.s = 1.0f; r.y_norm = 1;
    r.a_out = b.a; r.w_next = L.lc_pre; r.lo = L.c_lc_start.lo_in; r.hi = L.c_lc_start.hi_in;
    r.a_q8 = f8 ? L.q8_lc_start : 0.f;
    AE_TRY(rowop_t(m, r, s));
  }
  // ---- light conv
  {
    EpiArgs e = ep_of(b.big, H, L.c_lc_start.lo_out, L.c_lc_start.hi_out);
    if (f8) {
      e.cs = L.cs_lc_start;
      AE_TRY(gemm8_t(b.a, T, H, L.tm_lc_start, 2 * H, EPI_GLU, e, s));
    } else {
      AE_TRY(gemm_t(m, b.a, T, H, L.lc_start, tc ? &L.tm_lc_start : nullptr, 2 * H, EPI_GLU, e, s));
    }
    AE_TRY(timed(AE_K_LCONV, 0.0, (double)T * 2 * H * act, s, [&] {
      return launch_lconv(m, b.big, L.lc_dw, L.lc_norm, L.c_lc_end.lo_in, L.c_lc_end.hi_in, b.o, b.pos, T, s);
    }));
    // this residual is a plain add (no norm), so the projection adds its clamped
    // output into h itself; the row pass only forms the next operand
    AE_TRY(gemm_t(m, b.o, T, H, L.lc_end, tc ? &L.tm_lc_end : nullptr, H, EPI_ADD_F32,
                  ep_of(b.h, H, L.c_lc_end.lo_out, L.c_lc_end.hi_out), s));
    RowArgs r = row_of(b.h, H, T);
    r.a_out = b.a; r.w_next = L.ff2_pre; r.lo = L.c_ff2_w1.lo_in; r.hi = L.c_ff2_w1.hi_in;
    r.a_q8 = f8 ? L.q8_ff2_w1 : 0.f;
    AE_TRY(rowop_t(m, r, s));
  }
  // ---- FFN2, norm_out, and the next consumer's input
  AE_TRY(ffn(L.ff2_w1, &L.tm_ff2_w1, L.c_ff2_w1, L.ff2_w2, &L.tm_ff2_w2, L.c_ff2_w2, L.cs_ff2_w1, L.cs_ff2_w2,
             L.q8_ff2_w2));
  {
    RowArgs r = row_of(b.h, H, T);
    r.y = b.y; r.wy = L.ff2_post; r.s = rw; r.y_norm = 1;
    r.w_out = L.norm_out;
    if (next == kNextLayer) {
      const LayerDev &N = m->layers[li + 1];
      r.a_out = b.a; r.w_next = N.ff1_pre; r.lo = N.c_ff1_w1.lo_in; r.hi = N.c_ff1_w1.hi_in;
      r.a_q8 = f8 ? N.q8_ff1_w1 : 0.f;
    } else if (next == kNextPlain) {
      r.a_out = b.a; r.a_rms = 0;
    }
    AE_TRY(rowop_t(m, r, s));
  }
  return cudaSuccess;
}

// Head: out_proj + bias, weightless RMS norm, embed. b.a holds h in the operand type.
static cudaError_t run_head(const ae_model *m, const Bufs &b, int64_t T, float *out, cudaStream_t s) {
  const int H = m->cfg.hidden, OD = m->cfg.out_dim, ED = m->cfg.embed_dim;
  const bool tc = m->dtype != AE_F32;
  EpiArgs e = ep_of(b.y, OD, -INFINITY, INFINITY);
  e.bias = m->out_bias;
  AE_TRY(gemm_t(m,b.a, T, H, m->out_proj, tc ? &m->tm_out_proj : nullptr, OD, EPI_F32, e, s));
  RowArgs r = row_of(b.y, OD, T);
  r.a_out = b.big;
  AE_TRY(rowop_t(m, r, s));
  return gemm_t(m, b.big, T, OD, m->embed, tc ? &m->tm_embed : nullptr, ED, EPI_F32,
                ep_of(out, ED, -INFINITY, INFINITY), s);
}

static Bufs bufs_of(void *ws, const WsLayout &L, const ClipTablesDev &td) {
  uint8_t *w = static_cast<uint8_t *>(ws);
  Bufs b;
  b.h = reinterpret_cast<float *>(w + L.h);
  b.a = w + L.a;
  b.big = w + L.big;
  b.y = reinterpret_cast<float *>(w + L.y);
  b.o = w + L.o;
  b.pos = td.pos;
  return b;
}

static ae_status cuda_fail(cudaError_t e, const char *where) {
  return fail(AE_ECUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

static ae_status check_model(const ae_model *m) {
  if (!m) return fail(AE_EINVAL, "model is null");
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(AE_ECUDA, "no CUDA device");
  if (dev != m->device) return fail(AE_EINVAL, "the current device is not the model's device");
  return AE_OK;
}

static ae_status check_ws(void *ws, size_t have, size_t need) {
  if (need > 0 && !ws) return fail(AE_EINVAL, "d_ws is null");
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0) return fail(AE_EINVAL, "d_ws must be 256-byte aligned");
  if (have < need)
    return fail(AE_EWORKSPACE, "workspace of " + std::to_string(have) + " bytes, " + std::to_string(need) + " needed");
  return AE_OK;
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// The encode sequence on device buffers (shared by ae_encode and ae_encode_host).
// Optional per-stage copies of one pass (the page's `trace` of encode_mels):
// the log-mel rows and the residual stream after in_proj and after each layer.
struct TraceOut {
  float *mel = nullptr;     // [sum frames][128]
  float *layers = nullptr;  // [n_layers + 1][sum tokens][hidden]
};

static ae_status encode_one(const ae_model *m, const float *d_wave, const ClipTables &T, float *d_out, void *d_ws,
                            const WsLayout &L, cudaStream_t s, const TraceOut *tr = nullptr) {
  ClipTablesDev td;
  cudaError_t e = tables_t(T, d_ws, L, &td, true, s);
  if (e != cudaSuccess) return cuda_fail(e, "table upload");
  if (T.total_tokens == 0) return AE_OK;
  uint8_t *w = static_cast<uint8_t *>(d_ws);
  float *mel = reinterpret_cast<float *>(w + L.mel);
  Bufs b = bufs_of(d_ws, L, td);
  if ((e = logmel_t(d_wave, mel, td, T, s)) != cudaSuccess) return cuda_fail(e, "logmel");
  const size_t h_bytes = (size_t)T.total_tokens * m->cfg.hidden * 4;
  auto trace_h = [&](int slot) -> cudaError_t {  // the residual stream into trace slot `slot`
    if (!tr || !tr->layers) return cudaSuccess;
    return cudaMemcpyAsync(reinterpret_cast<uint8_t *>(tr->layers) + (size_t)slot * h_bytes, b.h, h_bytes,
                           cudaMemcpyDeviceToDevice, s);
  };
  if (tr && tr->mel &&
      (e = cudaMemcpyAsync(tr->mel, mel, (size_t)T.total_frames * kMels * 4, cudaMemcpyDeviceToDevice, s)) !=
          cudaSuccess)
    return cuda_fail(e, "trace copy");
  if ((e = conv0_t(m, mel, w + L.y0, td, T, s)) != cudaSuccess) return cuda_fail(e, "conv0");
  if ((e = conv1_t(m, w + L.y0, w + L.xs, td, T, s)) != cudaSuccess)
    return cuda_fail(e, "conv1");
  if ((e = gemm_t(m, w + L.xs, T.total_tokens, kHidden, m->in_proj, m->dtype != AE_F32 ? &m->tm_in_proj : nullptr,
                m->cfg.hidden, EPI_F32, ep_of(b.h, m->cfg.hidden, -INFINITY, INFINITY), s)) != cudaSuccess)
    return cuda_fail(e, "in_proj");
  if ((e = trace_h(0)) != cudaSuccess) return cuda_fail(e, "trace copy");
  const int nl = m->cfg.n_layers;
  for (int li = 0; li < nl; ++li) {
    e = run_layer(m, li, b, T.total_tokens, li > 0, li + 1 < nl ? kNextLayer : kNextPlain, s);
    if (e != cudaSuccess) return cuda_fail(e, "layer");
    if ((e = trace_h(li + 1)) != cudaSuccess) return cuda_fail(e, "trace copy");
  }
  if (nl == 0) {
    RowArgs r = row_of(b.h, m->cfg.hidden, T.total_tokens);
    r.a_out = b.a;
    r.a_rms = 0;
    if ((e = rowop_t(m, r, s)) != cudaSuccess) return cuda_fail(e, "head input");
  }
  if ((e = run_head(m, b, T.total_tokens, d_out, s)) != cudaSuccess) return cuda_fail(e, "head");
  return AE_OK;
}

// Workspace of ae_encode: the layout of the whole batch plus room for the
// rounding of two half-batch layouts (every region of a half is a prefix-sum
// share of the whole, the stem regions dominate both halves' unions, and each
// region rounds up to 256 bytes at most once more per half).
constexpr size_t kSplitSlack = 64 * 1024;
constexpr int64_t kSplitMinTokens = 4096;
// Above this the halves' kernels fill the GPU on their own and the second
// stream only adds contention (measured on the 96k-token ragged batch: one
// pass 62.5-62.8 ms per step, two halves 63.5-63.9 ms, same box, interleaved).
constexpr int64_t kSplitMaxTokens = 32768;

static size_t encode_ws_bytes(const ae_model *m, int64_t n_clips, int64_t frames, int64_t tokens) {
  return ws_layout(m, n_clips, frames, tokens, true).total + kSplitSlack;
}

// Clips [a, b) of T as a table of their own (offsets rebased to clip a).
static ClipTables sub_tables(const ClipTables &T, int a, int b) {
  std::vector<int64_t> off(b - a + 1);
  for (int i = a; i <= b; ++i) off[i - a] = T.sample_off[i] - T.sample_off[a];
  ClipTables S;
  build_tables(off.data(), b - a, kSamples, S, "h_sample_off");
  return S;
}

// The whole forward. A batch of kSplitMinTokens to kSplitMaxTokens tokens in two or
// more clips runs as two halves of about equal token count, the first on s and
// the second on the model's side stream, each with its own workspace layout;
// the clips are independent, so the halves only share the weights. Outputs
// land in the same rows as for one pass. Not while profiling (the per-kernel
// event timing assumes one stream), and not when the caller asks for one pass
// (the asynchronous host entry point, whose callers overlap whole calls on
// their own streams: measured, a second split only adds contention there).
static ae_status encode_dev(const ae_model *m, const float *d_wave, const ClipTables &T, float *d_out, void *d_ws,
                            size_t ws_bytes, cudaStream_t s, bool may_split) {
  const WsLayout L = ws_layout(m, T.n_clips, T.total_frames, T.total_tokens, true);
  if (!may_split || g_prof.on || T.n_clips < 2 || T.total_tokens < kSplitMinTokens ||
      T.total_tokens > kSplitMaxTokens || !m->side[0])
    return encode_one(m, d_wave, T, d_out, d_ws, L, s);
  int k = 1;  // first clip of the second half
  while (k < T.n_clips - 1 && 2 * (int64_t)T.tok_off[k] < T.total_tokens) ++k;
  const ClipTables A = sub_tables(T, 0, k), B = sub_tables(T, k, T.n_clips);
  const WsLayout LA = ws_layout(m, A.n_clips, A.total_frames, A.total_tokens, true);
  const WsLayout LB = ws_layout(m, B.n_clips, B.total_frames, B.total_tokens, true);
  const size_t b_off = al256(LA.total);
  if (b_off + LB.total > ws_bytes || A.total_tokens == 0 || B.total_tokens == 0)
    return encode_one(m, d_wave, T, d_out, d_ws, L, s);
  ae_model *mm = const_cast<ae_model *>(m);
  std::lock_guard<std::mutex> guard(mm->split_mu);
  const int si = mm->next_side;
  mm->next_side ^= 1;
  cudaStream_t side = mm->side[si];
  cudaError_t e = cudaEventRecord(mm->fork[si], s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(side, mm->fork[si], 0);
  if (e != cudaSuccess) return cuda_fail(e, "fork");
  ae_status sa = encode_one(m, d_wave, A, d_out, d_ws, LA, s);
  ae_status sb = sa ? sa
                    : encode_one(m, d_wave + T.sample_off[k], B, d_out + (int64_t)T.tok_off[k] * m->cfg.embed_dim,
                                 static_cast<uint8_t *>(d_ws) + b_off, LB, side);
  e = cudaEventRecord(mm->join[si], side);  // joined whatever happened above
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, mm->join[si], 0);
  if (sb) return sb;
  if (e != cudaSuccess) return cuda_fail(e, "join");
  return AE_OK;
}

// ------------------------------------------------------------------ log-mel without a workspace

// The clip tables of ae_logmel_noalloc live in this file-scope device array
// (every GPU that loads the library holds it until the process exits). In
// host code the name is only a stand-in: its device address is looked up
// with cudaGetSymbolAddress, with the device current, and passed to the
// kernels. The address is cached per device together with the CUDA context
// it was taken in; a different current context (after cudaDeviceReset, say)
// makes the next call look it up again.
constexpr int kNoAllocMaxClips = 4000;
constexpr size_t kNoAllocScratchBytes = 131072;
static __device__ __align__(256) unsigned char g_logmel_scratch[kNoAllocScratchBytes];

static std::mutex g_noalloc_mu;
static void *g_noalloc_ptr[64] = {nullptr};
static void *g_noalloc_ctx[64] = {nullptr};

// The current CUDA context (driver cuCtxGetCurrent, looked up at run time), or
// nullptr if the entry point is unavailable.
static void *current_context() {
  using Fn = int (*)(void **);
  static Fn fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<Fn>(p);
    return static_cast<Fn>(nullptr);
  }();
  void *ctx = nullptr;
  if (!fn || fn(&ctx) != 0) return nullptr;
  return ctx;
}

// Device address of the scratch array on the current device.
static ae_status noalloc_scratch(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return fail(AE_ECUDA, "no CUDA device");
  if (dev >= 64) return fail(AE_EUNSUPPORTED, "device index above 63");
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  void *ctx = current_context();
  if (!g_noalloc_ptr[dev] || !ctx || ctx != g_noalloc_ctx[dev]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_logmel_scratch);
    if (e != cudaSuccess || !p) return cuda_fail(e, "cudaGetSymbolAddress of the log-mel scratch");
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = current_context();  // the lookup may have created the primary context
  }
  *out = g_noalloc_ptr[dev];
  return AE_OK;
}

}  // namespace ae

using namespace ae;

// ====================================================================== ABI

extern "C" {

int64_t ae_num_frames(int64_t n) { return frames_of_samples(n); }
int64_t ae_num_tokens(int64_t n) { return tokens_of_frames(frames_of_samples(n)); }

const char *ae_last_error(void) { return g_last_error.c_str(); }
const char *ae_version(void) { return "0.1.0"; }

ae_status ae_device_status(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return fail(AE_ECUDA, "device reported an error");
  const unsigned v = read_and_clear_status();
  if (v == ~0u) return fail(AE_ECUDA, "status word unreadable");
  if (v) return fail(AE_EDEVICE, "a kernel gave up a bounded wait");
  return AE_OK;
}

uint64_t ae_launch_count(void) { return launch_counter().load(std::memory_order_relaxed); }

ae_status ae_selftest_bounded_wait(uint32_t limit_us, int arrive, ae_stream stream) {
  if (limit_us < 1 || limit_us > 1000000) return fail(AE_EINVAL, "limit_us must be in [1, 1000000]");
  const cudaError_t e =
      launch_wait_probe(1000ull * limit_us, arrive ? 1 : 0, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "wait probe");
  return AE_OK;
}

ae_status ae_attention_tables(const float *relk, const float *pds, int hidden, int heads, int left, float *R,
                              float *qscale, float *k_scale) {
  if (!relk || !pds || !R || !qscale || !k_scale) return fail(AE_EINVAL, "null pointer");
  if (hidden <= 0 || heads <= 0 || hidden % heads || hidden % 2 || left <= 0)
    return fail(AE_EINVAL, "bad hidden/heads/left");
  attention_tables_host(relk, pds, hidden, heads, left, R, qscale, k_scale);
  return AE_OK;
}

void ae_model_destroy(ae_model *m) {
  if (!m) return;
  for (void *p : m->allocs) cudaFree(p);
  for (int i = 0; i < 2; ++i) {
    if (m->side[i]) cudaStreamDestroy(m->side[i]);
    if (m->fork[i]) cudaEventDestroy(m->fork[i]);
    if (m->join[i]) cudaEventDestroy(m->join[i]);
  }
  delete m;
}

ae_status ae_model_create(const ae_config *cfg, const ae_host_weights *w, ae_dtype dtype, ae_model **out) {
  if (!out) return fail(AE_EINVAL, "out is null");
  *out = nullptr;
  if (!cfg || !w) return fail(AE_EINVAL, "cfg or weights is null");
  const ae_config &c = *cfg;
  if (c.n_mels != kMels || c.c0 != kC0 || c.c1 != kC1 || c.hidden != kHidden || c.heads != kHeads ||
      c.left != kLeft || c.kernel != kKernel)
    return fail(AE_EUNSUPPORTED, "kernels are built for n_mels 128, c0 128, c1 32, hidden 1024, heads 8, left 12, "
                                 "kernel 5");
  if (c.ffn <= 0 || c.ffn % 256 || c.embed_dim <= 0 || c.embed_dim % 256)
    return fail(AE_EUNSUPPORTED, "ffn and embed_dim must be positive multiples of 256");
  if (c.out_dim != 1024 && c.out_dim != 1536 && c.out_dim != 2048)
    return fail(AE_EUNSUPPORTED, "out_dim must be 1024, 1536 or 2048");
  if (c.n_layers < 0 || c.n_layers > 4096) return fail(AE_EINVAL, "n_layers out of range");
  if (!(c.softcap > 0.f) || !std::isfinite(c.softcap) || !std::isfinite(c.residual_weight))
    return fail(AE_EINVAL, "softcap must be positive and finite, residual_weight finite");
  if (dtype != AE_F32 && dtype != AE_BF16 && dtype != AE_FP8) return fail(AE_EINVAL, "dtype");
  if (!w->conv0 || !w->ln0 || !w->conv1 || !w->ln1 || !w->in_proj || !w->out_proj || !w->out_bias || !w->embed ||
      (c.n_layers > 0 && !w->layers))
    return fail(AE_EINVAL, "a stem or head weight pointer is null");
  for (int i = 0; i < c.n_layers; ++i) {
    const ae_host_layer &l = w->layers[i];
    const void *ps[] = {l.ff1_pre, l.ff1_w1, l.ff1_w2, l.ff1_post, l.ff2_pre, l.ff2_w1, l.ff2_w2, l.ff2_post,
                        l.norm_pre_attn, l.norm_post_attn, l.norm_out, l.q, l.k, l.v, l.post, l.per_dim_scale,
                        l.relative_k, l.lc_pre, l.lc_start, l.lc_dw, l.lc_norm, l.lc_end};
    for (const void *p : ps)
      if (!p) return fail(AE_EINVAL, "a weight pointer of layer " + std::to_string(i) + " is null");
    const ae_clip cs[] = {l.clip_ff1_w1, l.clip_ff1_w2, l.clip_q, l.clip_k, l.clip_v, l.clip_post,
                          l.clip_lc_start, l.clip_lc_end, l.clip_ff2_w1, l.clip_ff2_w2};
    for (const ae_clip &b : cs)
      if (bad_clip(b)) return fail(AE_EINVAL, "a clamp bound of layer " + std::to_string(i) + " is NaN or inverted");
    if (l.clip_q.lo_in != l.clip_k.lo_in || l.clip_q.lo_in != l.clip_v.lo_in || l.clip_q.hi_in != l.clip_k.hi_in ||
        l.clip_q.hi_in != l.clip_v.hi_in)
      return fail(AE_EUNSUPPORTED, "q, k and v input bounds differ in layer " + std::to_string(i));
    if (dtype == AE_FP8 && !(q8_ok(l.clip_ff1_w1) && q8_ok(l.clip_ff1_w2) && q8_ok(l.clip_ff2_w1) &&
                             q8_ok(l.clip_ff2_w2) && q8_ok(l.clip_q) && q8_ok(l.clip_lc_start)))
      return fail(AE_EUNSUPPORTED, "AE_FP8 needs finite, nonzero input bounds on FFN W1/W2, q/k/v and lc_start "
                                   "(layer " + std::to_string(i) + ")");
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(AE_ECUDA, "no CUDA device");
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return fail(AE_ECUDA, "device properties");
  if (prop.major != 10 || prop.minor != 0)
    return fail(AE_EUNSUPPORTED, "this library is built for sm_100a (B200); device is sm_" +
                                     std::to_string(prop.major) + std::to_string(prop.minor));

  ae_model *m = new ae_model();
  m->cfg = c;
  m->dtype = dtype;
  m->device = dev;
  {
    cudaError_t e = cudaSuccess;
    for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
      e = cudaStreamCreateWithFlags(&m->side[i], cudaStreamNonBlocking);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&m->fork[i], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&m->join[i], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) {
      ae_model_destroy(m);
      return cuda_fail(e, "side stream");
    }
  }
  Uploader up{m};
  const int H = c.hidden;
  // conv0: taps minus their channel mean, and their channel covariance (float64)
  {
    std::vector<double> mean(9, 0.0);
    for (int ch = 0; ch < kC0; ++ch)
      for (int k = 0; k < 9; ++k) mean[k] += w->conv0[ch * 9 + k];
    for (int k = 0; k < 9; ++k) mean[k] /= kC0;
    std::vector<float> wc(kC0 * 9), cov(81);
    std::vector<double> cd(81, 0.0);
    for (int ch = 0; ch < kC0; ++ch)
      for (int a = 0; a < 9; ++a) {
        const double da = w->conv0[ch * 9 + a] - mean[a];
        wc[ch * 9 + a] = (float)(da * (double)w->ln0[ch]);  // LayerNorm gain folded into the centred taps
        for (int b2 = 0; b2 < 9; ++b2) cd[a * 9 + b2] += da * (w->conv0[ch * 9 + b2] - mean[b2]);
      }
    for (int i = 0; i < 81; ++i) cov[i] = (float)(cd[i] / kC0);
    m->conv0c = up.f32(wc.data(), wc.size());
    m->conv0cov = up.f32(cov.data(), cov.size());
    if (dtype != AE_F32) {
      // the tensor-core conv0's B rows: k = 0..8 hi parts, 9..17 lo parts, 18..26 hi parts
      // again, against A = (p_hi, p_hi, p_lo): p_hi w_hi + p_hi w_lo + p_lo w_hi
      std::vector<uint16_t> b((size_t)kC0 * 64, 0);
      for (int ch = 0; ch < kC0; ++ch)
        for (int k = 0; k < 9; ++k) {
          const float v = wc[ch * 9 + k];
          const uint16_t hi = f2bf(v);
          float hf;
          const uint32_t hu = (uint32_t)hi << 16;
          std::memcpy(&hf, &hu, 4);
          const uint16_t lo = f2bf(v - hf);
          b[(size_t)ch * 64 + k] = hi;
          b[(size_t)ch * 64 + 9 + k] = lo;
          b[(size_t)ch * 64 + 18 + k] = hi;
        }
      uint16_t *d = up.alloc<uint16_t>(b.size());
      if (d && cudaMemcpy(d, b.data(), b.size() * 2, cudaMemcpyHostToDevice) != cudaSuccess) up.ok = false;
      m->conv0b = d;
    }
  }
  m->ln0 = up.f32(w->ln0, kC0);
  m->ln1 = up.f32(w->ln1, kC1);
  {
    std::vector<float> w1((size_t)kC1 * 9 * kC0);  // [c1][tap * c0 + ci]
    for (int o = 0; o < kC1; ++o)
      for (int ci = 0; ci < kC0; ++ci)
        for (int tap = 0; tap < 9; ++tap) w1[(size_t)o * 9 * kC0 + tap * kC0 + ci] = w->conv1[((size_t)o * kC0 + ci) * 9 + tap];
    m->conv1 = up.mat(w1);
  }
  m->in_proj = up.mat(w->in_proj, (size_t)H * kHidden);
  m->out_proj = up.mat(w->out_proj, (size_t)c.out_dim * H);
  m->out_bias = up.f32(w->out_bias, c.out_dim);
  m->embed = up.mat(w->embed, (size_t)c.embed_dim * c.out_dim);
  std::vector<float> R((size_t)kLeft * H), qs(kHeadDim);
  for (int i = 0; i < c.n_layers && up.ok; ++i) {
    const ae_host_layer &l = w->layers[i];
    LayerDev L;
    std::memset(&L, 0, sizeof(L));
    L.ff1_pre = up.f32(l.ff1_pre, H);
    L.ff1_post = up.f32(l.ff1_post, H);
    L.ff2_pre = up.f32(l.ff2_pre, H);
    L.ff2_post = up.f32(l.ff2_post, H);
    L.norm_pre_attn = up.f32(l.norm_pre_attn, H);
    L.norm_post_attn = up.f32(l.norm_post_attn, H);
    L.norm_out = up.f32(l.norm_out, H);
    L.lc_pre = up.f32(l.lc_pre, H);
    L.lc_norm = up.f32(l.lc_norm, H);
    {
      std::vector<float> t((size_t)kKernel * H);  // tap-major
      for (int ch = 0; ch < H; ++ch)
        for (int k = 0; k < kKernel; ++k) t[(size_t)k * H + ch] = l.lc_dw[(size_t)ch * kKernel + k];
      L.lc_dw = up.f32(t.data(), t.size());
    }
    float ks;
    attention_tables_host(l.relative_k, l.per_dim_scale, H, c.heads, kLeft, R.data(), qs.data(), &ks);
    m->k_scale = ks;
    L.R = up.f32(R.data(), R.size());
    L.qscale = up.f32(qs.data(), qs.size());
    const bool f8 = dtype == AE_FP8;
    if (f8) {
      L.q8_ff1_w1 = q8_of(l.clip_ff1_w1);
      L.q8_ff1_w2 = q8_of(l.clip_ff1_w2);
      L.q8_ff2_w1 = q8_of(l.clip_ff2_w1);
      L.q8_ff2_w2 = q8_of(l.clip_ff2_w2);
      L.q8_qkv = q8_of(l.clip_q);
      L.q8_lc_start = q8_of(l.clip_lc_start);
      L.ff1_w1 = up.mat_e4m3(l.ff1_w1, c.ffn, H, L.q8_ff1_w1, &L.cs_ff1_w1);
      L.ff1_w2 = up.mat_e4m3(l.ff1_w2, H, c.ffn, L.q8_ff1_w2, &L.cs_ff1_w2);
      L.ff2_w1 = up.mat_e4m3(l.ff2_w1, c.ffn, H, L.q8_ff2_w1, &L.cs_ff2_w1);
      L.ff2_w2 = up.mat_e4m3(l.ff2_w2, H, c.ffn, L.q8_ff2_w2, &L.cs_ff2_w2);
    } else {
      L.ff1_w1 = up.mat(l.ff1_w1, (size_t)c.ffn * H);
      L.ff1_w2 = up.mat(l.ff1_w2, (size_t)H * c.ffn);
      L.ff2_w1 = up.mat(l.ff2_w1, (size_t)c.ffn * H);
      L.ff2_w2 = up.mat(l.ff2_w2, (size_t)H * c.ffn);
    }
    {
      std::vector<float> qkv((size_t)3 * H * H);
      std::memcpy(qkv.data(), l.q, (size_t)H * H * 4);
      std::memcpy(qkv.data() + (size_t)H * H, l.k, (size_t)H * H * 4);
      std::memcpy(qkv.data() + (size_t)2 * H * H, l.v, (size_t)H * H * 4);
      L.qkv = f8 ? up.mat_e4m3(qkv, 3 * H, H, L.q8_qkv, &L.cs_qkv) : up.mat(qkv);
    }
    L.post = up.mat(l.post, (size_t)H * H);
    L.lc_end = up.mat(l.lc_end, (size_t)H * H);
    {
      std::vector<float> ls((size_t)2 * H * H);  // rows interleaved: (a_c, b_c) adjacent
      for (int r = 0; r < H; ++r) {
        std::memcpy(ls.data() + (size_t)(2 * r) * H, l.lc_start + (size_t)r * H, (size_t)H * 4);
        std::memcpy(ls.data() + (size_t)(2 * r + 1) * H, l.lc_start + (size_t)(H + r) * H, (size_t)H * 4);
      }
      L.lc_start = f8 ? up.mat_e4m3(ls, 2 * H, H, L.q8_lc_start, &L.cs_lc_start) : up.mat(ls);
    }
    L.c_ff1_w1 = l.clip_ff1_w1; L.c_ff1_w2 = l.clip_ff1_w2; L.c_ff2_w1 = l.clip_ff2_w1; L.c_ff2_w2 = l.clip_ff2_w2;
    L.c_q = l.clip_q; L.c_k = l.clip_k; L.c_v = l.clip_v; L.c_post = l.clip_post;
    L.c_lc_start = l.clip_lc_start; L.c_lc_end = l.clip_lc_end;
    m->layers.push_back(L);
  }
  if (c.n_layers == 0) m->k_scale = (float)(std::log(1.0 + std::exp(1.0)) / std::log(2.0));
  if (!up.ok) {
    ae_model_destroy(m);
    return fail(AE_ENOMEM, "device allocation or copy failed while uploading the weights");
  }
  if (dtype != AE_F32) {
    bool ok = make_tmap_2d_bf16(&m->tm_conv1, m->conv1, 9 * kC0, kC1, 9 * kC0 * 2, 64, kC1) &&
              make_tmap_2d_bf16(&m->tm_in_proj, m->in_proj, kHidden, H, kHidden * 2, 64, 128) &&
              make_tmap_2d_bf16(&m->tm_out_proj, m->out_proj, H, c.out_dim, H * 2, 64, 128) &&
              make_tmap_2d_bf16(&m->tm_embed, m->embed, c.out_dim, c.embed_dim, c.out_dim * 2, 64, 128);
    for (auto &L : m->layers) {
      if (dtype == AE_FP8) {  // 8-bit maps: one 128-byte row segment = 128 codes
        ok = ok && make_tmap_2d_u8(&L.tm_ff1_w1, L.ff1_w1, H, c.ffn, H, 128, 128) &&
             make_tmap_2d_u8(&L.tm_ff1_w2, L.ff1_w2, c.ffn, H, (uint64_t)c.ffn, 128, 128) &&
             make_tmap_2d_u8(&L.tm_ff2_w1, L.ff2_w1, H, c.ffn, H, 128, 128) &&
             make_tmap_2d_u8(&L.tm_ff2_w2, L.ff2_w2, c.ffn, H, (uint64_t)c.ffn, 128, 128) &&
             make_tmap_2d_u8(&L.tm_qkv, L.qkv, H, 3 * H, H, 128, 128) &&
             make_tmap_2d_bf16(&L.tm_post, L.post, H, H, H * 2, 64, 128) &&
             make_tmap_2d_u8(&L.tm_lc_start, L.lc_start, H, 2 * H, H, 128, 128) &&
             make_tmap_2d_bf16(&L.tm_lc_end, L.lc_end, H, H, H * 2, 64, 128);
        continue;
      }
      ok = ok && make_tmap_2d_bf16(&L.tm_ff1_w1, L.ff1_w1, H, c.ffn, H * 2, 64, 128) &&
           make_tmap_2d_bf16(&L.tm_ff1_w2, L.ff1_w2, c.ffn, H, (uint64_t)c.ffn * 2, 64, 128) &&
           make_tmap_2d_bf16(&L.tm_ff2_w1, L.ff2_w1, H, c.ffn, H * 2, 64, 128) &&
           make_tmap_2d_bf16(&L.tm_ff2_w2, L.ff2_w2, c.ffn, H, (uint64_t)c.ffn * 2, 64, 128) &&
           make_tmap_2d_bf16(&L.tm_qkv, L.qkv, H, 3 * H, H * 2, 64, 128) &&
           make_tmap_2d_bf16(&L.tm_post, L.post, H, H, H * 2, 64, 128) &&
           make_tmap_2d_bf16(&L.tm_lc_start, L.lc_start, H, 2 * H, H * 2, 64, 128) &&
           make_tmap_2d_bf16(&L.tm_lc_end, L.lc_end, H, H, H * 2, 64, 128);
    }
    if (!ok) {
      ae_model_destroy(m);
      return fail(AE_ECUDA, "tensor map encoding failed");
    }
  }
  *out = m;
  return AE_OK;
}

size_t ae_workspace_size(const ae_model *m, int64_t n_clips, int64_t total_frames, int64_t total_tokens) {
  if (n_clips < 0 || total_frames < 0 || total_tokens < 0) return 0;
  if (!m) return ws_layout(m, n_clips, total_frames, total_tokens, false).total;
  return encode_ws_bytes(m, n_clips, total_frames, total_tokens);
}

ae_status ae_logmel(const float *d_wave, const int64_t *h_sample_off, int n_clips, float *d_mel, void *d_ws,
                    size_t ws_bytes, ae_stream stream) {
  ClipTables T;
  ae_status st = build_tables(h_sample_off, n_clips, kSamples, T, "h_sample_off");
  if (st) return st;
  if (T.total_frames > 0 && (!d_wave || !d_mel)) return fail(AE_EINVAL, "d_wave or d_mel is null");
  const WsLayout L = ws_layout(nullptr, T.n_clips, T.total_frames, 0, false);  // no token positions needed
  if (n_clips == 0) return AE_OK;
  if ((st = check_ws(d_ws, ws_bytes, L.total))) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  ClipTablesDev td;
  cudaError_t e = tables_t(T, d_ws, L, &td, false, s);
  if (e != cudaSuccess) return cuda_fail(e, "table upload");
  if ((e = logmel_t(d_wave, d_mel, td, T, s)) != cudaSuccess) return cuda_fail(e, "logmel");
  return AE_OK;
}

ae_status ae_subsample(const ae_model *m, const float *d_mel, const int64_t *h_frame_off, int n_clips, float *d_h,
                       void *d_ws, size_t ws_bytes, ae_stream stream) {
  ae_status st = check_model(m);
  if (st) return st;
  ClipTables T;
  if ((st = build_tables(h_frame_off, n_clips, kFrames, T, "h_frame_off"))) return st;
  if (T.total_tokens > 0 && (!d_mel || !d_h)) return fail(AE_EINVAL, "d_mel or d_h is null");
  if (!aligned16(d_h)) return fail(AE_EINVAL, "d_h is not 16-byte aligned");
  const WsLayout L = ws_layout(m, T.n_clips, T.total_frames, T.total_tokens, true);
  if (n_clips == 0) return AE_OK;
  if ((st = check_ws(d_ws, ws_bytes, L.total))) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  ClipTablesDev td;
  cudaError_t e = tables_t(T, d_ws, L, &td, false, s);
  if (e != cudaSuccess) return cuda_fail(e, "table upload");
  if (T.total_tokens == 0) return AE_OK;
  uint8_t *w = static_cast<uint8_t *>(d_ws);
  if ((e = conv0_t(m, d_mel, w + L.y0, td, T, s)) != cudaSuccess) return cuda_fail(e, "conv0");
  if ((e = conv1_t(m, w + L.y0, w + L.xs, td, T, s)) != cudaSuccess)
    return cuda_fail(e, "conv1");
  if ((e = gemm_t(m, w + L.xs, T.total_tokens, kHidden, m->in_proj, m->dtype != AE_F32 ? &m->tm_in_proj : nullptr,
                m->cfg.hidden, EPI_F32, ep_of(d_h, m->cfg.hidden, -INFINITY, INFINITY), s)) != cudaSuccess)
    return cuda_fail(e, "in_proj");
  return AE_OK;
}

ae_status ae_conformer_layer(const ae_model *m, int layer, float *d_h, const int64_t *h_tok_off, int n_clips,
                             void *d_ws, size_t ws_bytes, ae_stream stream) {
  ae_status st = check_model(m);
  if (st) return st;
  if (layer < 0 || layer >= m->cfg.n_layers) return fail(AE_EINVAL, "layer index out of range");
  ClipTables T;
  if ((st = build_tables(h_tok_off, n_clips, kTokens, T, "h_tok_off"))) return st;
  if (T.total_tokens > 0 && !d_h) return fail(AE_EINVAL, "d_h is null");
  const WsLayout L = ws_layout(m, T.n_clips, T.total_frames, T.total_tokens, true);
  if (T.total_tokens == 0) return AE_OK;
  if ((st = check_ws(d_ws, ws_bytes, L.total))) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  ClipTablesDev td;
  cudaError_t e = tables_t(T, d_ws, L, &td, true, s);
  if (e != cudaSuccess) return cuda_fail(e, "table upload");
  Bufs b = bufs_of(d_ws, L, td);
  b.h = d_h;
  if ((e = run_layer(m, layer, b, T.total_tokens, false, kNextNone, s)) != cudaSuccess) return cuda_fail(e, "layer");
  return AE_OK;
}

ae_status ae_encode(const ae_model *m, const float *d_wave, const int64_t *h_sample_off, int n_clips, float *d_out,
                    void *d_ws, size_t ws_bytes, ae_stream stream) {
  ae_status st = check_model(m);
  if (st) return st;
  ClipTables T;
  if ((st = build_tables(h_sample_off, n_clips, kSamples, T, "h_sample_off"))) return st;
  if (T.total_tokens > 0 && (!d_wave || !d_out)) return fail(AE_EINVAL, "d_wave or d_out is null");
  if (!aligned16(d_out)) return fail(AE_EINVAL, "d_out is not 16-byte aligned");
  const size_t need = encode_ws_bytes(m, T.n_clips, T.total_frames, T.total_tokens);
  if (n_clips == 0) return AE_OK;
  if ((st = check_ws(d_ws, ws_bytes, need))) return st;
  return encode_dev(m, d_wave, T, d_out, d_ws, need, reinterpret_cast<cudaStream_t>(stream), true);
}

ae_status ae_encode_trace(const ae_model *m, const float *d_wave, const int64_t *h_sample_off, int n_clips,
                          float *d_out, float *d_mel, float *d_trace, void *d_ws, size_t ws_bytes, ae_stream stream) {
  ae_status st = check_model(m);
  if (st) return st;
  ClipTables T;
  if ((st = build_tables(h_sample_off, n_clips, kSamples, T, "h_sample_off"))) return st;
  if (T.total_tokens > 0 && (!d_wave || !d_out)) return fail(AE_EINVAL, "d_wave or d_out is null");
  if (!aligned16(d_out)) return fail(AE_EINVAL, "d_out is not 16-byte aligned");
  const size_t need = encode_ws_bytes(m, T.n_clips, T.total_frames, T.total_tokens);
  if (n_clips == 0) return AE_OK;
  if ((st = check_ws(d_ws, ws_bytes, need))) return st;
  TraceOut tr;
  tr.mel = d_mel;
  tr.layers = d_trace;
  const WsLayout L = ws_layout(m, T.n_clips, T.total_frames, T.total_tokens, true);
  return encode_one(m, d_wave, T, d_out, d_ws, L, reinterpret_cast<cudaStream_t>(stream), &tr);
}

size_t ae_encode_host_workspace_size(const ae_model *m, const int64_t *h_sample_off, int n_clips) {
  ClipTables T;
  if (!m || build_tables(h_sample_off, n_clips, kSamples, T, "h_sample_off") != AE_OK) return 0;
  return encode_ws_bytes(m, T.n_clips, T.total_frames, T.total_tokens) + al256((size_t)T.total_samples * 4) +
         al256((size_t)T.total_tokens * m->cfg.embed_dim * 4);
}

static ae_status encode_host(const ae_model *m, const float *h_wave, const int64_t *h_sample_off, int n_clips,
                             float *h_out, void *d_ws, size_t ws_bytes, ae_stream stream, bool may_split) {
  ae_status st = check_model(m);
  if (st) return st;
  ClipTables T;
  if ((st = build_tables(h_sample_off, n_clips, kSamples, T, "h_sample_off"))) return st;
  if (T.total_samples > 0 && !h_wave) return fail(AE_EINVAL, "h_wave is null");
  if (T.total_tokens > 0 && !h_out) return fail(AE_EINVAL, "h_out is null");
  const size_t enc = encode_ws_bytes(m, T.n_clips, T.total_frames, T.total_tokens);
  const size_t wave_b = al256((size_t)T.total_samples * 4);
  const size_t out_b = al256((size_t)T.total_tokens * m->cfg.embed_dim * 4);
  if (n_clips == 0) return AE_OK;
  if ((st = check_ws(d_ws, ws_bytes, enc + wave_b + out_b))) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *w = static_cast<uint8_t *>(d_ws);
  float *d_wave = reinterpret_cast<float *>(w + enc);
  float *d_out = reinterpret_cast<float *>(w + enc + wave_b);
  cudaError_t e;
  if (T.total_samples > 0 &&
      (e = cudaMemcpyAsync(d_wave, h_wave, (size_t)T.total_samples * 4, cudaMemcpyHostToDevice, s)) != cudaSuccess)
    return cuda_fail(e, "copy in");
  if ((st = encode_dev(m, d_wave, T, d_out, d_ws, enc, s, may_split))) return st;
  if (T.total_tokens > 0 &&
      (e = cudaMemcpyAsync(h_out, d_out, (size_t)T.total_tokens * m->cfg.embed_dim * 4, cudaMemcpyDeviceToHost, s)) !=
          cudaSuccess)
    return cuda_fail(e, "copy out");
  return AE_OK;
}

ae_status ae_encode_host_async(const ae_model *m, const float *h_wave, const int64_t *h_sample_off, int n_clips,
                               float *h_out, void *d_ws, size_t ws_bytes, ae_stream stream) {
  return encode_host(m, h_wave, h_sample_off, n_clips, h_out, d_ws, ws_bytes, stream, false);
}

ae_status ae_encode_host(const ae_model *m, const float *h_wave, const int64_t *h_sample_off, int n_clips,
                         float *h_out, void *d_ws, size_t ws_bytes, ae_stream stream) {
  ae_status st = encode_host(m, h_wave, h_sample_off, n_clips, h_out, d_ws, ws_bytes, stream, true);
  if (st) return st;
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream");
  return AE_OK;
}

ae_status ae_local_attention(const void *d_q, const void *d_k, const void *d_v, int64_t ld_qkv, ae_dtype dtype,
                             const float *d_R, const float *d_qscale, float k_scale, float softcap,
                             const int64_t *h_tok_off, int n_clips, void *d_out, int64_t ld_out, void *d_ws,
                             size_t ws_bytes, ae_stream stream) {
  if (dtype != AE_F32 && dtype != AE_BF16) return fail(AE_EINVAL, "dtype");
  ClipTables T;
  ae_status st = build_tables(h_tok_off, n_clips, kTokens, T, "h_tok_off");
  if (st) return st;
  if (T.total_tokens > 0) {
    if (!d_q || !d_k || !d_v || !d_out || !d_R || !d_qscale) return fail(AE_EINVAL, "a device pointer is null");
    if (!aligned16(d_q) || !aligned16(d_k) || !aligned16(d_v) || !aligned16(d_out) || !aligned16(d_R))
      return fail(AE_EINVAL, "q, k, v, out and R must be 16-byte aligned");
    const int64_t vec = dtype == AE_BF16 ? 8 : 4;
    if (ld_qkv < kHidden || ld_out < kHidden || ld_qkv % vec || ld_out % vec)
      return fail(AE_EINVAL, "row strides must be >= 1024 and a multiple of 16 bytes");
    if (!(softcap > 0.f) || !std::isfinite(softcap) || !std::isfinite(k_scale))
      return fail(AE_EINVAL, "softcap must be positive and finite");
  }
  const WsLayout L = ws_layout(nullptr, T.n_clips, 0, T.total_tokens, false);
  if (T.total_tokens == 0) return AE_OK;
  if ((st = check_ws(d_ws, ws_bytes, L.total))) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  ClipTablesDev td;
  cudaError_t e = tables_t(T, d_ws, L, &td, true, s);
  if (e != cudaSuccess) return cuda_fail(e, "table upload");
  const double abytes = 4.0 * (dtype == AE_BF16 ? 2 : 4) * kHidden * (double)T.total_tokens;
  if ((e = timed(AE_K_ATTENTION, 0.0, abytes, s, [&] {
         return launch_attention(dtype == AE_BF16, d_q, d_k, d_v, ld_qkv, d_R, d_qscale, k_scale, softcap, td.pos,
                                 T.total_tokens, d_out, ld_out, -INFINITY, INFINITY, s);
       })) != cudaSuccess)
    return cuda_fail(e, "attention");
  return AE_OK;
}

ae_status ae_linear_e4m3(const void *d_x, const void *d_w, const float *d_cs, int64_t M, int32_t N, int32_t K,
                         float lo, float hi, ae_lin_out out, float lo2, float hi2, float q_out, void *d_y,
                         ae_stream stream) {
  if (out != AE_LIN_BF16 && out != AE_LIN_SILU_E4M3) return fail(AE_EINVAL, "out");
  if (M < 0 || M > INT32_MAX) return fail(AE_EINVAL, "M must be in [0, 2^31)");
  if (K <= 0 || K % 128 || K > 65536) return fail(AE_EINVAL, "K must be a positive multiple of 128 up to 65536");
  if (N <= 0 || N % 256 || N > 65536) return fail(AE_EINVAL, "N must be a positive multiple of 256 up to 65536");
  if (std::isnan(lo) || std::isnan(hi) || lo > hi) return fail(AE_EINVAL, "lo, hi");
  if (out == AE_LIN_SILU_E4M3 && (std::isnan(lo2) || std::isnan(hi2) || lo2 > hi2 || !(q_out > 0.f) ||
                                  !std::isfinite(q_out)))
    return fail(AE_EINVAL, "lo2, hi2 or q_out");
  if (M == 0) return AE_OK;
  if (!d_x || !d_w || !d_cs || !d_y) return fail(AE_EINVAL, "a device pointer is null");
  if (!aligned16(d_x) || !aligned16(d_w) || !aligned16(d_cs) || (reinterpret_cast<uintptr_t>(d_y) & 31))
    return fail(AE_EINVAL, "x, w and cs must be 16-byte aligned, y 32-byte aligned");
  CUtensorMap tW;
  if (!make_tmap_2d_u8(&tW, d_w, (uint64_t)K, (uint64_t)N, (uint64_t)K, 128, 128))
    return fail(AE_ECUDA, "tensor map encoding failed");
  EpiArgs e = ep_of(d_y, N, lo, hi);
  e.cs = d_cs;
  if (out == AE_LIN_SILU_E4M3) {
    e.lo2 = lo2;
    e.hi2 = hi2;
    e.clamp2 = silu_clamp_binds(hi, lo2, hi2);
    e.q8 = q_out;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const cudaError_t err = gemm8_t(d_x, M, K, tW, N, out == AE_LIN_BF16 ? EPI_BF16 : EPI_SILU_Q8, e, s);
  if (err != cudaSuccess) return cuda_fail(err, "e4m3 projection");
  return AE_OK;
}

// ------------------------------------------------------------------ second log-mel front-end

namespace {
bool lfm_cfg_ok(const ae_lfm_config *c) {
  return c && c->n_fft == 512 && c->win_length >= 2 && c->win_length <= 512 && c->win_length % 2 == 0 &&
         c->hop >= 2 && c->hop <= 320 && c->hop % 2 == 0 && c->n_mels >= 1 && c->n_mels <= kLfmMaxMels &&
         c->sample_rate >= 1000 && c->sample_rate <= 1000000 && std::isfinite(c->preemph) &&
         std::isfinite(c->log_floor) && c->log_floor > 0.f && std::isfinite(c->var_eps) && c->var_eps > 0.f;
}

struct LfmLayout {
  size_t sample_off, frame_off, tile_off, eff, bank_lo, bank_cnt, bank_off, bank_w, moments, total;
};
LfmLayout lfm_layout(int n_clips) {
  LfmLayout L;
  const size_t B1 = (size_t)n_clips + 1;
  size_t off = 0;
  L.sample_off = off; off += al256(B1 * 8);
  L.frame_off = off; off += al256(B1 * 4);
  L.tile_off = off; off += al256(B1 * 4);
  L.eff = off; off += al256(std::max<size_t>(n_clips, 1) * 4);
  L.bank_lo = off; off += al256((size_t)kLfmMaxMels * 4);
  L.bank_cnt = off; off += al256((size_t)kLfmMaxMels * 4);
  L.bank_off = off; off += al256((size_t)kLfmMaxMels * 4);
  L.bank_w = off; off += al256((size_t)kLfmMaxMels * kLfmMaxBins * 4);
  L.moments = off; off += al256(std::max<size_t>(n_clips, 1) * kLfmMaxMels * 2 * 8);
  L.total = off;
  return L;
}
}  // namespace

void ae_lfm_default_config(ae_lfm_config *cfg) {
  if (!cfg) return;
  cfg->sample_rate = 16000;
  cfg->n_fft = 512;
  cfg->win_length = 400;
  cfg->hop = 160;
  cfg->n_mels = 128;
  cfg->preemph = 0.97f;
  cfg->log_floor = 5.9604644775390625e-08f;  // 2^-24
  cfg->var_eps = 1e-5f;
}

int64_t ae_lfm_num_frames(const ae_lfm_config *cfg, int64_t n_samples) {
  if (!lfm_cfg_ok(cfg)) return -1;
  return n_samples > 0 ? 1 + n_samples / cfg->hop : 0;
}

size_t ae_lfm_workspace_size(const ae_lfm_config *cfg, int n_clips) {
  if (!lfm_cfg_ok(cfg) || n_clips < 0) return 0;
  return lfm_layout(n_clips).total;
}

ae_status ae_lfm_logmel(const ae_lfm_config *cfg, const float *d_wave, const int64_t *h_sample_off, int n_clips,
                        float *d_out, void *d_ws, size_t ws_bytes, ae_stream stream) {
  if (!cfg) return fail(AE_EINVAL, "cfg is null");
  if (!lfm_cfg_ok(cfg))
    return fail(AE_EUNSUPPORTED, "supported: n_fft 512, even win_length in [2, 512], even hop in [2, 320], n_mels "
                                 "in [1, 128], sample_rate in [1000, 1e6], finite preemph, log_floor > 0, var_eps > 0");
  if (n_clips < 0 || n_clips > kMaxClips) return fail(AE_EINVAL, "n_clips out of range");
  if (!h_sample_off) return fail(AE_EINVAL, "h_sample_off is null");
  if (h_sample_off[0] != 0) return fail(AE_EINVAL, "h_sample_off[0] must be 0");
  std::vector<int64_t> so(h_sample_off, h_sample_off + n_clips + 1);
  std::vector<int32_t> fo(n_clips + 1, 0), to(n_clips + 1, 0), eff(std::max(n_clips, 1), 0);
  int64_t frames = 0, tiles = 0;
  for (int i = 0; i < n_clips; ++i) {
    const int64_t n = so[i + 1] - so[i];
    if (n < 0) return fail(AE_EINVAL, "h_sample_off is not non-decreasing at clip " + std::to_string(i));
    const int64_t nf = n > 0 ? 1 + n / cfg->hop : 0;
    frames += nf;
    tiles += (nf + kLfmTile - 1) / kLfmTile;
    if (frames > INT32_MAX) return fail(AE_EINVAL, "more than 2^31 - 1 frames in one call");
    fo[i + 1] = (int32_t)frames;
    to[i + 1] = (int32_t)tiles;
    eff[i] = (int32_t)((n + cfg->hop - 1) / cfg->hop);
  }
  // the packed bank of the last configuration this thread used (built in
  // float64 on the host; the sample rate, n_fft and n_mels decide it)
  thread_local struct {
    int32_t sr = 0, n_fft = 0, n_mels = 0;
    bool ok = false;
    LfmPackedBank P;
  } bank;
  if (bank.sr != cfg->sample_rate || bank.n_fft != cfg->n_fft || bank.n_mels != cfg->n_mels) {
    std::vector<int32_t> blo;
    std::vector<float> bw;
    int widest = 0;
    bank.ok = lfm_bank(*cfg, blo, bw, &widest, kLfmMaxBins);
    bank.P = bank.ok ? lfm_bank_pack(blo, bw, cfg->n_mels, kLfmMaxBins, kLfmWarps) : LfmPackedBank{};
    bank.sr = cfg->sample_rate;
    bank.n_fft = cfg->n_fft;
    bank.n_mels = cfg->n_mels;
  }
  if (!bank.ok) return fail(AE_EUNSUPPORTED, "a mel band spans more than 32 FFT bins");
  const LfmPackedBank &P = bank.P;
  if (frames == 0) return AE_OK;
  if (!d_wave || !d_out) return fail(AE_EINVAL, "d_wave or d_out is null");
  if (!aligned16(d_out)) return fail(AE_EINVAL, "d_out must be 16-byte aligned");
  const LfmLayout L = lfm_layout(n_clips);
  ae_status st = check_ws(d_ws, ws_bytes, L.total);
  if (st) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *w = static_cast<uint8_t *>(d_ws);
  std::vector<uint8_t> h(L.bank_w + P.w.size() * 4, 0);  // the tables up to the packed weights in use
  auto put = [&](const void *src, size_t bytes, size_t off) { if (bytes) std::memcpy(h.data() + off, src, bytes); };
  put(so.data(), so.size() * 8, L.sample_off);
  put(fo.data(), fo.size() * 4, L.frame_off);
  put(to.data(), to.size() * 4, L.tile_off);
  put(eff.data(), eff.size() * 4, L.eff);
  put(P.lo.data(), P.lo.size() * 4, L.bank_lo);
  put(P.cnt.data(), P.cnt.size() * 4, L.bank_cnt);
  put(P.off.data(), P.off.size() * 4, L.bank_off);
  put(P.w.data(), P.w.size() * 4, L.bank_w);
  cudaError_t e = launch_upload_bytes(h.data(), h.size(), w, s);
  if (e != cudaSuccess) return cuda_fail(e, "table upload");
  LfmTablesDev t;
  t.n_clips = n_clips;
  t.n_tiles = (int)tiles;
  t.sample_off = reinterpret_cast<const int64_t *>(w + L.sample_off);
  t.frame_off = reinterpret_cast<const int32_t *>(w + L.frame_off);
  t.tile_off = reinterpret_cast<const int32_t *>(w + L.tile_off);
  t.eff = reinterpret_cast<const int32_t *>(w + L.eff);
  t.bank_lo = reinterpret_cast<const int32_t *>(w + L.bank_lo);
  t.bank_cnt = reinterpret_cast<const int32_t *>(w + L.bank_cnt);
  t.bank_off = reinterpret_cast<const int32_t *>(w + L.bank_off);
  t.bank_w = reinterpret_cast<const float *>(w + L.bank_w);
  t.moments = reinterpret_cast<unsigned long long *>(w + L.moments);
  LfmParams prm;
  prm.n_mels = cfg->n_mels;
  prm.hop = cfg->hop;
  prm.win_length = cfg->win_length;
  prm.nnz = (int)P.w.size();
  prm.wave_floats = ((kLfmTile - 1) * cfg->hop + 516 + 3) / 4 * 4;  // span + the predecessor + alignment shift
  prm.vec16 = aligned16(d_wave) ? 1 : 0;
  prm.preemph = cfg->preemph;
  prm.log_floor = cfg->log_floor;
  prm.var_eps = cfg->var_eps;
  for (int i = 0; i <= kLfmWarps; ++i) prm.wband[i] = P.wband[i];
  const double bytes = 4.0 * (double)so[n_clips] + 12.0 * (double)frames * cfg->n_mels;
  if ((e = timed(AE_K_LFM, 0.0, bytes, s, [&] { return launch_lfm(d_wave, d_out, t, prm, s); })) != cudaSuccess)
    return cuda_fail(e, "lfm front-end");
  return AE_OK;
}

// ------------------------------------------------------------------ mixdown and resampling

namespace {
constexpr int32_t kMaxRate = 1000000;
constexpr int kMaxChannels = 64;
constexpr int64_t kMaxRsTable = int64_t(1) << 26;  // taps in the per-call table
constexpr int64_t kMaxRsSamples = int64_t(1) << 40;

struct RsTables {
  std::vector<int64_t> in_off, out_off;
  std::vector<int32_t> tile_off;
  int64_t total_in = 0, total_out = 0;
  int64_t n_tiles = 0;
};

struct RsLayout {
  size_t in_off = 0, out_off = 0, tile_off = 0, lo = 0, coef = 0, bmat = 0, mono = 0, total = 0;
};

ae_status rs_check_rates(int32_t rate_in, int32_t rate_out) {
  if (rate_in <= 0 || rate_out <= 0 || rate_in > kMaxRate || rate_out > kMaxRate)
    return fail(AE_EINVAL, "rates must be in 1 .. 1000000");
  return AE_OK;
}

ae_status rs_tables(const int64_t *off, int n, int32_t rate_in, int32_t rate_out, const RsPlan &pl, RsTables &t) {
  if (n < 0) return fail(AE_EINVAL, "n_clips is negative");
  if (n > kMaxClips) return fail(AE_EINVAL, "n_clips above 1048576");
  if (!off) return fail(AE_EINVAL, "h_sample_off is null");
  if (off[0] != 0) return fail(AE_EINVAL, "h_sample_off[0] must be 0");
  t = RsTables();
  t.in_off.assign(n + 1, 0);
  t.out_off.assign(n + 1, 0);
  t.tile_off.assign(n + 1, 0);
  for (int i = 0; i < n; ++i) {
    const int64_t len = off[i + 1] - off[i];
    if (len < 0) return fail(AE_EINVAL, "h_sample_off is not non-decreasing at clip " + std::to_string(i));
    t.in_off[i + 1] = off[i + 1];
    const int64_t out = rs_len(len, rate_in, rate_out);
    t.out_off[i + 1] = t.out_off[i] + out;
    const int64_t units = (out + pl.U - 1) / pl.U, per_type = (units + pl.NT - 1) / pl.NT;
    // tensor-core form: tiles of 128 rows of tcN outputs
    const int64_t tiles = rate_in == rate_out ? 0
                          : pl.tc         ? ((out + pl.tcN - 1) / pl.tcN + 127) / 128
                                          : (per_type + pl.Q - 1) / pl.Q;
    if ((t.n_tiles + tiles) * pl.n_groups > INT32_MAX)
      return fail(AE_EUNSUPPORTED, "too many resampler tiles in one call");
    t.n_tiles += tiles;
    t.tile_off[i + 1] = (int32_t)t.n_tiles;
  }
  t.total_in = off[n];
  t.total_out = t.out_off[n];
  if (t.total_in > kMaxRsSamples) return fail(AE_EINVAL, "more than 2^40 input samples");
  return AE_OK;
}

RsLayout rs_layout(int n_clips, const RsPlan &pl, int64_t total_in, int channels, bool equal) {
  RsLayout L;
  size_t off = 0;
  const size_t B1 = (size_t)n_clips + 1;
  L.in_off = off;
  off += al256(B1 * 8);
  L.out_off = off;
  off += al256(B1 * 8);
  L.tile_off = off;
  off += al256(B1 * 4);
  L.lo = off;
  off += equal || pl.tc ? 0 : al256((size_t)pl.NT * 4);
  L.coef = off;
  off += equal || pl.tc ? 0 : al256((size_t)pl.NT * pl.W_pad * pl.U * 4);
  L.bmat = off;  // the tensor-core form's taps: bf16 high and low parts, [tcN][tcK] each
  off += !equal && pl.tc ? al256((size_t)2 * pl.tcN * pl.tcK * 2) : 0;
  L.mono = off;
  off += (channels > 1 && !equal) ? al256((size_t)total_in * 4) : 0;
  L.total = off;
  return L;
}
}  // namespace

int64_t ae_resample_len(int64_t n_samples, int32_t rate_in, int32_t rate_out) {
  if (rate_in > kMaxRate || rate_out > kMaxRate) return -1;
  return rs_len(n_samples, rate_in, rate_out);
}

size_t ae_resample_workspace_size(const int64_t *h_sample_off, int n_clips, int32_t rate_in, int32_t rate_out,
                                  int channels) {
  if (rs_check_rates(rate_in, rate_out) || channels < 1 || channels > kMaxChannels) return 0;
  const RsPlan pl = rs_plan(rate_in, rate_out);
  RsTables T;
  if (rs_tables(h_sample_off, n_clips, rate_in, rate_out, pl, T) != AE_OK) return 0;
  return rs_layout(n_clips, pl, T.total_in, channels, rate_in == rate_out).total;
}

ae_status ae_partition_clips(const int64_t *h_sample_off, int n_clips, int n_parts, int32_t *h_part,
                             int64_t *h_tokens) {
  if (n_parts < 1 || n_parts > 65536) return fail(AE_EINVAL, "n_parts must lie in [1, 65536]");
  if (n_clips < 0) return fail(AE_EINVAL, "n_clips is negative");
  if (!h_sample_off) return fail(AE_EINVAL, "h_sample_off is null");
  if (n_clips > 0 && !h_part) return fail(AE_EINVAL, "h_part is null");
  if (h_sample_off[0] != 0) return fail(AE_EINVAL, "h_sample_off[0] must be 0");
  std::vector<int64_t> tok((size_t)n_clips);
  for (int i = 0; i < n_clips; ++i) {
    const int64_t n = h_sample_off[i + 1] - h_sample_off[i];
    if (n < 0) return fail(AE_EINVAL, "h_sample_off is not non-decreasing at clip " + std::to_string(i));
    tok[(size_t)i] = tokens_of_frames(frames_of_samples(n));
  }
  std::vector<int> order((size_t)n_clips);
  for (int i = 0; i < n_clips; ++i) order[(size_t)i] = i;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return tok[(size_t)a] > tok[(size_t)b]; });
  // min-heap of (tokens so far, part index): the lightest part, lowest index first
  using Load = std::pair<int64_t, int>;
  std::vector<Load> heap((size_t)n_parts);
  for (int p = 0; p < n_parts; ++p) heap[(size_t)p] = Load(0, p);
  auto heavier = [](const Load &a, const Load &b) { return a > b; };
  std::make_heap(heap.begin(), heap.end(), heavier);
  for (int i : order) {
    std::pop_heap(heap.begin(), heap.end(), heavier);
    Load &l = heap.back();
    h_part[i] = l.second;
    l.first += tok[(size_t)i];
    std::push_heap(heap.begin(), heap.end(), heavier);
  }
  if (h_tokens)
    for (const Load &l : heap) h_tokens[l.second] = l.first;
  return AE_OK;
}

ae_status ae_resample(const float *d_x, int channels, int64_t ch_stride, const int64_t *h_sample_off, int n_clips,
                      int32_t rate_in, int32_t rate_out, float *d_y, void *d_ws, size_t ws_bytes,
                      ae_stream stream) {
  ae_status st = rs_check_rates(rate_in, rate_out);
  if (st) return st;
  if (channels < 1 || channels > kMaxChannels) return fail(AE_EINVAL, "channels must be in 1 .. 64");
  const RsPlan pl = rs_plan(rate_in, rate_out);
  const bool equal = rate_in == rate_out;
  if (!equal && (int64_t)pl.NT * pl.W_pad * pl.U > kMaxRsTable)
    return fail(AE_EUNSUPPORTED, "the reduced output rate " + std::to_string(pl.p) + " needs a tap table above 2^26");
  RsTables T;
  if ((st = rs_tables(h_sample_off, n_clips, rate_in, rate_out, pl, T))) return st;
  if (channels > 1 && ch_stride < T.total_in) return fail(AE_EINVAL, "ch_stride is below the packed sample count");
  if (T.total_in > 0 && (!d_x || !d_y)) return fail(AE_EINVAL, "d_x or d_y is null");
  const RsLayout L = rs_layout(n_clips, pl, T.total_in, channels, equal);
  if (T.total_out == 0) return AE_OK;
  if ((st = check_ws(d_ws, ws_bytes, L.total))) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *w = static_cast<uint8_t *>(d_ws);
  cudaError_t e;
  const double in_bytes = 4.0 * channels * (double)T.total_in, out_bytes = 4.0 * (double)T.total_out;
  if (equal) {  // mono is the output
    if ((e = timed(AE_K_RESAMPLE, 0.0, in_bytes + out_bytes, s, [&] {
           return launch_rs_mix(d_x, channels, ch_stride, T.total_in, d_y, s);
         })) != cudaSuccess)
      return cuda_fail(e, "mixdown");
    return AE_OK;
  }
  int64_t *in_off = reinterpret_cast<int64_t *>(w + L.in_off);
  int64_t *out_off = reinterpret_cast<int64_t *>(w + L.out_off);
  int32_t *tile_off = reinterpret_cast<int32_t *>(w + L.tile_off);
  int32_t *lo = reinterpret_cast<int32_t *>(w + L.lo);
  float *coef = reinterpret_cast<float *>(w + L.coef);
  void *bmat = w + L.bmat;
  const float *mono = d_x;
  if ((e = timed(AE_K_TABLES, 0.0, 0.0, s, [&] {
         cudaError_t r = launch_upload_bytes(T.in_off.data(), T.in_off.size() * 8, in_off, s);
         if (r == cudaSuccess) r = launch_upload_bytes(T.out_off.data(), T.out_off.size() * 8, out_off, s);
         if (r == cudaSuccess) r = launch_upload_bytes(T.tile_off.data(), T.tile_off.size() * 4, tile_off, s);
         return r;
       })) != cudaSuccess)
    return cuda_fail(e, "table upload");
  if (pl.tc) {
    if ((e = timed(AE_K_RESAMPLE, 0.0, 4.0 * pl.tcN * pl.tcK, s, [&] { return launch_rs_btc(pl, bmat, s); })) !=
        cudaSuccess)
      return cuda_fail(e, "resampler taps");
  } else if ((e = timed(AE_K_RESAMPLE, 0.0, 4.0 * pl.U * pl.NT * pl.W_pad, s,
                        [&] { return launch_rs_table(pl, coef, lo, s); })) != cudaSuccess) {
    return cuda_fail(e, "resampler taps");
  }
  if (channels > 1) {
    float *m = reinterpret_cast<float *>(w + L.mono);
    if ((e = timed(AE_K_RESAMPLE, 0.0, in_bytes + 4.0 * T.total_in, s, [&] {
           return launch_rs_mix(d_x, channels, ch_stride, T.total_in, m, s);
         })) != cudaSuccess)
      return cuda_fail(e, "mixdown");
    mono = m;
  }
  const double taps = (double)(2 * (int)std::ceil(pl.half) + 1);
  if ((e = timed(AE_K_RESAMPLE, 2.0 * taps * (double)T.total_out, 4.0 * (double)T.total_in + out_bytes, s, [&] {
         if (pl.tc) return launch_rs_fir_tc(pl, mono, d_y, bmat, in_off, out_off, tile_off, n_clips, (int)T.n_tiles, s);
         return launch_rs_fir(pl, mono, d_y, coef, lo, in_off, out_off, tile_off, n_clips, (int)T.n_tiles, s);
       })) != cudaSuccess)
    return cuda_fail(e, "resampler");
  return AE_OK;
}

ae_status ae_logmel_noalloc(const float *d_wave, const int64_t *h_sample_off, int n_clips, float *d_mel,
                            ae_stream stream) {
  if (n_clips > kNoAllocMaxClips)
    return fail(AE_EINVAL, "ae_logmel_noalloc takes at most " + std::to_string(kNoAllocMaxClips) +
                               " clips per call (got " + std::to_string(n_clips) + "); split the batch");
  ClipTables T;
  ae_status st = build_tables(h_sample_off, n_clips, kSamples, T, "h_sample_off");
  if (st) return st;
  if (T.total_frames > 0 && (!d_wave || !d_mel)) return fail(AE_EINVAL, "d_wave or d_mel is null");
  if (n_clips == 0) return AE_OK;
  const WsLayout L = ws_layout(nullptr, T.n_clips, T.total_frames, 0, false);  // the tables alone
  if (L.total > kNoAllocScratchBytes) return fail(AE_EINVAL, "clip tables exceed the fixed scratch array");
  void *scratch = nullptr;
  if ((st = noalloc_scratch(&scratch))) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the upload rewrites every table word the front-end reads: nothing relies
  // on the array's earlier contents
  ClipTablesDev td;
  cudaError_t e = tables_t(T, scratch, L, &td, false, s);
  if (e != cudaSuccess) return cuda_fail(e, "table upload");
  if ((e = logmel_t(d_wave, d_mel, td, T, s)) != cudaSuccess) return cuda_fail(e, "logmel");
  return AE_OK;
}

ae_status ae_profile_enable(int on) {
  Profiler &P = g_prof;
  if (on && P.ev.empty()) {
    const size_t cap = 16384;
    P.ev.resize(2 * cap);
    for (auto &e : P.ev)
      if (cudaEventCreate(&e) != cudaSuccess) {
        for (auto &x : P.ev)
          if (x) cudaEventDestroy(x);
        P.ev.clear();
        return fail(AE_ECUDA, "could not create the timing events");
      }
    P.recs.resize(cap);
    P.cap = cap;
  }
  P.on = on != 0;
  return AE_OK;
}

ae_status ae_profile_read(double *ms, int64_t *launches, double *flops, double *bytes, int64_t *dropped) {
  Profiler &P = g_prof;
  double t[AE_K_COUNT] = {0}, f[AE_K_COUNT] = {0}, b[AE_K_COUNT] = {0};
  int64_t n[AE_K_COUNT] = {0};
  if (P.n > 0) {
    cudaError_t e = cudaEventSynchronize(P.ev[2 * P.n - 1]);
    if (e != cudaSuccess) return cuda_fail(e, "timing events");
    for (size_t i = 0; i < P.n; ++i) {
      float x = 0.f;
      if ((e = cudaEventElapsedTime(&x, P.ev[2 * i], P.ev[2 * i + 1])) != cudaSuccess) return cuda_fail(e, "timing");
      const int c = P.recs[i].cls;
      t[c] += x;
      n[c] += 1;
      f[c] += P.recs[i].flops;
      b[c] += P.recs[i].bytes;
    }
  }
  for (int c = 0; c < AE_K_COUNT; ++c) {
    if (ms) ms[c] = t[c];
    if (launches) launches[c] = n[c];
    if (flops) flops[c] = f[c];
    if (bytes) bytes[c] = b[c];
  }
  if (dropped) *dropped = P.dropped;
  P.n = 0;
  P.dropped = 0;
  return AE_OK;
}

}  // extern "C"
