// Host side of the LFM2A Conformer encoder (include/ae.h, ae_lenc_*): weight
// upload, per-call clip tables and workspace, and the sequence of kernels of
// encode_audio_gpu / macaron_ffn / conv_stem_gpu (cera 0.5.3,
// audio_encoder_gpu.rs).
//
// Layout choices: the stem's activations are channels-last bf16 rows, so the
// pointwise convolutions are GEMMs over positions and the flatten before
// pre_encode_out is free once that matrix's columns are permuted from the
// page's (channel, freq) order to (freq, channel) here. q, k and v are one
// stacked projection; pw1's rows are interleaved (a_c, b_c) so the GLU pairs
// land in one epilogue thread; the position projections of all layers are
// stacked into one matrix, so one GEMM per call gives every layer's position
// rows.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <string>
#include <vector>

#include "ae_internal.h"

struct ae_lenc {
  ae_lenc_config cfg;
  std::vector<void *> allocs;
  float *b0, *w1, *b1, *b2, *w3, *b3, *b4, *pre_b;
  void *w0b;  // the first stem convolution's taps as the tensor-core B operand (split in bf16 parts)
  void *w2, *w4, *pre_w;
  CUtensorMap tm_w2, tm_w4, tm_pre;
  struct Block {
    float *f1_nw, *f1_nb, *f1_ub, *f1_db, *ln1_w, *ln1_b, *qkv_b, *o_b, *bu, *bv;
    float *nc_w, *nc_b, *pw1_b, *dw_w, *dw_b, *cn_w, *cn_b, *pw2_b;
    float *f2_nw, *f2_nb, *f2_ub, *f2_db, *ln2_w, *ln2_b;
    void *f1_up, *f1_down, *qkv, *o, *pw1, *pw2, *f2_up, *f2_down;
    CUtensorMap tm_f1_up, tm_f1_down, tm_qkv, tm_o, tm_pw1, tm_pw2, tm_f2_up, tm_f2_down;
  };
  std::vector<Block> blocks;
  void *pos_w;  // [n_layers * n_embd][n_embd]
  CUtensorMap tm_pos;
  float *ad_nw, *ad_nb, *ad_ub, *ad_db;
  void *ad_up, *ad_down;
  CUtensorMap tm_ad_up, tm_ad_down;
};

namespace ae {
namespace {

ae_status lfail(ae_status st, const std::string &msg) {
  set_error(msg);
  return st;
}
ae_status lcuda(cudaError_t e, const char *where) {
  return lfail(AE_ECUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

uint16_t to_bf16(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return 0x7fc0;
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

float from_bf16(uint16_t b) {
  const uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

int64_t half_up(int64_t n) { return n > 0 ? (n + 1) / 2 : 0; }
int64_t stem_tokens(int64_t F) { return half_up(half_up(half_up(F))); }

struct Up {
  ae_lenc *m;
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
  float *f32(const std::vector<float> &h) { return f32(h.data(), h.size()); }
  // [rows][cols] bf16 and its tensor map (the GEMM's B operand: 64-wide k boxes of 128 rows)
  void *mat(const std::vector<float> &h, size_t rows, size_t cols, CUtensorMap *tm) {
    std::vector<uint16_t> b(h.size());
    for (size_t i = 0; i < h.size(); ++i) b[i] = to_bf16(h[i]);
    uint16_t *d = alloc<uint16_t>(b.size());
    if (d && cudaMemcpy(d, b.data(), b.size() * 2, cudaMemcpyHostToDevice) != cudaSuccess) ok = false;
    if (d && !make_tmap_2d_bf16(tm, d, (uint64_t)cols, (uint64_t)rows, (uint64_t)cols * 2, 64, 128)) ok = false;
    return d;
  }
  void *mat(const float *h, size_t rows, size_t cols, CUtensorMap *tm) {
    return mat(std::vector<float>(h, h + rows * cols), rows, cols, tm);
  }
};

bool cfg_ok(const ae_lenc_config *c, std::string *why) {
  auto bad = [&](const char *w) {
    *why = w;
    return false;
  };
  if (!c) return bad("cfg is null");
  if (c->n_mels != kLencMels) return bad("n_mels must be 128");
  if (c->n_embd != kLencEmbd || c->n_head != kLencHeads) return bad("n_embd must be 512 with 8 heads of 64");
  if (c->stem_ch != kLencStemCh) return bad("stem_ch must be 256");
  if (c->n_layers < 0 || c->n_layers > 64) return bad("n_layers must lie in [0, 64]");
  if (c->n_ff < 256 || c->n_ff % 256 || c->n_ff > 16384) return bad("n_ff must be a multiple of 256 up to 16384");
  if (c->adapter_ff < 256 || c->adapter_ff % 256 || c->adapter_ff > 16384)
    return bad("adapter_ff must be a multiple of 256 up to 16384");
  if (c->llm_hidden < 256 || c->llm_hidden % 256 || c->llm_hidden > 16384)
    return bad("llm_hidden must be a multiple of 256 up to 16384");
  if (c->conv_k < 1 || c->conv_k > kLencMaxConvK) return bad("conv_k must lie in [1, 33]");
  if (!std::isfinite(c->eps) || c->eps <= 0.f) return bad("eps must be positive");
  return true;
}

// Per-call tables: frame, stem-row, token and query-block offsets.
struct LencTables {
  int n_clips = 0;
  int64_t frames = 0, s2_rows = 0, tokens = 0, qblk = 0, s2_items = 0;
  int t_max = 0;
  std::vector<int32_t> frame_off, s2_off, tok_off, qblk_off, s2item_off;
};

// kind 0: frame offsets; kind 1: token offsets (the block call)
ae_status lenc_tables(const int64_t *off, int n, int kind, LencTables &T) {
  if (n < 0 || n > (1 << 20)) return lfail(AE_EINVAL, "n_clips must lie in [0, 1048576]");
  if (!off) return lfail(AE_EINVAL, "offsets are null");
  if (off[0] != 0) return lfail(AE_EINVAL, "offsets must start at 0");
  T = LencTables();
  T.n_clips = n;
  T.frame_off.assign(n + 1, 0);
  T.s2_off.assign(n + 1, 0);
  T.tok_off.assign(n + 1, 0);
  T.qblk_off.assign(n + 1, 0);
  T.s2item_off.assign(n + 1, 0);
  for (int c = 0; c < n; ++c) {
    const int64_t len = off[c + 1] - off[c];
    if (len < 0) return lfail(AE_EINVAL, "offsets are not non-decreasing at clip " + std::to_string(c));
    const int64_t F = kind == 0 ? len : 0;
    const int64_t t = kind == 0 ? stem_tokens(F) : len;
    if (t > kLencMaxTok)
      return lfail(AE_EUNSUPPORTED, "clip " + std::to_string(c) + " has more than 4096 rows after the stem");
    T.frames += F;
    T.s2_rows += half_up(half_up(F));
    T.s2_items += (half_up(half_up(F)) + kLencStemRun - 1) / kLencStemRun;
    T.tokens += t;
    T.qblk += (t + 127) / 128;
    if (T.frames > 64000000 || T.s2_rows > 4000000 || T.tokens > 2000000)
      return lfail(AE_EINVAL, "batch too large for one call");
    T.t_max = std::max<int>(T.t_max, (int)t);
    T.frame_off[c + 1] = (int32_t)T.frames;
    T.s2_off[c + 1] = (int32_t)T.s2_rows;
    T.tok_off[c + 1] = (int32_t)T.tokens;
    T.qblk_off[c + 1] = (int32_t)T.qblk;
    T.s2item_off[c + 1] = (int32_t)T.s2_items;
  }
  return AE_OK;
}

struct LencLayout {
  size_t tables, x, y2, y2b, y3, y3b, a, big, qkv, o, cbuf, pe, P, total;
};

LencLayout lenc_layout(const ae_lenc_config &c, const LencTables &T) {
  LencLayout L{};
  size_t off = 0;
  auto put = [&](size_t bytes) {
    const size_t o = off;
    off += al256(bytes);
    return o;
  };
  const size_t B1 = (size_t)T.n_clips + 1;
  L.tables = put(5 * B1 * 4);
  L.x = put((size_t)T.tokens * kLencEmbd * 4);
  const size_t u0 = off;  // the stem's buffers and the blocks' share this region
  L.y2 = put((size_t)T.s2_rows * 32 * kLencStemCh * 2);
  L.y2b = put((size_t)T.s2_rows * 32 * kLencStemCh * 2);
  L.y3 = put((size_t)T.tokens * 16 * kLencStemCh * 2);
  L.y3b = put((size_t)T.tokens * 16 * kLencStemCh * 2);
  const size_t stem_end = off;
  off = u0;
  const size_t wide = (size_t)std::max({c.n_ff, c.adapter_ff, 2 * kLencEmbd});
  L.a = put((size_t)T.tokens * kLencEmbd * 2);
  L.big = put((size_t)T.tokens * wide * 2);
  L.qkv = put((size_t)T.tokens * 3 * kLencEmbd * 2);
  L.o = put((size_t)T.tokens * kLencEmbd * 2);
  L.cbuf = put((size_t)T.tokens * kLencEmbd * 2);
  const size_t prow = T.t_max > 0 ? (size_t)(2 * T.t_max - 1) : 0;
  L.pe = put(prow * kLencEmbd * 2);
  L.P = put(prow * (size_t)std::max(c.n_layers, 1) * kLencEmbd * 2);
  L.total = std::max(off, stem_end) + 256;
  return L;
}

ae_status upload_tables(const LencTables &T, void *ws, const LencLayout &L, LencTablesDev *td, cudaStream_t s) {
  const size_t B1 = (size_t)T.n_clips + 1;
  std::vector<int32_t> h(5 * B1);
  std::copy(T.frame_off.begin(), T.frame_off.end(), h.begin());
  std::copy(T.s2_off.begin(), T.s2_off.end(), h.begin() + B1);
  std::copy(T.tok_off.begin(), T.tok_off.end(), h.begin() + 2 * B1);
  std::copy(T.qblk_off.begin(), T.qblk_off.end(), h.begin() + 3 * B1);
  std::copy(T.s2item_off.begin(), T.s2item_off.end(), h.begin() + 4 * B1);
  int32_t *d = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + L.tables);
  const cudaError_t e = profiled_f(AE_K_TABLES, 0.0, 0.0, s, [&] { return launch_upload_bytes(h.data(), h.size() * 4, d, s); });
  if (e != cudaSuccess) return lcuda(e, "clip tables");
  td->n_clips = T.n_clips;
  td->frame_off = d;
  td->s2_off = d + B1;
  td->tok_off = d + 2 * B1;
  td->qblk_off = d + 3 * B1;
  td->s2item_off = d + 4 * B1;
  return AE_OK;
}

EpiArgs epi(void *out, int64_t ld, const float *bias) {
  EpiArgs e;
  std::memset(&e, 0, sizeof(e));
  e.out = out;
  e.ld = ld;
  e.bias = bias;
  e.lo = -INFINITY;
  e.hi = INFINITY;
  e.lo2 = -INFINITY;
  e.hi2 = INFINITY;
  e.clamp2 = 0;
  e.alpha = 1.0f;
  return e;
}

#define LE_TRY(x)                     \
  do {                                \
    cudaError_t e_ = (x);             \
    if (e_ != cudaSuccess) return e_; \
  } while (0)

// one projection, timed as the encoder's GEMM class
cudaError_t proj(const void *x, int64_t M, int K, const CUtensorMap &tm, int N, int mode, const EpiArgs &ep,
                 cudaStream_t s) {
  const double fl = 2.0 * (double)M * N * K;
  const double by = 2.0 * ((double)M * K + (double)N * K) + (double)M * N * (mode == EPI_F32 ? 4 : 2);
  return profiled_f(AE_K_LENC_GEMM, fl, by, s, [&] { return gemm_bf16(x, M, K, tm, N, mode, ep, s); });
}

// x's rows through LayerNorm(w1, b1), written back to x if write_x; then the
// bf16 operand a of those rows, or of LayerNorm(w2, b2) of them when w2 is given
cudaError_t ln(float *x, int64_t rows, float eps, const float *w1, const float *b1, bool write_x, bf16 *a,
               cudaStream_t s, const float *w2 = nullptr, const float *b2 = nullptr) {
  LencLnArgs r;
  std::memset(&r, 0, sizeof(r));
  r.x = x;
  r.rows = rows;
  r.eps = eps;
  r.w1 = w1;
  r.b1 = b1;
  r.write_x = write_x ? 1 : 0;
  r.a = a;
  r.w2 = w2;
  r.b2 = b2;
  const double by = (double)rows * kLencEmbd * (4.0 + (write_x ? 4.0 : 0.0) + (a ? 2.0 : 0.0));
  return profiled_f(AE_K_LENC_ROW, 0.0, by, s, [&] { return launch_lenc_ln(r, s); });
}

struct Bufs {
  float *x;
  uint8_t *ws;
  LencLayout L;
  LencTablesDev td;
  const LencTables *T;
};

cudaError_t run_stem(const ae_lenc *m, const float *mel, const Bufs &b, cudaStream_t s) {
  const LencTables &T = *b.T;
  uint8_t *y2 = b.ws + b.L.y2, *y2b = b.ws + b.L.y2b, *y3 = b.ws + b.L.y3, *y3b = b.ws + b.L.y3b;
  const int C = kLencStemCh;
  LE_TRY(profiled_f(AE_K_LENC_ROW, 2.0 * 9 * 10 * C * 32.0 * T.s2_rows,
                    4.0 * T.frames * kLencMels + 2.0 * T.s2_rows * 32 * C, s,
                    [&] { return launch_lenc_stem01(mel, m->w0b, m->b0, m->w1, m->b1, y2, b.td, T.s2_items, s); }));
  EpiArgs e = epi(y2b, C, m->b2);
  e.lo = 0.f;  // ReLU
  LE_TRY(proj(y2, T.s2_rows * 32, C, m->tm_w2, C, EPI_BIAS_BF16, e, s));
  LE_TRY(profiled_f(AE_K_LENC_ROW, 2.0 * 9 * C * 16.0 * T.tokens, 2.0 * T.s2_rows * 32 * C + 2.0 * T.tokens * 16 * C,
                    s, [&] { return launch_lenc_dw2(y2b, m->w3, m->b3, y3, b.td, T.tokens, s); }));
  e = epi(y3b, C, m->b4);
  e.lo = 0.f;
  LE_TRY(proj(y3, T.tokens * 16, C, m->tm_w4, C, EPI_BIAS_BF16, e, s));
  return proj(y3b, T.tokens, 16 * C, m->tm_pre, kLencEmbd, EPI_F32, epi(b.x, kLencEmbd, m->pre_b), s);
}

// The position rows of every layer for this call's longest clip: the table
// [2 t_max - 1][512] and its projection through the stacked linear_pos.
cudaError_t run_positions(const ae_lenc *m, const Bufs &b, cudaStream_t s) {
  const int t_max = b.T->t_max;
  if (t_max <= 0 || m->cfg.n_layers == 0) return cudaSuccess;
  const int64_t rows = 2 * (int64_t)t_max - 1;
  LE_TRY(profiled_f(AE_K_LENC_ROW, 0.0, 2.0 * rows * kLencEmbd, s,
                    [&] { return launch_lenc_relpos(b.ws + b.L.pe, t_max, s); }));
  return proj(b.ws + b.L.pe, rows, kLencEmbd, m->tm_pos, m->cfg.n_layers * kLencEmbd, EPI_BF16,
              epi(b.ws + b.L.P, (int64_t)m->cfg.n_layers * kLencEmbd, nullptr), s);
}

// One block. With `first_ready` the operand of the first FFN's LayerNorm is
// already in a (the previous block's closing pass made it); with next_w the
// closing LayerNorm also makes the operand of the LayerNorm that follows (the
// next block's first, or the adapter's), in the same pass over the rows.
cudaError_t run_block(const ae_lenc *m, int li, const Bufs &b, cudaStream_t s, bool first_ready = false,
                      const float *next_w = nullptr, const float *next_b = nullptr) {
  const ae_lenc::Block &B = m->blocks[li];
  const LencTables &T = *b.T;
  const int64_t n = T.tokens;
  const int D = kLencEmbd, F = m->cfg.n_ff;
  const float eps = m->cfg.eps;
  bf16 *a = reinterpret_cast<bf16 *>(b.ws + b.L.a);
  void *big = b.ws + b.L.big, *qkv = b.ws + b.L.qkv, *o = b.ws + b.L.o, *cb = b.ws + b.L.cbuf;
  auto ffn = [&](const float *nw, const float *nb, const CUtensorMap &up, const float *ub, const CUtensorMap &down,
                 const float *db, bool ready) -> cudaError_t {
    if (!ready) LE_TRY(ln(b.x, n, eps, nw, nb, false, a, s));
    LE_TRY(proj(a, n, D, up, F, EPI_BIAS_SILU, epi(big, F, ub), s));
    EpiArgs e = epi(b.x, D, db);
    e.alpha = 0.5f;  // macaron half weight
    return proj(big, n, F, down, D, EPI_BIAS_ADD_F32, e, s);
  };
  LE_TRY(ffn(B.f1_nw, B.f1_nb, B.tm_f1_up, B.f1_ub, B.tm_f1_down, B.f1_db, first_ready));
  // attention
  LE_TRY(ln(b.x, n, eps, B.ln1_w, B.ln1_b, false, a, s));
  LE_TRY(proj(a, n, D, B.tm_qkv, 3 * D, EPI_BIAS_BF16, epi(qkv, 3 * D, B.qkv_b), s));
  {
    const int64_t prow = 2 * (int64_t)T.t_max - 1;
    double fl = 0.0;
    for (int c = 0; c < T.n_clips; ++c) {
      const double t = T.tok_off[c + 1] - T.tok_off[c];
      fl += 2.0 * 2.0 * t * t * D + 2.0 * t * t * D;  // two score terms and P V, one pass
    }
    LE_TRY(profiled_f(AE_K_LENC_ATTENTION, fl, 2.0 * n * 4 * D, s, [&] {
      return launch_lenc_xlattn(qkv, n, b.ws + b.L.P, prow, (int64_t)m->cfg.n_layers * D, li * D, B.bu, B.bv,
                                b.td.tok_off, b.td.qblk_off, T.n_clips, (int)T.qblk, T.t_max, o, s);
    }));
  }
  LE_TRY(proj(o, n, D, B.tm_o, D, EPI_BIAS_ADD_F32, epi(b.x, D, B.o_b), s));
  // conv module
  LE_TRY(ln(b.x, n, eps, B.nc_w, B.nc_b, false, a, s));
  LE_TRY(proj(a, n, D, B.tm_pw1, 2 * D, EPI_BIAS_GLU, epi(big, D, B.pw1_b), s));
  LE_TRY(profiled_f(AE_K_LENC_ROW, 2.0 * n * D * m->cfg.conv_k, 4.0 * n * D, s, [&] {
    return launch_lenc_dwconv(big, B.dw_w, B.dw_b, B.cn_w, B.cn_b, m->cfg.conv_k, cb, b.td.tok_off, T.n_clips, n, s);
  }));
  LE_TRY(proj(cb, n, D, B.tm_pw2, D, EPI_BIAS_ADD_F32, epi(b.x, D, B.pw2_b), s));
  LE_TRY(ffn(B.f2_nw, B.f2_nb, B.tm_f2_up, B.f2_ub, B.tm_f2_down, B.f2_db, false));
  return ln(b.x, n, eps, B.ln2_w, B.ln2_b, true, next_w ? a : nullptr, s, next_w, next_b);
}

cudaError_t run_adapter(const ae_lenc *m, const Bufs &b, float *out, cudaStream_t s, bool norm_ready = false) {
  const int64_t n = b.T->tokens;
  bf16 *a = reinterpret_cast<bf16 *>(b.ws + b.L.a);
  void *big = b.ws + b.L.big;
  if (!norm_ready) LE_TRY(ln(b.x, n, m->cfg.eps, m->ad_nw, m->ad_nb, false, a, s));
  LE_TRY(proj(a, n, kLencEmbd, m->tm_ad_up, m->cfg.adapter_ff, EPI_BIAS_GELU, epi(big, m->cfg.adapter_ff, m->ad_ub),
              s));
  return proj(big, n, m->cfg.adapter_ff, m->tm_ad_down, m->cfg.llm_hidden, EPI_F32,
              epi(out, m->cfg.llm_hidden, m->ad_db), s);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

ae_status prepare(const ae_lenc *m, const int64_t *off, int n_clips, int kind, void *d_ws, size_t ws_bytes,
                  LencTables &T, Bufs &b, cudaStream_t s) {
  if (!m) return lfail(AE_EINVAL, "model is null");
  if (ae_status st = lenc_tables(off, n_clips, kind, T)) return st;
  b.L = lenc_layout(m->cfg, T);
  b.T = &T;
  if (!d_ws) return lfail(AE_EINVAL, "d_ws is null");
  if (ws_bytes < b.L.total) return lfail(AE_EWORKSPACE, "ws_bytes below the workspace size");
  b.ws = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(d_ws) + 255) & ~uintptr_t(255));
  if ((size_t)(b.ws - static_cast<uint8_t *>(d_ws)) + b.L.total - 256 > ws_bytes)
    return lfail(AE_EWORKSPACE, "ws_bytes below the workspace size");
  b.x = reinterpret_cast<float *>(b.ws + b.L.x);
  return upload_tables(T, b.ws, b.L, &b.td, s);
}

}  // namespace
}  // namespace ae

using namespace ae;

extern "C" {

void ae_lenc_default_config(ae_lenc_config *c) {
  if (!c) return;
  c->n_mels = kLencMels;
  c->n_embd = kLencEmbd;
  c->n_head = kLencHeads;
  c->n_layers = 17;
  c->n_ff = 2048;
  c->conv_k = 9;
  c->stem_ch = kLencStemCh;
  c->adapter_ff = 2048;
  c->llm_hidden = 2048;
  c->eps = 1e-5f;
}

int64_t ae_lenc_num_tokens(int64_t n_frames) { return stem_tokens(n_frames); }

void ae_lenc_destroy(ae_lenc *m) {
  if (!m) return;
  for (void *p : m->allocs) cudaFree(p);
  delete m;
}

ae_status ae_lenc_create(const ae_lenc_config *cfg, const ae_lenc_host_weights *w, ae_lenc **out) {
  if (!out) return lfail(AE_EINVAL, "out is null");
  *out = nullptr;
  std::string why;
  if (!cfg_ok(cfg, &why)) return lfail(cfg ? AE_EUNSUPPORTED : AE_EINVAL, why);
  if (!w) return lfail(AE_EINVAL, "weights are null");
  for (int i = 0; i < 5; ++i)
    if (!w->stem_w[i] || !w->stem_b[i]) return lfail(AE_EINVAL, "stem layer " + std::to_string(i) + " is null");
  if (!w->pre_w || !w->pre_b || !w->ad_norm_w || !w->ad_norm_b || !w->ad_up_w || !w->ad_up_b || !w->ad_down_w ||
      !w->ad_down_b)
    return lfail(AE_EINVAL, "pre_encode_out or adapter weights are null");
  if (cfg->n_layers > 0 && !w->blocks) return lfail(AE_EINVAL, "blocks are null");
  const int L = cfg->n_layers, D = kLencEmbd, F = cfg->n_ff, C = kLencStemCh, K = cfg->conv_k;
  for (int l = 0; l < L; ++l) {
    const ae_lenc_host_block &h = w->blocks[l];
    const float *const *p = &h.ffn1_norm_w;
    for (size_t i = 0; i < sizeof(ae_lenc_host_block) / sizeof(float *); ++i)
      if (!p[i]) return lfail(AE_EINVAL, "block " + std::to_string(l) + " has a null weight");
  }
  ae_lenc *m = new ae_lenc();
  m->cfg = *cfg;
  Up up{m};
  {
    // channel c's row of 64 bf16: (w_hi, w_lo, w_hi) of its 9 taps, zeros after, against
    // the patch row (p_hi, p_hi, p_lo): p_hi w_hi + p_hi w_lo + p_lo w_hi, about 16 bits
    std::vector<uint16_t> wb((size_t)C * 64, 0);
    for (int c = 0; c < C; ++c)
      for (int k = 0; k < 9; ++k) {
        const float v = w->stem_w[0][(size_t)c * 9 + k];
        const uint16_t hi = to_bf16(v);
        wb[(size_t)c * 64 + k] = hi;
        wb[(size_t)c * 64 + 9 + k] = to_bf16(v - from_bf16(hi));
        wb[(size_t)c * 64 + 18 + k] = hi;
      }
    uint16_t *d = up.alloc<uint16_t>(wb.size());
    if (d && cudaMemcpy(d, wb.data(), wb.size() * 2, cudaMemcpyHostToDevice) != cudaSuccess) up.ok = false;
    m->w0b = d;
  }
  m->b0 = up.f32(w->stem_b[0], C);
  m->w1 = up.f32(w->stem_w[1], (size_t)C * 9);
  m->b1 = up.f32(w->stem_b[1], C);
  m->w2 = up.mat(w->stem_w[2], C, C, &m->tm_w2);
  m->b2 = up.f32(w->stem_b[2], C);
  m->w3 = up.f32(w->stem_w[3], (size_t)C * 9);
  m->b3 = up.f32(w->stem_b[3], C);
  m->w4 = up.mat(w->stem_w[4], C, C, &m->tm_w4);
  m->b4 = up.f32(w->stem_b[4], C);
  {
    // pre_encode_out: the page's column c * 16 + f to this layout's f * C + c
    const int FQ = kLencMels / 8;
    std::vector<float> pp((size_t)D * FQ * C);
    for (int r = 0; r < D; ++r)
      for (int c = 0; c < C; ++c)
        for (int f = 0; f < FQ; ++f) pp[(size_t)r * FQ * C + f * C + c] = w->pre_w[(size_t)r * FQ * C + c * FQ + f];
    m->pre_w = up.mat(pp, D, (size_t)FQ * C, &m->tm_pre);
  }
  m->pre_b = up.f32(w->pre_b, D);
  m->blocks.resize(L);
  std::vector<float> pos((size_t)std::max(L, 1) * D * D, 0.f);
  for (int l = 0; l < L; ++l) {
    const ae_lenc_host_block &h = w->blocks[l];
    ae_lenc::Block &B = m->blocks[l];
    B.f1_nw = up.f32(h.ffn1_norm_w, D);
    B.f1_nb = up.f32(h.ffn1_norm_b, D);
    B.f1_up = up.mat(h.ffn1_up_w, F, D, &B.tm_f1_up);
    B.f1_ub = up.f32(h.ffn1_up_b, F);
    B.f1_down = up.mat(h.ffn1_down_w, D, F, &B.tm_f1_down);
    B.f1_db = up.f32(h.ffn1_down_b, D);
    B.ln1_w = up.f32(h.ln1_w, D);
    B.ln1_b = up.f32(h.ln1_b, D);
    {
      std::vector<float> qkv((size_t)3 * D * D), qb((size_t)3 * D);
      std::copy(h.q_w, h.q_w + (size_t)D * D, qkv.begin());
      std::copy(h.k_w, h.k_w + (size_t)D * D, qkv.begin() + (size_t)D * D);
      std::copy(h.v_w, h.v_w + (size_t)D * D, qkv.begin() + (size_t)2 * D * D);
      std::copy(h.q_b, h.q_b + D, qb.begin());
      std::copy(h.k_b, h.k_b + D, qb.begin() + D);
      std::copy(h.v_b, h.v_b + D, qb.begin() + 2 * D);
      B.qkv = up.mat(qkv, 3 * D, D, &B.tm_qkv);
      B.qkv_b = up.f32(qb);
    }
    B.o = up.mat(h.o_w, D, D, &B.tm_o);
    B.o_b = up.f32(h.o_b, D);
    std::copy(h.linear_pos_w, h.linear_pos_w + (size_t)D * D, pos.begin() + (size_t)l * D * D);
    B.bu = up.f32(h.pos_bias_u, D);
    B.bv = up.f32(h.pos_bias_v, D);
    B.nc_w = up.f32(h.norm_conv_w, D);
    B.nc_b = up.f32(h.norm_conv_b, D);
    {
      // pw1 rows interleaved (a_c, b_c): the GLU epilogue sees both halves of channel c together
      std::vector<float> pw((size_t)2 * D * D), pb((size_t)2 * D);
      for (int c = 0; c < D; ++c) {
        std::copy(h.pw1_w + (size_t)c * D, h.pw1_w + (size_t)(c + 1) * D, pw.begin() + (size_t)(2 * c) * D);
        std::copy(h.pw1_w + (size_t)(D + c) * D, h.pw1_w + (size_t)(D + c + 1) * D, pw.begin() + (size_t)(2 * c + 1) * D);
        pb[2 * c] = h.pw1_b[c];
        pb[2 * c + 1] = h.pw1_b[D + c];
      }
      B.pw1 = up.mat(pw, 2 * D, D, &B.tm_pw1);
      B.pw1_b = up.f32(pb);
    }
    B.dw_w = up.f32(h.dw_w, (size_t)K * D);
    B.dw_b = up.f32(h.dw_b, D);
    B.cn_w = up.f32(h.conv_norm_w, D);
    B.cn_b = up.f32(h.conv_norm_b, D);
    B.pw2 = up.mat(h.pw2_w, D, D, &B.tm_pw2);
    B.pw2_b = up.f32(h.pw2_b, D);
    B.f2_nw = up.f32(h.ffn2_norm_w, D);
    B.f2_nb = up.f32(h.ffn2_norm_b, D);
    B.f2_up = up.mat(h.ffn2_up_w, F, D, &B.tm_f2_up);
    B.f2_ub = up.f32(h.ffn2_up_b, F);
    B.f2_down = up.mat(h.ffn2_down_w, D, F, &B.tm_f2_down);
    B.f2_db = up.f32(h.ffn2_down_b, D);
    B.ln2_w = up.f32(h.ln2_w, D);
    B.ln2_b = up.f32(h.ln2_b, D);
  }
  m->pos_w = up.mat(pos, (size_t)std::max(L, 1) * D, D, &m->tm_pos);
  m->ad_nw = up.f32(w->ad_norm_w, D);
  m->ad_nb = up.f32(w->ad_norm_b, D);
  m->ad_up = up.mat(w->ad_up_w, cfg->adapter_ff, D, &m->tm_ad_up);
  m->ad_ub = up.f32(w->ad_up_b, cfg->adapter_ff);
  m->ad_down = up.mat(w->ad_down_w, cfg->llm_hidden, cfg->adapter_ff, &m->tm_ad_down);
  m->ad_db = up.f32(w->ad_down_b, cfg->llm_hidden);
  if (!up.ok) {
    ae_lenc_destroy(m);
    return lfail(AE_ENOMEM, "device memory for the encoder could not be allocated or filled");
  }
  *out = m;
  return AE_OK;
}

size_t ae_lenc_workspace_size(const ae_lenc *m, const int64_t *h_frame_off, int n_clips) {
  LencTables T;
  if (!m || lenc_tables(h_frame_off, n_clips, 0, T) != AE_OK) return 0;
  return lenc_layout(m->cfg, T).total + 256;
}

size_t ae_lenc_block_workspace_size(const ae_lenc *m, const int64_t *h_tok_off, int n_clips) {
  LencTables T;
  if (!m || lenc_tables(h_tok_off, n_clips, 1, T) != AE_OK) return 0;
  return lenc_layout(m->cfg, T).total + 256;
}

ae_status ae_lenc_stem(const ae_lenc *m, const float *d_mel, const int64_t *h_frame_off, int n_clips, float *d_x,
                       void *d_ws, size_t ws_bytes, ae_stream stream) {
  LencTables T;
  Bufs b;
  if (ae_status st = prepare(m, h_frame_off, n_clips, 0, d_ws, ws_bytes, T, b, (cudaStream_t)stream)) return st;
  if (T.tokens > 0 && (!d_mel || !d_x)) return lfail(AE_EINVAL, "d_mel or d_x is null");
  if (T.tokens > 0 && !aligned16(d_x)) return lfail(AE_EINVAL, "d_x must be 16-byte aligned");
  if (T.tokens == 0) return AE_OK;
  Bufs bb = b;
  bb.x = d_x;
  const cudaError_t e = run_stem(m, d_mel, bb, (cudaStream_t)stream);
  return e == cudaSuccess ? AE_OK : lcuda(e, "ae_lenc_stem");
}

ae_status ae_lenc_block(const ae_lenc *m, int layer, float *d_x, const int64_t *h_tok_off, int n_clips, void *d_ws,
                        size_t ws_bytes, ae_stream stream) {
  if (!m) return lfail(AE_EINVAL, "model is null");
  if (layer < 0 || layer >= m->cfg.n_layers) return lfail(AE_EINVAL, "layer out of range");
  LencTables T;
  Bufs b;
  if (ae_status st = prepare(m, h_tok_off, n_clips, 1, d_ws, ws_bytes, T, b, (cudaStream_t)stream)) return st;
  if (T.tokens > 0 && (!d_x || !aligned16(d_x))) return lfail(AE_EINVAL, "d_x is null or not 16-byte aligned");
  if (T.tokens == 0) return AE_OK;
  b.x = d_x;
  cudaError_t e = run_positions(m, b, (cudaStream_t)stream);
  if (e == cudaSuccess) e = run_block(m, layer, b, (cudaStream_t)stream);
  return e == cudaSuccess ? AE_OK : lcuda(e, "ae_lenc_block");
}

ae_status ae_lenc_encode(const ae_lenc *m, const float *d_mel, const int64_t *h_frame_off, int n_clips, float *d_out,
                         void *d_ws, size_t ws_bytes, ae_stream stream) {
  LencTables T;
  Bufs b;
  if (ae_status st = prepare(m, h_frame_off, n_clips, 0, d_ws, ws_bytes, T, b, (cudaStream_t)stream)) return st;
  if (T.tokens > 0 && (!d_mel || !d_out)) return lfail(AE_EINVAL, "d_mel or d_out is null");
  if (T.tokens > 0 && !aligned16(d_out)) return lfail(AE_EINVAL, "d_out must be 16-byte aligned");
  if (T.tokens == 0) return AE_OK;
  const cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = run_stem(m, d_mel, b, s);
  if (e == cudaSuccess) e = run_positions(m, b, s);
  const int L = m->cfg.n_layers;
  for (int l = 0; l < L && e == cudaSuccess; ++l) {
    const bool last = l + 1 == L;
    e = run_block(m, l, b, s, l > 0, last ? m->ad_nw : m->blocks[l + 1].f1_nw,
                  last ? m->ad_nb : m->blocks[l + 1].f1_nb);
  }
  if (e == cudaSuccess) e = run_adapter(m, b, d_out, s, L > 0);
  return e == cudaSuccess ? AE_OK : lcuda(e, "ae_lenc_encode");
}

}  // extern "C"
