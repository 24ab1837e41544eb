// Row-wise kernels of the Conformer layer and the head, and the per-call
// table upload.
//
// k_rowop fuses, per row of the float32 residual stream, the page's
// add_normed (h += s * rms_w(y)), the plain residual add of the light conv,
// the layer's closing rms(norm_out), and the next projection's input:
// a = clamp(rms(h) * w, lo, hi) in the GEMM operand type, or as e4m3 codes of
// a * q for the e4m3 projections (q = 448 over the clamp's larger bound). One
// warp owns a row; each lane holds width/32 values in registers, so h is read
// and written once per call.
//
// k_lconv is the light-conv middle (dwconv, glu already applied by the
// lc_start epilogue): the causal depthwise conv over 5 rows that does not
// reach before the clip start (AudioTower::dwconv), the conv_norm RMS norm,
// SiLU (norm_silu) and lc_end's input clamp.
#include "ae_internal.h"
#include "common.cuh"

#include <algorithm>
#include <cstring>

namespace ae {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr float kEps = 1e-6f;

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// NV = width / 128: lane l holds columns (i * 32 + l) * 4 .. +3, i < NV. The
// row's h and y are loaded first; the weight vectors are staged in shared
// memory while those loads are in flight, so a row costs one memory round
// trip.
template <int NV, typename ActT>
__global__ void __launch_bounds__(256, NV <= 8 ? 3 : 2) k_rowop(const RowArgs r) {
  constexpr int W = NV * 128;
  __shared__ __align__(16) float s_wy[W], s_wo[W], s_wn[W];
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const bool live = row < r.rows;
  for (int i = threadIdx.x; i < W / 4; i += blockDim.x) {  // the norm weights this pass uses
    if (r.wy) reinterpret_cast<float4 *>(s_wy)[i] = __ldg(reinterpret_cast<const float4 *>(r.wy) + i);
    if (r.w_out) reinterpret_cast<float4 *>(s_wo)[i] = __ldg(reinterpret_cast<const float4 *>(r.w_out) + i);
    if (r.w_next) reinterpret_cast<float4 *>(s_wn)[i] = __ldg(reinterpret_cast<const float4 *>(r.w_next) + i);
  }
  float *hrow = r.h + (live ? row : 0) * W;
  float h[NV][4], y[NV][4];
  if (live) {
#pragma unroll
    for (int i = 0; i < NV; ++i) load4(hrow + (i * 32 + lane) * 4, h[i]);
    if (r.y) {
#pragma unroll
      for (int i = 0; i < NV; ++i) load4(static_cast<const ActT *>(r.y) + row * W + (i * 32 + lane) * 4, y[i]);
    }
  }
  __syncthreads();
  if (!live) return;
  bool changed = false;
  if (r.y) {
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i)
#pragma unroll
      for (int u = 0; u < 4; ++u) ss = fmaf(y[i][u], y[i][u], ss);
    float sc = r.s;
    if (r.y_norm) sc *= rsqrtf(warp_sum(ss) * (1.0f / W) + kEps);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      float w[4] = {1.f, 1.f, 1.f, 1.f};
      if (r.y_norm && r.wy) load4(s_wy + (i * 32 + lane) * 4, w);
#pragma unroll
      for (int u = 0; u < 4; ++u) h[i][u] = fmaf(sc * w[u], y[i][u], h[i][u]);
    }
    changed = true;
  }
  if (r.w_out) {
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i)
#pragma unroll
      for (int u = 0; u < 4; ++u) ss = fmaf(h[i][u], h[i][u], ss);
    const float inv = rsqrtf(warp_sum(ss) * (1.0f / W) + kEps);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      float w[4];
      load4(s_wo + (i * 32 + lane) * 4, w);
#pragma unroll
      for (int u = 0; u < 4; ++u) h[i][u] = h[i][u] * inv * w[u];
    }
    changed = true;
  }
  if (changed) {
#pragma unroll
    for (int i = 0; i < NV; ++i) store4(hrow + (i * 32 + lane) * 4, h[i]);
  }
  if (r.a_out) {
    float inv = 1.f;
    if (r.a_rms) {
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < NV; ++i)
#pragma unroll
        for (int u = 0; u < 4; ++u) ss = fmaf(h[i][u], h[i][u], ss);
      inv = rsqrtf(warp_sum(ss) * (1.0f / W) + kEps);
    }
    ActT *arow = static_cast<ActT *>(r.a_out) + row * W;
    uint32_t *qrow = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(r.a_out) + row * W);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      float w[4] = {1.f, 1.f, 1.f, 1.f};
      if (r.w_next) load4(s_wn + (i * 32 + lane) * 4, w);
      float a[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) a[u] = clampf(h[i][u] * inv * w[u], r.lo, r.hi);
      if (r.a_q8 > 0.f)  // e4m3 operand: 4 codes per lane, 128 contiguous bytes per warp
        qrow[i * 32 + lane] = pack_e4m3x4(a[0] * r.a_q8, a[1] * r.a_q8, a[2] * r.a_q8, a[3] * r.a_q8);
      else
        store4(arow + (i * 32 + lane) * 4, a);
    }
  }
}

template <typename ActT>
static cudaError_t rowop_width(const RowArgs &r, cudaStream_t s) {
  const unsigned grid = (unsigned)((r.rows + 7) / 8);
  switch (r.width) {
    case 1024: return launch_k(k_rowop<8, ActT>, dim3(grid), dim3(256), 0, s, r);
    case 1536: return launch_k(k_rowop<12, ActT>, dim3(grid), dim3(256), 0, s, r);
    case 2048: return launch_k(k_rowop<16, ActT>, dim3(grid), dim3(256), 0, s, r);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_rowop(const ae_model *m, const RowArgs &r, cudaStream_t s) {
  if (r.rows <= 0) return cudaSuccess;
  return m->dtype == AE_F32 ? rowop_width<float>(r, s) : rowop_width<bf16>(r, s);
}

// ------------------------------------------------------------------ light conv middle

// w_dw is stored tap-major [kernel][hidden]. Thread t of a 256-thread CTA
// owns channels 4t .. 4t+3 for kLcRows consecutive rows: its 5 x 4 taps and
// 4 norm weights stay in registers, as channel pairs for the packed two-lane
// FMA, and it loads its 8-byte slice of the rows (plus the 4 before them),
// one coalesced load per row. The conv outputs of its rows stay in registers;
// SiLU runs on the packed two-lane pipe.
// The per-row sums of squares are reduced across the warp with a butterfly
// that halves the rows at every step (after it, lanes 4r .. 4r+3 hold row r),
// then across the CTA's 8 warps once for all rows.
constexpr int kLcRows = 8;
constexpr int kLcHalo = kKernel - 1;

// Four CTAs per SM (64 registers): on the ragged batch 1.49 ms per step against about
// 1.60 ms at three (a few bytes of spill in the bf16 form); the tower's short launches
// lose about 4 %.
template <typename ActT>
__global__ void __launch_bounds__(256, 4) k_lconv(const ActT *__restrict__ gl, const float *__restrict__ w_dw,
                                               const float *__restrict__ w_norm, float lo, float hi,
                                               ActT *__restrict__ out, const int32_t *__restrict__ pos, int64_t T) {
  static_assert(kLcRows == 8, "the butterfly below reduces 8 rows");
  __shared__ float s_ss[8][kLcRows];
  __shared__ float s_inv[kLcRows];
  const int ch = 4 * threadIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t t0 = (int64_t)blockIdx.x * kLcRows;
  float2 w[kKernel][2], wn[2];
#pragma unroll
  for (int k = 0; k < kKernel; ++k) {
    float t[4];
    load4(w_dw + k * kHidden + ch, t);
    w[k][0] = make_float2(t[0], t[1]);
    w[k][1] = make_float2(t[2], t[3]);
  }
  {
    float t[4];
    load4(w_norm + ch, t);
    wn[0] = make_float2(t[0], t[1]);
    wn[1] = make_float2(t[2], t[3]);
  }
  float2 x[kLcRows + kLcHalo][2];
#pragma unroll
  for (int r = 0; r < kLcRows + kLcHalo; ++r) {
    const int64_t tok = t0 - kLcHalo + r;
    float t[4] = {0.f, 0.f, 0.f, 0.f};
    if (tok >= 0 && tok < T) load4(gl + tok * kHidden + ch, t);
    x[r][0] = make_float2(t[0], t[1]);
    x[r][1] = make_float2(t[2], t[3]);
  }
  float2 c[kLcRows][2];
  float ss[kLcRows];
#pragma unroll
  for (int r = 0; r < kLcRows; ++r) {
    const int64_t tok = t0 + r;
    const int p = tok < T ? pos[tok] : 0;
    c[r][0] = c[r][1] = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kKernel; ++k) {
      const int back = kKernel - 1 - k;
      if (back <= p) {
        ffma2(c[r][0], w[k][0], x[r + kLcHalo - back][0]);
        ffma2(c[r][1], w[k][1], x[r + kLcHalo - back][1]);
      }
    }
    float2 q = make_float2(0.f, 0.f);
    ffma2(q, c[r][0], c[r][0]);
    ffma2(q, c[r][1], c[r][1]);
    ss[r] = q.x + q.y;
  }
  // butterfly reduce-scatter: 8 rows -> 4 -> 2 -> 1 per lane, then a sum over the 4 lanes
  {
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
    float v4[4], v2[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float mine = b4 ? ss[i + 4] : ss[i], other = b4 ? ss[i] : ss[i + 4];
      v4[i] = mine + __shfl_xor_sync(0xffffffffu, other, 16);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float mine = b3 ? v4[i + 2] : v4[i], other = b3 ? v4[i] : v4[i + 2];
      v2[i] = mine + __shfl_xor_sync(0xffffffffu, other, 8);
    }
    float v = (b2 ? v2[1] : v2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? v2[0] : v2[1], 4);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    if ((lane & 3) == 0) s_ss[warp][lane >> 2] = v;  // row (lane >> 2): bits 4, 3, 2 of the lane
  }
  __syncthreads();
  if (threadIdx.x < kLcRows) {
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) sum += s_ss[q][threadIdx.x];
    s_inv[threadIdx.x] = rsqrtf(sum * (1.0f / kHidden) + kEps);
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kLcRows; ++r) {
    const int64_t tok = t0 + r;
    if (tok >= T) break;
    const float2 inv = make_float2(s_inv[r], s_inv[r]);
    float v[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // silu(y) = y / (1 + 2^(-y log2 e)), two channels per packed op
      const float2 y = __fmul2_rn(c[r][h], __fmul2_rn(inv, wn[h]));
      const float2 e = __fmul2_rn(y, make_float2(-1.4426950408889634f, -1.4426950408889634f));
      const float2 d = __fadd2_rn(make_float2(ex2_approx(e.x), ex2_approx(e.y)), make_float2(1.0f, 1.0f));
      const float2 sl = __fmul2_rn(y, make_float2(rcp_approx(d.x), rcp_approx(d.y)));
      v[2 * h] = clampf(sl.x, lo, hi);
      v[2 * h + 1] = clampf(sl.y, lo, hi);
    }
    store4(out + tok * kHidden + ch, v);
  }
}

cudaError_t launch_lconv(const ae_model *m, const void *gl, const float *w_dw, const float *w_norm, float lo,
                         float hi, void *out, const int32_t *pos, int64_t T, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const unsigned grid = (unsigned)((T + kLcRows - 1) / kLcRows);
  if (m->dtype != AE_F32)
    return launch_k(k_lconv<bf16>, dim3(grid), dim3(256), 0, s, static_cast<const bf16 *>(gl), w_dw, w_norm, lo, hi,
                    static_cast<bf16 *>(out), pos, T);
  return launch_k(k_lconv<float>, dim3(grid), dim3(256), 0, s, static_cast<const float *>(gl), w_dw, w_norm, lo, hi,
                  static_cast<float *>(out), pos, T);
}

// ------------------------------------------------------------------ tables

// The per-call tables travel as kernel parameters (copied at launch, so the
// call never waits on the host and stays capturable).
template <int W>
struct UploadChunk {
  int64_t dst;  // byte offset in the workspace
  int n;        // 32-bit words
  uint32_t w[W];
};

template <int W>
__global__ void k_upload(uint8_t *base, const UploadChunk<W> ch) {
  uint32_t *d = reinterpret_cast<uint32_t *>(base + ch.dst);
  for (int i = threadIdx.x; i < ch.n; i += blockDim.x) d[i] = ch.w[i];
}

// Copies nw words from the host to dev in chunks of at most 7936 words, each in
// the smallest parameter block that holds it (a launch copies its whole
// parameter block, so a few tables do not pay for 31 KB).
template <int W>
static cudaError_t upload_chunk(const uint32_t *src, size_t n, uint8_t *dst, cudaStream_t s) {
  static thread_local UploadChunk<W> ch;
  ch.dst = 0;
  ch.n = (int)n;
  std::memcpy(ch.w, src, n * 4);
  return launch_k(k_upload<W>, dim3(1), dim3(256), 0, s, dst, ch);
}

static cudaError_t upload_words(const uint32_t *src, size_t nw, uint8_t *dst, cudaStream_t s) {
  for (size_t w0 = 0; w0 < nw; w0 += 7936) {
    const size_t n = nw - w0 < 7936 ? nw - w0 : 7936;
    const cudaError_t e = n <= 512    ? upload_chunk<512>(src + w0, n, dst + 4 * w0, s)
                          : n <= 2048 ? upload_chunk<2048>(src + w0, n, dst + 4 * w0, s)
                                      : upload_chunk<7936>(src + w0, n, dst + 4 * w0, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

__global__ void k_pos(int32_t *pos, const int32_t *tok_off) {
  const int c = blockIdx.x;
  const int b = tok_off[c], n = tok_off[c + 1] - b;
  for (int i = threadIdx.x; i < n; i += blockDim.x) pos[b + i] = i;
}

cudaError_t launch_pos(int32_t *pos, const int32_t *tok_off, int n_clips, cudaStream_t s) {
  if (n_clips <= 0) return cudaSuccess;
  return launch_k(k_pos, dim3(n_clips), dim3(256), 0, s, pos, tok_off);
}

static size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

cudaError_t launch_upload_bytes(const void *host, size_t bytes, void *dev, cudaStream_t s) {
  std::vector<uint32_t> words((bytes + 3) / 4, 0u);
  std::memcpy(words.data(), host, bytes);
  return upload_words(words.data(), words.size(), static_cast<uint8_t *>(dev), s);
}

size_t tables_bytes(int64_t n_clips) {
  const size_t B1 = (size_t)n_clips + 1;
  return al256(B1 * 8) + 5 * al256(B1 * 4);
}

cudaError_t launch_upload_tables(const ClipTables &t, void *ws, const WsLayout &L, ClipTablesDev *dev,
                                 bool with_pos, cudaStream_t s) {
  const size_t B1 = (size_t)t.n_clips + 1;
  // layout inside the tables region: sample_off (int64), then five int32 arrays
  std::vector<uint32_t> words;
  words.resize(tables_bytes(t.n_clips) / 4, 0u);
  uint8_t *hb = reinterpret_cast<uint8_t *>(words.data());
  size_t off = 0;
  auto put = [&](const void *src, size_t bytes) {
    std::memcpy(hb + off, src, bytes);
    const size_t o = off;
    off += al256(bytes);
    return o;
  };
  const size_t o_s = put(t.sample_off.data(), B1 * 8);
  const size_t o_f = put(t.frame_off.data(), B1 * 4);
  const size_t o_t = put(t.tok_off.data(), B1 * 4);
  const size_t o_st = put(t.stem_off.data(), B1 * 4);
  const size_t o_mt = put(t.mel_tile_off.data(), B1 * 4);
  const size_t o_ct = put(t.conv1_tile_off.data(), B1 * 4);
  uint8_t *base = static_cast<uint8_t *>(ws) + L.tables;
  if (const cudaError_t e = upload_words(words.data(), off / 4, base, s)) return e;
  dev->n_clips = t.n_clips;
  dev->sample_off = reinterpret_cast<const int64_t *>(base + o_s);
  dev->frame_off = reinterpret_cast<const int32_t *>(base + o_f);
  dev->tok_off = reinterpret_cast<const int32_t *>(base + o_t);
  dev->stem_off = reinterpret_cast<const int32_t *>(base + o_st);
  dev->mel_tile_off = reinterpret_cast<const int32_t *>(base + o_mt);
  dev->conv1_tile_off = reinterpret_cast<const int32_t *>(base + o_ct);
  int32_t *pos = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + L.pos);
  dev->pos = pos;
  if (with_pos && t.total_tokens > 0) return launch_pos(pos, dev->tok_off, t.n_clips, s);
  return cudaSuccess;
}

}  // namespace ae
