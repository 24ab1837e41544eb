// Row-wise kernels of the Conformer layer and the head, and the per-call
// table upload.
//
// k_rowop fuses, per row of the float32 residual stream, the page's
// add_normed (h += s * rms_w(y)), the plain residual add of the light conv,
// the layer's closing rms(norm_out), and the next projection's input:
// a = clamp(rms(h) * w, lo, hi) in the GEMM operand type. One warp owns a
// row; each lane holds width/32 values in registers, so h is read and
// written once per call.
//
// k_lconv is the light-conv middle (dwconv, glu already applied by the
// lc_start epilogue): the causal depthwise conv over 5 rows that does not
// reach before the clip start (AudioTower::dwconv), the conv_norm RMS norm,
// SiLU (norm_silu) and lc_end's input clamp.
#include "ae_internal.h"
#include "common.cuh"

#include <cstring>

namespace ae {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr float kEps = 1e-6f;

// NV = width / 128: lane l holds columns (i * 32 + l) * 4 .. +3, i < NV.
template <int NV, typename ActT>
__global__ void __launch_bounds__(256) k_rowop(const RowArgs r) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= r.rows) return;
  constexpr int W = NV * 128;
  float *hrow = r.h + row * W;
  float h[NV][4];
#pragma unroll
  for (int i = 0; i < NV; ++i) load4(hrow + (i * 32 + lane) * 4, h[i]);
  bool changed = false;
  if (r.y) {
    const float *yrow = r.y + row * W;
    float y[NV][4];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      load4(yrow + (i * 32 + lane) * 4, y[i]);
#pragma unroll
      for (int u = 0; u < 4; ++u) ss = fmaf(y[i][u], y[i][u], ss);
    }
    float sc = r.s;
    if (r.y_norm) sc *= rsqrtf(warp_sum(ss) * (1.0f / W) + kEps);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      float w[4] = {1.f, 1.f, 1.f, 1.f};
      if (r.y_norm && r.wy) load4(r.wy + (i * 32 + lane) * 4, w);
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
      load4(r.w_out + (i * 32 + lane) * 4, w);
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
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      float w[4] = {1.f, 1.f, 1.f, 1.f};
      if (r.w_next) load4(r.w_next + (i * 32 + lane) * 4, w);
      float a[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) a[u] = clampf(h[i][u] * inv * w[u], r.lo, r.hi);
      store4(arow + (i * 32 + lane) * 4, a);
    }
  }
}

template <typename ActT>
static cudaError_t rowop_width(const RowArgs &r, cudaStream_t s) {
  const unsigned grid = (unsigned)((r.rows + 7) / 8);
  switch (r.width) {
    case 1024: k_rowop<8, ActT><<<grid, 256, 0, s>>>(r); break;
    case 1536: k_rowop<12, ActT><<<grid, 256, 0, s>>>(r); break;
    case 2048: k_rowop<16, ActT><<<grid, 256, 0, s>>>(r); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_rowop(const ae_model *m, const RowArgs &r, cudaStream_t s) {
  if (r.rows <= 0) return cudaSuccess;
  return m->dtype == AE_BF16 ? rowop_width<bf16>(r, s) : rowop_width<float>(r, s);
}

// ------------------------------------------------------------------ light conv middle

// w_dw is stored tap-major [kernel][hidden] (20 KB, read through L1). A CTA
// owns kLcRows consecutive rows: it stages those rows plus the 4 before them
// in shared memory with coalesced 16-byte loads; each warp then computes
// kLcRows / 8 rows, lane l owning channels (i * 32 + l) * 4 .. +3.
constexpr int kLcRows = 16;
constexpr int kLcHalo = kKernel - 1;

template <typename ActT>
__global__ void __launch_bounds__(256) k_lconv(const ActT *__restrict__ gl, const float *__restrict__ w_dw,
                                               const float *__restrict__ w_norm, float lo, float hi,
                                               ActT *__restrict__ out, const int32_t *__restrict__ pos, int64_t T) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const float *s_w = w_dw;
  ActT *s_x = reinterpret_cast<ActT *>(smem_raw);                        // [kLcRows + halo][hidden]
  const int lane = threadIdx.x & 31;
  const int64_t t0 = (int64_t)blockIdx.x * kLcRows;
  constexpr int VEC = 16 / sizeof(ActT);                                 // elements per 16-byte load
  constexpr int ROW_V = kHidden / VEC;
  for (int i = threadIdx.x; i < (kLcRows + kLcHalo) * ROW_V; i += blockDim.x) {
    const int r = i / ROW_V, cv = i % ROW_V;
    const int64_t tok = t0 - kLcHalo + r;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (tok >= 0 && tok < T) v = __ldg(reinterpret_cast<const uint4 *>(gl + tok * kHidden) + cv);
    reinterpret_cast<uint4 *>(s_x + (int64_t)r * kHidden)[cv] = v;
  }
  __syncthreads();
  constexpr int NV = kHidden / 128;
  for (int rr = 0; rr < kLcRows / 8; ++rr) {
    const int lr = (threadIdx.x >> 5) * (kLcRows / 8) + rr;  // local output row
    const int64_t t = t0 + lr;
    if (t >= T) return;
    const int p = pos[t];
    float c[NV][4];
#pragma unroll
    for (int i = 0; i < NV; ++i)
#pragma unroll
      for (int u = 0; u < 4; ++u) c[i][u] = 0.f;
#pragma unroll
    for (int k = 0; k < kKernel; ++k) {
      const int back = kKernel - 1 - k;
      if (back > p) continue;
      const ActT *src = s_x + (int64_t)(lr + kLcHalo - back) * kHidden;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        float x[4], w[4];
        load4(src + (i * 32 + lane) * 4, x);
        load4(s_w + k * kHidden + (i * 32 + lane) * 4, w);
#pragma unroll
        for (int u = 0; u < 4; ++u) c[i][u] = fmaf(w[u], x[u], c[i][u]);
      }
    }
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i)
#pragma unroll
      for (int u = 0; u < 4; ++u) ss = fmaf(c[i][u], c[i][u], ss);
    const float inv = rsqrtf(warp_sum(ss) * (1.0f / kHidden) + kEps);
    ActT *orow = out + t * kHidden;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      float w[4], v[4];
      load4(w_norm + (i * 32 + lane) * 4, w);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float y = c[i][u] * inv * w[u];
        v[u] = clampf(y / (1.0f + __expf(-y)), lo, hi);
      }
      store4(orow + (i * 32 + lane) * 4, v);
    }
  }
}

cudaError_t launch_lconv(const ae_model *m, const void *gl, const float *w_dw, const float *w_norm, float lo,
                         float hi, void *out, const int32_t *pos, int64_t T, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const unsigned grid = (unsigned)((T + kLcRows - 1) / kLcRows);
  const size_t base = (size_t)(kLcRows + kLcHalo) * kHidden;
  if (m->dtype == AE_BF16) {
    const size_t smem = base * 2;
    static bool attr = false;
    if (!attr) {
      cudaError_t e = cudaFuncSetAttribute(k_lconv<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      attr = true;
    }
    k_lconv<bf16><<<grid, 256, smem, s>>>(static_cast<const bf16 *>(gl), w_dw, w_norm, lo, hi,
                                          static_cast<bf16 *>(out), pos, T);
  } else {
    const size_t smem = base * 4;
    static bool attr = false;
    if (!attr) {
      cudaError_t e = cudaFuncSetAttribute(k_lconv<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      attr = true;
    }
    k_lconv<float><<<grid, 256, smem, s>>>(static_cast<const float *>(gl), w_dw, w_norm, lo, hi,
                                           static_cast<float *>(out), pos, T);
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------------ tables

// The per-call tables travel as kernel parameters (copied at launch, so the
// call never waits on the host and stays capturable).
struct UploadChunk {
  int64_t dst;  // byte offset in the workspace
  int n;        // 32-bit words
  uint32_t w[7936];
};

__global__ void k_upload(uint8_t *base, const UploadChunk ch) {
  uint32_t *d = reinterpret_cast<uint32_t *>(base + ch.dst);
  for (int i = threadIdx.x; i < ch.n; i += blockDim.x) d[i] = ch.w[i];
}

__global__ void k_pos(int32_t *pos, const int32_t *tok_off) {
  const int c = blockIdx.x;
  const int b = tok_off[c], n = tok_off[c + 1] - b;
  for (int i = threadIdx.x; i < n; i += blockDim.x) pos[b + i] = i;
}

cudaError_t launch_pos(int32_t *pos, const int32_t *tok_off, int n_clips, cudaStream_t s) {
  if (n_clips <= 0) return cudaSuccess;
  k_pos<<<n_clips, 256, 0, s>>>(pos, tok_off);
  return cudaGetLastError();
}

static size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

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
  const size_t nw = off / 4;
  static thread_local UploadChunk ch;
  for (size_t w0 = 0; w0 < nw; w0 += 7936) {
    const size_t n = nw - w0 < 7936 ? nw - w0 : 7936;
    ch.dst = (int64_t)(w0 * 4);
    ch.n = (int)n;
    std::memcpy(ch.w, words.data() + w0, n * 4);
    k_upload<<<1, 256, 0, s>>>(base, ch);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
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
