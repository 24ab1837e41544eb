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

// w_dw is stored tap-major [kernel][hidden]. Persistent CTAs of 256 threads;
// the work item is a tile of kLcRows consecutive rows. The rows a tile reads
// (its own and the kKernel - 1 before them) are contiguous in memory, so one
// bulk copy brings them into shared memory; each CTA keeps two tiles in
// flight (double buffer, one mbarrier per buffer) and issues the copy of the
// tile after next as soon as every thread has read the current buffer.
// Thread t owns channels 4t .. 4t+3: its 5 x 4 taps and 4 norm weights stay
// in registers as channel pairs for the packed two-lane FMA, and it adds each
// buffered row into the (up to five) outputs that use it as the row arrives,
// so no window of rows is held in registers. The per-row sums of squares are
// reduced across the warp with a butterfly that halves the rows at every step
// (after it, lanes 4r .. 4r+3 hold row r), then across the CTA's 8 warps once
// for all rows; SiLU runs on the packed two-lane pipe.
constexpr int kLcRows = 8;
constexpr int kLcHalo = kKernel - 1;

template <typename ActT>
__host__ __device__ constexpr int lc_buf_bytes() {
  return (kLcRows + kLcHalo) * kHidden * (int)sizeof(ActT);
}

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void lds4(const float *p, float2 (&v)[2]) {
  const float4 t = *reinterpret_cast<const float4 *>(p);
  v[0] = make_float2(t.x, t.y);
  v[1] = make_float2(t.z, t.w);
}
__device__ __forceinline__ void lds4(const bf16 *p, float2 (&v)[2]) {
  const uint2 t = *reinterpret_cast<const uint2 *>(p);
  v[0] = make_float2(bf16lo(t.x), bf16hi(t.x));
  v[1] = make_float2(bf16lo(t.y), bf16hi(t.y));
}

template <typename ActT>
__global__ void __launch_bounds__(256, 3) k_lconv(const ActT *__restrict__ gl, const float *__restrict__ w_dw,
                                               const float *__restrict__ w_norm, float lo, float hi,
                                               ActT *__restrict__ out, const int32_t *__restrict__ pos, int64_t T,
                                               int64_t n_tiles, unsigned *status) {
  static_assert(kLcRows == 8, "the butterfly below reduces 8 rows");
  constexpr int kBuf = lc_buf_bytes<ActT>();
  constexpr int kRowBytes = kHidden * (int)sizeof(ActT);
  extern __shared__ __align__(128) uint8_t lc_smem[];
  __shared__ uint64_t bar[2];
  __shared__ float s_ss[8][kLcRows];
  __shared__ float s_inv[kLcRows];
  __shared__ int s_pos[2][kLcRows];  // positions of the buffered tiles' rows in their clips
  const int ch = 4 * threadIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
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
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  const int64_t my = (int64_t)blockIdx.x < n_tiles ? (n_tiles - 1 - (int64_t)blockIdx.x) / gridDim.x + 1 : 0;
  // row r of item k: its position, read by thread r two items ahead so that
  // no item waits on a global load
  auto pos_of = [&](int64_t k, int r) {
    const int64_t tok = ((int64_t)blockIdx.x + k * gridDim.x) * kLcRows + r;
    return k < my && tok < T ? pos[tok] : 0;
  };
  if (threadIdx.x < kLcRows) {
    s_pos[0][threadIdx.x] = pos_of(0, threadIdx.x);
    s_pos[1][threadIdx.x] = pos_of(1, threadIdx.x);
  }
  __syncthreads();
  // buffer row i of item k holds token t0 - kLcHalo + i; tokens before 0 or from T on are not copied
  auto issue = [&](int64_t k) {
    const int64_t t0 = ((int64_t)blockIdx.x + k * gridDim.x) * kLcRows;
    const int64_t a = t0 - kLcHalo > 0 ? t0 - kLcHalo : 0, b = t0 + kLcRows < T ? t0 + kLcRows : T;
    const uint32_t bytes = (uint32_t)((b - a) * kRowBytes);
    mbar_arrive_expect_tx(&bar[k & 1], bytes);
    bulk_load(lc_smem + (k & 1) * kBuf + (a - (t0 - kLcHalo)) * kRowBytes, gl + a * kHidden, bytes, &bar[k & 1]);
  };
  if (threadIdx.x == 0) {
    if (my > 0) issue(0);
    if (my > 1) issue(1);
  }
  for (int64_t k = 0; k < my; ++k) {
    const int64_t t0 = ((int64_t)blockIdx.x + k * gridDim.x) * kLcRows;
    const int pn = threadIdx.x < kLcRows ? pos_of(k + 2, threadIdx.x) : 0;  // stored at the end of this item
    if (!__syncthreads_and(mbar_wait(&bar[k & 1], (uint32_t)((k >> 1) & 1)))) {
      if (threadIdx.x == 0) atomicOr(status, kStatusWaitTimeout);
      break;
    }
    int p[kLcRows];  // position of each row in its clip (taps never reach before the clip start)
#pragma unroll
    for (int r = 0; r < kLcRows; ++r) p[r] = s_pos[k & 1][r];
    const ActT *sx = reinterpret_cast<const ActT *>(lc_smem + (k & 1) * kBuf) + ch;
    float2 c[kLcRows][2];
#pragma unroll
    for (int r = 0; r < kLcRows; ++r) c[r][0] = c[r][1] = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kLcRows + kLcHalo; ++i) {  // buffer row i feeds outputs r = i - 4 .. i with tap i - r
      float2 x[2];
      lds4(sx + i * kHidden, x);
#pragma unroll
      for (int r = (i - kLcHalo > 0 ? i - kLcHalo : 0); r <= (i < kLcRows - 1 ? i : kLcRows - 1); ++r) {
        if (r + kLcHalo - i <= p[r]) {
          ffma2(c[r][0], w[i - r][0], x[0]);
          ffma2(c[r][1], w[i - r][1], x[1]);
        }
      }
    }
    float ss[kLcRows];
#pragma unroll
    for (int r = 0; r < kLcRows; ++r) {
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
    __syncthreads();  // sums in; every thread is done with this buffer
    if (threadIdx.x == 0 && k + 2 < my) issue(k + 2);
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
    if (threadIdx.x < kLcRows) s_pos[k & 1][threadIdx.x] = pn;  // every thread read this item's after two barriers
  }
}

cudaError_t launch_lconv(const ae_model *m, const void *gl, const float *w_dw, const float *w_norm, float lo,
                         float hi, void *out, const int32_t *pos, int64_t T, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  if ((reinterpret_cast<uintptr_t>(gl) & 15) != 0) return cudaErrorMisalignedAddress;  // bulk copies
  const int64_t tiles = (T + kLcRows - 1) / kLcRows;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // resident CTAs per SM: three by registers; the float32 form's buffers allow two
  const int64_t slots = (m->dtype != AE_F32 ? 3 : 2) * (int64_t)sms;
  const unsigned grid = (unsigned)(tiles < slots ? tiles : slots);
  if (m->dtype != AE_F32) {
    static std::atomic<uint64_t> attr{0};
    constexpr size_t smem = 2 * lc_buf_bytes<bf16>();
    if (const cudaError_t e = smem_attr(k_lconv<bf16>, smem, attr)) return e;
    return launch_k(k_lconv<bf16>, dim3(grid), dim3(256), smem, s, static_cast<const bf16 *>(gl), w_dw, w_norm, lo,
                    hi, static_cast<bf16 *>(out), pos, T, tiles, device_status_word());
  }
  static std::atomic<uint64_t> attr{0};
  constexpr size_t smem = 2 * lc_buf_bytes<float>();
  if (const cudaError_t e = smem_attr(k_lconv<float>, smem, attr)) return e;
  return launch_k(k_lconv<float>, dim3(grid), dim3(256), smem, s, static_cast<const float *>(gl), w_dw, w_norm, lo,
                  hi, static_cast<float *>(out), pos, T, tiles, device_status_word());
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
