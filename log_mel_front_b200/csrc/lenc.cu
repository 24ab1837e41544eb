// Row and convolution kernels of the LFM2A Conformer encoder (cera 0.5.3,
// audio_encoder_gpu.rs: conv_stem_gpu with STEM_LAYER_MODES and
// STEM_RELU_AFTER, the layernorm, chan_affine_silu and conv2d ops of the
// block, and the relative-position table of relative_pos_emb). The
// projections run on the tensor-core GEMM (gemm.cu) and the attention in
// lenc_attention.cu.
//
// Stem layout: channels-last rows [time][freq][C] in bf16, clip after clip.
// k_lenc_stem01 computes the first two convolutions in one pass: the
// depthwise 3x3 stride-2 conv of ReLU(3x3 stride-2 conv of the mel + bias),
// evaluating the first convolution's outputs where the second reads them
// (its zero padding is the second's input padding); the pointwise 1x1
// convolutions are GEMMs over the positions (bias, ReLU); k_lenc_dw2 is the
// second depthwise conv. The last pointwise GEMM's output [T][16][C] is the
// flattened [T][16 C] input of pre_encode_out, whose columns are permuted at
// model creation from the page's channel-major flatten.
#include "ae_internal.h"
#include "common.cuh"

namespace ae {

// Clip of a packed row index, by binary search over a prefix array [B+1].
__device__ __forceinline__ int lenc_clip_of(const int32_t *off, int n_clips, int64_t r) {
  int lo = 0, hi = n_clips;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (off[mid] <= r) lo = mid; else hi = mid;
  }
  return lo;
}

// ------------------------------------------------------------------ stem: conv0 + ReLU + depthwise conv1

// One CTA per output row (t2 of one clip): [32 freq][C] outputs. Thread t
// owns channels 2t, 2t+1 (C = 2 x blockDim). The seven mel rows the row
// reads (4 t2 - 3 .. 4 t2 + 3) are staged in shared memory with a zero band
// on the left. Walking f2, the thread keeps the first convolution's column
// f1 = 2 f2 - 1 from the previous step and evaluates the columns 2 f2 and
// 2 f2 + 1 for the three time rows t1 = 2 t2 - 1 .. 2 t2 + 1.
__global__ void __launch_bounds__(128) k_lenc_stem01(const float *__restrict__ mel, const float *__restrict__ w0,
                                                     const float *__restrict__ b0, const float *__restrict__ w1,
                                                     const float *__restrict__ b1, bf16 *__restrict__ y2,
                                                     const LencTablesDev t) {
  constexpr int MP = kLencMels + 1;  // one zero column in front (mel column -1)
  __shared__ float s_mel[7][MP];
  const int64_t row = blockIdx.x;
  const int c = lenc_clip_of(t.s2_off, t.n_clips, row);
  const int t2 = (int)(row - t.s2_off[c]);
  const int F = t.frame_off[c + 1] - t.frame_off[c];
  const int T1 = (F + 1) / 2;
  const float *m = mel + (int64_t)t.frame_off[c] * kLencMels;
  for (int i = threadIdx.x; i < 7 * MP; i += blockDim.x) {
    const int rr = i / MP, cc = i % MP, fr = 4 * t2 - 3 + rr, col = cc - 1;
    s_mel[rr][cc] = (fr >= 0 && fr < F && col >= 0) ? __ldg(m + (int64_t)fr * kLencMels + col) : 0.f;
  }
  const int ch = 2 * threadIdx.x;
  float2 wa[9], wb[9], ba, bb;
#pragma unroll
  for (int k = 0; k < 9; ++k) {
    wa[k] = make_float2(__ldg(w0 + ch * 9 + k), __ldg(w0 + (ch + 1) * 9 + k));
    wb[k] = make_float2(__ldg(w1 + ch * 9 + k), __ldg(w1 + (ch + 1) * 9 + k));
  }
  ba = make_float2(__ldg(b0 + ch), __ldg(b0 + ch + 1));
  bb = make_float2(__ldg(b1 + ch), __ldg(b1 + ch + 1));
  __syncthreads();
  bool tv[3];  // first-convolution rows t1 = 2 t2 - 1 + k inside the clip
#pragma unroll
  for (int k = 0; k < 3; ++k) tv[k] = (2 * t2 - 1 + k) >= 0 && (2 * t2 - 1 + k) < T1;
  float2 prev[3];  // column f1 = 2 f2 - 1 (the zero padding at f2 = 0)
#pragma unroll
  for (int k = 0; k < 3; ++k) prev[k] = make_float2(0.f, 0.f);
  bf16 *out = y2 + row * (int64_t)(32 * kLencStemCh) + ch;
#pragma unroll 1
  for (int f2 = 0; f2 < 32; ++f2) {
    // mel columns 4 f2 - 1 .. 4 f2 + 3 (staged at +1) of the seven rows: column
    // f1 = 2 f2 + jj reads 4 f2 + 2 jj + df - 1
    float mv[7][5];
#pragma unroll
    for (int rr = 0; rr < 7; ++rr)
#pragma unroll
      for (int j = 0; j < 5; ++j) mv[rr][j] = s_mel[rr][4 * f2 + j];
    float2 cur[2][3];  // columns f1 = 2 f2 (j = 0) and 2 f2 + 1 (j = 1)
#pragma unroll
    for (int jj = 0; jj < 2; ++jj)
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        float2 a = ba;
#pragma unroll
        for (int dt = 0; dt < 3; ++dt)
#pragma unroll
          for (int df = 0; df < 3; ++df) {
            const float v = mv[2 * k + dt][2 * jj + df];
            ffma2(a, wa[dt * 3 + df], make_float2(v, v));
          }
        cur[jj][k] = tv[k] ? make_float2(fmaxf(a.x, 0.f), fmaxf(a.y, 0.f)) : make_float2(0.f, 0.f);
      }
    float2 o = bb;
#pragma unroll
    for (int dt = 0; dt < 3; ++dt) {
      ffma2(o, wb[dt * 3 + 0], prev[dt]);
      ffma2(o, wb[dt * 3 + 1], cur[0][dt]);
      ffma2(o, wb[dt * 3 + 2], cur[1][dt]);
    }
#pragma unroll
    for (int k = 0; k < 3; ++k) prev[k] = cur[1][k];
    *reinterpret_cast<uint32_t *>(out + f2 * kLencStemCh) = pack_bf16(o.x, o.y);
  }
}

// ------------------------------------------------------------------ stem: depthwise conv3

// One CTA per output row (t3 of one clip): [16 freq][C] from the rows
// 2 t3 - 1 .. 2 t3 + 1 of [T2][32][C] (zero outside the clip and at f = -1).
__global__ void __launch_bounds__(128) k_lenc_dw2(const bf16 *__restrict__ y, const float *__restrict__ w,
                                                  const float *__restrict__ b, bf16 *__restrict__ out,
                                                  const LencTablesDev t) {
  const int64_t row = blockIdx.x;
  const int c = lenc_clip_of(t.tok_off, t.n_clips, row);
  const int t3 = (int)(row - t.tok_off[c]);
  const int T2 = t.s2_off[c + 1] - t.s2_off[c];
  const int ch = 2 * threadIdx.x;
  float2 wk[9];
#pragma unroll
  for (int k = 0; k < 9; ++k) wk[k] = make_float2(__ldg(w + ch * 9 + k), __ldg(w + (ch + 1) * 9 + k));
  const float2 bias = make_float2(__ldg(b + ch), __ldg(b + ch + 1));
  const bf16 *src = y + (int64_t)t.s2_off[c] * (32 * kLencStemCh) + ch;
#pragma unroll 1
  for (int f3 = 0; f3 < 16; ++f3) {
    float2 a = bias;
#pragma unroll
    for (int dt = 0; dt < 3; ++dt) {
      const int tr = 2 * t3 + dt - 1;
      if (tr < 0 || tr >= T2) continue;
#pragma unroll
      for (int df = 0; df < 3; ++df) {
        const int fr = 2 * f3 + df - 1;
        if (fr < 0) continue;
        const uint32_t v = *reinterpret_cast<const uint32_t *>(src + ((int64_t)tr * 32 + fr) * kLencStemCh);
        ffma2(a, wk[dt * 3 + df], make_float2(bf16lo(v), bf16hi(v)));
      }
    }
    *reinterpret_cast<uint32_t *>(out + (row * 16 + f3) * (int64_t)kLencStemCh + ch) = pack_bf16(a.x, a.y);
  }
}

// ------------------------------------------------------------------ LayerNorm rows

// One warp per row of 512: lane l holds columns (32 i + l) * 4 .. +3, i < 4.
// y = (x - mean) / sqrt(var + eps) * w1 + b1 (biased variance, two passes over
// the registers); optionally written back to x; then the bf16 operand a =
// y, or LN(y; w2, b2) when w2 is given.
__global__ void __launch_bounds__(256) k_lenc_ln(const LencLnArgs r) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= r.rows) return;
  float *xr = r.x + row * kLencEmbd;
  float v[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) load4(xr + (i * 32 + lane) * 4, v[i]);
  auto norm = [&](const float *w, const float *b) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int u = 0; u < 4; ++u) s += v[i][u];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mean = s * (1.0f / kLencEmbd);
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        v[i][u] -= mean;
        q = fmaf(v[i][u], v[i][u], q);
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    const float inv = rsqrtf(q * (1.0f / kLencEmbd) + r.eps);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float wv[4], bv[4];
      load4(w + (i * 32 + lane) * 4, wv);
      load4(b + (i * 32 + lane) * 4, bv);
#pragma unroll
      for (int u = 0; u < 4; ++u) v[i][u] = fmaf(v[i][u] * inv, wv[u], bv[u]);
    }
  };
  norm(r.w1, r.b1);
  if (r.write_x) {
#pragma unroll
    for (int i = 0; i < 4; ++i) store4(xr + (i * 32 + lane) * 4, v[i]);
  }
  if (r.a) {
    if (r.w2) norm(r.w2, r.b2);
    bf16 *ar = r.a + row * kLencEmbd;
#pragma unroll
    for (int i = 0; i < 4; ++i) store4(ar + (i * 32 + lane) * 4, v[i]);
  }
}

// ------------------------------------------------------------------ conv module: depthwise conv + affine + SiLU

// The conv module's middle (the page's conv2d with groups = channels, then
// chan_affine_silu): y[t][c] = silu((db[c] + sum_m w[m][c] g[t + m - lo][c])
// * aw[c] + ab[c]), lo = (k - 1) / 2, taps outside the clip skipped. A CTA
// stages kDwRows rows plus the k - 1 halo rows of all 512 channels in shared
// memory (bf16) and each thread computes two channels of every row.
constexpr int kDwRows = 32;

// KT > 0: the tap count known at compile time (the taps of the thread's two
// channels in registers); KT = 0: any k <= 33, taps read per use.
template <int KT>
__global__ void __launch_bounds__(256) k_lenc_dwconv(const bf16 *__restrict__ g, const float *__restrict__ w,
                                                     const float *__restrict__ db, const float *__restrict__ aw,
                                                     const float *__restrict__ ab, int k_rt, bf16 *__restrict__ out,
                                                     const int32_t *__restrict__ tok_off, int n_clips, int64_t T) {
  extern __shared__ __align__(16) uint32_t s_g[];  // [kDwRows + k - 1][256] bf16 pairs
  const int k = KT > 0 ? KT : k_rt;
  const int lo = (k - 1) / 2;
  const int64_t t0 = (int64_t)blockIdx.x * kDwRows;
  const int nrows = kDwRows + k - 1;
  for (int i = threadIdx.x; i < nrows * 256; i += 256) {
    const int rr = i >> 8, cp = i & 255;
    const int64_t tr = t0 - lo + rr;
    s_g[i] = (tr >= 0 && tr < T) ? *reinterpret_cast<const uint32_t *>(g + tr * kLencEmbd + 2 * cp) : 0u;
  }
  const int ch = 2 * threadIdx.x;
  float2 wr[KT > 0 ? KT : 1];
  if (KT > 0) {
#pragma unroll
    for (int m = 0; m < (KT > 0 ? KT : 1); ++m) wr[m] = make_float2(__ldg(w + m * kLencEmbd + ch), __ldg(w + m * kLencEmbd + ch + 1));
  }
  __syncthreads();
  const float2 bias = make_float2(db[ch], db[ch + 1]), sc = make_float2(aw[ch], aw[ch + 1]),
               sh = make_float2(ab[ch], ab[ch + 1]);
  int c = lenc_clip_of(tok_off, n_clips, t0 < T ? t0 : T - 1);
#pragma unroll 1
  for (int r = 0; r < kDwRows; ++r) {
    const int64_t tt = t0 + r;
    if (tt >= T) break;
    while (tok_off[c + 1] <= tt) ++c;  // rows are in order; clips may be empty
    const int64_t s0 = tok_off[c], e = tok_off[c + 1];
    const int m0 = (int)max((int64_t)0, s0 - (tt - lo)), m1 = (int)min((int64_t)k, e - (tt - lo));
    float2 a = bias;
    if (KT > 0) {
#pragma unroll
      for (int m = 0; m < (KT > 0 ? KT : 1); ++m)
        if (m >= m0 && m < m1) {
          const uint32_t v = s_g[(r + m) * 256 + threadIdx.x];
          ffma2(a, wr[m], make_float2(bf16lo(v), bf16hi(v)));
        }
    } else {
      for (int m = m0; m < m1; ++m) {
        const uint32_t v = s_g[(r + m) * 256 + threadIdx.x];
        ffma2(a, make_float2(__ldg(w + m * kLencEmbd + ch), __ldg(w + m * kLencEmbd + ch + 1)),
              make_float2(bf16lo(v), bf16hi(v)));
      }
    }
    const float2 y = __ffma2_rn(a, sc, sh);
    const float2 z = make_float2(y.x / (1.0f + __expf(-y.x)), y.y / (1.0f + __expf(-y.y)));
    *reinterpret_cast<uint32_t *>(out + tt * kLencEmbd + ch) = pack_bf16(z.x, z.y);
  }
}

// ------------------------------------------------------------------ relative-position table

// Row r of [2 t_max - 1][D]: relative position p = t_max - 1 - r; columns
// 2i and 2i + 1 hold sin(p w_i) and cos(p w_i), w_i = 10000^(-2i / D), in
// float64, stored as bf16 (the operand of the position projection).
__global__ void k_lenc_relpos(bf16 *__restrict__ pe, int t_max, int D) {
  const int64_t n = (int64_t)(2 * t_max - 1) * (D / 2);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int r = (int)(i / (D / 2)), j = (int)(i % (D / 2));
    const double p = (double)(t_max - 1 - r);
    const double w = exp(-(double)(2 * j) * (9.210340371976184 / (double)D));  // ln(10000) = 9.2103...
    double sn, cs;
    sincos(p * w, &sn, &cs);
    *reinterpret_cast<uint32_t *>(pe + (int64_t)r * D + 2 * j) = pack_bf16((float)sn, (float)cs);
  }
}

// ------------------------------------------------------------------ launchers

cudaError_t launch_lenc_stem01(const float *mel, const float *w0, const float *b0, const float *w1, const float *b1,
                               void *y2, const LencTablesDev &t, int64_t s2_rows, cudaStream_t s) {
  if (s2_rows <= 0) return cudaSuccess;
  return launch_k(k_lenc_stem01, dim3((unsigned)s2_rows), dim3(kLencStemCh / 2), 0, s, mel, w0, b0, w1, b1,
                  static_cast<bf16 *>(y2), t);
}

cudaError_t launch_lenc_dw2(const void *y, const float *w, const float *b, void *out, const LencTablesDev &t,
                            int64_t tokens, cudaStream_t s) {
  if (tokens <= 0) return cudaSuccess;
  return launch_k(k_lenc_dw2, dim3((unsigned)tokens), dim3(kLencStemCh / 2), 0, s, static_cast<const bf16 *>(y), w, b,
                  static_cast<bf16 *>(out), t);
}

cudaError_t launch_lenc_ln(const LencLnArgs &r, cudaStream_t s) {
  if (r.rows <= 0) return cudaSuccess;
  return launch_k(k_lenc_ln, dim3((unsigned)((r.rows + 7) / 8)), dim3(256), 0, s, r);
}

cudaError_t launch_lenc_dwconv(const void *g, const float *w, const float *db, const float *aw, const float *ab, int k,
                               void *out, const int32_t *tok_off, int n_clips, int64_t T, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const size_t smem = (size_t)(kDwRows + k - 1) * 256 * 4;
  static std::atomic<uint64_t> attr9{0}, attr0{0};
  auto kern = k == 9 ? k_lenc_dwconv<9> : k_lenc_dwconv<0>;
  if (const cudaError_t e = smem_attr(kern, smem, k == 9 ? attr9 : attr0)) return e;
  return launch_k(kern, dim3((unsigned)((T + kDwRows - 1) / kDwRows)), dim3(256), smem, s,
                  static_cast<const bf16 *>(g), w, db, aw, ab, k, static_cast<bf16 *>(out), tok_off, n_clips, T);
}

cudaError_t launch_lenc_relpos(void *pe, int t_max, cudaStream_t s) {
  if (t_max <= 0) return cudaSuccess;
  const int64_t n = (int64_t)(2 * t_max - 1) * (kLencEmbd / 2);
  const unsigned grid = (unsigned)std::min<int64_t>((n + 255) / 256, 4096);
  return launch_k(k_lenc_relpos, dim3(grid), dim3(256), 0, s, static_cast<bf16 *>(pe), t_max, kLencEmbd);
}

}  // namespace ae
