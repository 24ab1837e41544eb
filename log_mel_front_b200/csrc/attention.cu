// Chunked local attention core (egemma2_audio.rs, AudioTower::attention):
// per head, token t attends to itself and the 11 tokens before it within its
// clip; logits z_d = (q s) . (k_scale k_{t-d}) + (q s) . R[d] with
// s = log2(e)/sqrt(128) * softplus(per_dim_scale), capped as
// cap * tanh(z / cap); natural-exp softmax over the distances; o_t =
// sum_d p_d v_{t-d}.
//
// A CTA owns one head and 128 consecutive tokens. It stages that head's
// k and v rows for the tokens and the 11-row halo before them in shared
// memory (coalesced 16-byte loads; rows padded so lanes reading
// consecutive rows hit distinct banks) plus the head's R[0..11] and the
// per-dim scales. Each thread then owns one query: the 12 dot products run
// over 16-dimension chunks held in registers, the softmax over the 12
// logits is private to the thread, and the weighted sum of v is written
// back chunk by chunk, clamped to the post projection's input bounds. No
// cross-thread reduction is needed.
#include "ae_internal.h"
#include "common.cuh"

namespace ae {

namespace {
constexpr int kTQ = 128;                 // queries per CTA
constexpr int kRows = kTQ + kLeft - 1;   // staged k/v rows
}  // namespace

template <typename T> struct AttnIO;
template <> struct AttnIO<bf16> {
  static constexpr int kPitch = kHeadDim + 8;  // elements per staged row (272 bytes)
  static constexpr int kChunks = kHeadDim * 2 / 16;
  // 16 consecutive values at p (32-byte aligned) as float
  static __device__ __forceinline__ void load16(const bf16 *p, float (&v)[16]) {
    const uint4 a = reinterpret_cast<const uint4 *>(p)[0], b = reinterpret_cast<const uint4 *>(p)[1];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = bf16lo(w[i]);
      v[2 * i + 1] = bf16hi(w[i]);
    }
  }
  static __device__ __forceinline__ void store16(bf16 *p, const float (&v)[16]) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = pack_bf16(v[2 * i], v[2 * i + 1]);
    reinterpret_cast<uint4 *>(p)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4 *>(p)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
};
template <> struct AttnIO<float> {
  static constexpr int kPitch = kHeadDim + 4;  // 528 bytes
  static constexpr int kChunks = kHeadDim * 4 / 16;
  static __device__ __forceinline__ void load16(const float *p, float (&v)[16]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 x = reinterpret_cast<const float4 *>(p)[i];
      v[4 * i] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
    }
  }
  static __device__ __forceinline__ void store16(float *p, const float (&v)[16]) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      reinterpret_cast<float4 *>(p)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
};

template <typename T>
__global__ void __launch_bounds__(kTQ) k_attention(const T *__restrict__ q, const T *__restrict__ k,
                                                   const T *__restrict__ v, int64_t ld, const float *__restrict__ R,
                                                   const float *__restrict__ qscale, float k_scale, float cap,
                                                   const int32_t *__restrict__ pos, int64_t T_total,
                                                   T *__restrict__ out, int64_t ld_out, float lo, float hi) {
  using IO = AttnIO<T>;
  extern __shared__ uint8_t smem_raw[];
  T *Ks = reinterpret_cast<T *>(smem_raw);
  T *Vs = Ks + kRows * IO::kPitch;
  float *Rs = reinterpret_cast<float *>(Vs + kRows * IO::kPitch);  // [12][128]
  float *Qs = Rs + kLeft * kHeadDim;                                // [128]

  const int h = blockIdx.y;
  const int64_t t0 = (int64_t)blockIdx.x * kTQ;
  const int tid = threadIdx.x;

  // ---- stage k, v rows t0-11 .. t0+127 of head h (zero outside [0, T))
  for (int idx = tid; idx < kRows * IO::kChunks; idx += kTQ) {
    const int r = idx / IO::kChunks, ch = idx % IO::kChunks;
    const int64_t tok = t0 - (kLeft - 1) + r;
    uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
    if (tok >= 0 && tok < T_total) {
      kv = *reinterpret_cast<const uint4 *>(k + tok * ld + h * kHeadDim + ch * (16 / sizeof(T)));
      vv = *reinterpret_cast<const uint4 *>(v + tok * ld + h * kHeadDim + ch * (16 / sizeof(T)));
    }
    *reinterpret_cast<uint4 *>(Ks + r * IO::kPitch + ch * (16 / sizeof(T))) = kv;
    *reinterpret_cast<uint4 *>(Vs + r * IO::kPitch + ch * (16 / sizeof(T))) = vv;
  }
  for (int i = tid; i < kLeft * kHeadDim; i += kTQ) Rs[i] = R[(i / kHeadDim) * kHidden + h * kHeadDim + i % kHeadDim];
  Qs[tid] = qscale[tid];
  __syncthreads();

  const int64_t t = t0 + tid;
  if (t >= T_total) return;
  const int span = min(pos[t] + 1, kLeft);
  const T *qrow = q + t * ld + h * kHeadDim;

  float d1[kLeft], d2[kLeft];
#pragma unroll
  for (int d = 0; d < kLeft; ++d) d1[d] = d2[d] = 0.f;
#pragma unroll 1
  for (int c = 0; c < kHeadDim / 16; ++c) {
    float qv[16];
    IO::load16(qrow + c * 16, qv);
#pragma unroll
    for (int i = 0; i < 16; ++i) qv[i] *= Qs[c * 16 + i];
#pragma unroll
    for (int d = 0; d < kLeft; ++d) {
      float kk[16];
      IO::load16(Ks + (tid + kLeft - 1 - d) * IO::kPitch + c * 16, kk);
      const float *rr = Rs + d * kHeadDim + c * 16;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        d1[d] = fmaf(qv[i], kk[i], d1[d]);
        d2[d] = fmaf(qv[i], rr[i], d2[d]);
      }
    }
  }
  // ---- capped logits, softmax over the distances inside the clip
  float p[kLeft];
  float mx = -INFINITY;
#pragma unroll
  for (int d = 0; d < kLeft; ++d) {
    const float z = cap * tanhf(fmaf(k_scale, d1[d], d2[d]) / cap);
    p[d] = (d < span) ? z : -INFINITY;
    mx = fmaxf(mx, p[d]);
  }
  float den = 0.f;
#pragma unroll
  for (int d = 0; d < kLeft; ++d) {
    p[d] = (d < span) ? expf(p[d] - mx) : 0.f;
    den += p[d];
  }
  const float rden = 1.0f / den;
#pragma unroll
  for (int d = 0; d < kLeft; ++d) p[d] *= rden;
  // ---- o = sum_d p_d v_{t-d}, clamped, chunk by chunk
  T *orow = out + t * ld_out + h * kHeadDim;
#pragma unroll 1
  for (int c = 0; c < kHeadDim / 16; ++c) {
    float o[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = 0.f;
#pragma unroll
    for (int d = 0; d < kLeft; ++d) {
      float vv[16];
      IO::load16(Vs + (tid + kLeft - 1 - d) * IO::kPitch + c * 16, vv);
#pragma unroll
      for (int i = 0; i < 16; ++i) o[i] = fmaf(p[d], vv[i], o[i]);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = clampf(o[i], lo, hi);
    IO::store16(orow + c * 16, o);
  }
}

template <typename T>
static cudaError_t attn_launch(const void *q, const void *k, const void *v, int64_t ld, const float *R,
                               const float *qscale, float k_scale, float cap, const int32_t *pos, int64_t n_tok,
                               void *out, int64_t ld_out, float lo, float hi, cudaStream_t s) {
  const size_t smem = 2 * kRows * AttnIO<T>::kPitch * sizeof(T) + (kLeft * kHeadDim + kHeadDim) * sizeof(float);
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_attention<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  dim3 grid((unsigned)((n_tok + kTQ - 1) / kTQ), kHeads);
  k_attention<T><<<grid, kTQ, smem, s>>>(static_cast<const T *>(q), static_cast<const T *>(k),
                                         static_cast<const T *>(v), ld, R, qscale, k_scale, cap, pos, n_tok,
                                         static_cast<T *>(out), ld_out, lo, hi);
  return cudaGetLastError();
}

cudaError_t launch_attention(bool is_bf16, const void *q, const void *k, const void *v, int64_t ld, const float *R,
                             const float *qscale, float k_scale, float cap, const int32_t *pos, int64_t T, void *out,
                             int64_t ld_out, float lo, float hi, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  if (is_bf16) return attn_launch<bf16>(q, k, v, ld, R, qscale, k_scale, cap, pos, T, out, ld_out, lo, hi, s);
  return attn_launch<float>(q, k, v, ld, R, qscale, k_scale, cap, pos, T, out, ld_out, lo, hi, s);
}

}  // namespace ae
