// Chunked local attention core (egemma2_audio.rs, AudioTower::attention):
// per head, token t attends to itself and the 11 tokens before it within its
// clip; logits z_d = (q s) . (k_scale k_{t-d}) + (q s) . R[d] with
// s = log2(e)/sqrt(128) * softplus(per_dim_scale), capped as
// cap * tanh(z / cap); natural-exp softmax over the distances; o_t =
// sum_d p_d v_{t-d}.
//
// bf16 kernel: a CTA owns one head and 256 consecutive tokens; each of its
// 128 threads owns two consecutive queries (t, t+1), which share 11 of the
// 13 key/value rows they read. The CTA stages the head's k rows (and then,
// in the same buffer, its v rows) for its tokens and the 11-row halo in
// shared memory; rows are 256 bytes with their 16-byte chunks XOR-swizzled
// by (row / 2) mod 8, so the eight lanes of a shared-memory phase, which read
// rows two apart, hit distinct banks. R[0..11] is staged pre-divided by
// k_scale, so q.k and q.R accumulate into one register per (query, distance)
// and z = k_scale * acc. Dot products and the weighted sum of v use the
// packed two-wide FMA (fma.rn.f32x2). The softmax over the 12 logits is
// private to the thread; no cross-thread reduction is needed.
//
// float32 kernel (the float32 model): one query per thread, padded rows.
#include "ae_internal.h"
#include "common.cuh"

namespace ae {

__device__ __forceinline__ float2 bf2(uint32_t w) { return make_float2(bf16lo(w), bf16hi(w)); }

namespace {
constexpr int A2_THREADS = 128;
constexpr int A2_TOK = 2 * A2_THREADS;          // tokens per CTA
constexpr int A2_ROWS = A2_TOK + kLeft - 1;     // staged rows
constexpr size_t A2_SMEM = (size_t)A2_ROWS * kHeadDim * 2 + (kLeft * kHeadDim + kHeadDim) * 4;
}  // namespace

// 16-byte chunk c (0..15) of staged row r
__device__ __forceinline__ const uint4 *a2_chunk(const bf16 *buf, int r, int c) {
  return reinterpret_cast<const uint4 *>(buf + r * kHeadDim) + (c ^ ((r >> 1) & 7));
}

__device__ __forceinline__ void a2_stage(bf16 *buf, const bf16 *__restrict__ src, int64_t ld, int h, int64_t t0,
                                         int64_t T) {
  for (int idx = threadIdx.x; idx < A2_ROWS * 16; idx += A2_THREADS) {
    const int r = idx >> 4, c = idx & 15;
    const int64_t tok = t0 - (kLeft - 1) + r;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (tok >= 0 && tok < T) v = __ldg(reinterpret_cast<const uint4 *>(src + tok * ld + h * kHeadDim) + c);
    reinterpret_cast<uint4 *>(buf + r * kHeadDim)[c ^ ((r >> 1) & 7)] = v;
  }
}

__global__ void __launch_bounds__(A2_THREADS, 3)
    k_attention_bf16(const bf16 *__restrict__ q, const bf16 *__restrict__ k, const bf16 *__restrict__ v, int64_t ld,
                     const float *__restrict__ R, const float *__restrict__ qscale, float k_scale, float cap,
                     const int32_t *__restrict__ pos, int64_t T, bf16 *__restrict__ out, int64_t ld_out, float lo,
                     float hi) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  bf16 *buf = reinterpret_cast<bf16 *>(smem_raw);
  float *Rt = reinterpret_cast<float *>(buf + A2_ROWS * kHeadDim);  // R / k_scale, [12][128]
  float *Qs = Rt + kLeft * kHeadDim;                                // [128]
  const int h = blockIdx.y;
  const int64_t t0 = (int64_t)blockIdx.x * A2_TOK;
  const int i = threadIdx.x;
  const float inv_ks = 1.0f / k_scale;
  for (int x = i; x < kLeft * kHeadDim; x += A2_THREADS)
    Rt[x] = R[(x / kHeadDim) * kHidden + h * kHeadDim + x % kHeadDim] * inv_ks;
  Qs[i] = qscale[i];
  a2_stage(buf, k, ld, h, t0, T);
  __syncthreads();

  const int64_t ta = t0 + 2 * i, tb = ta + 1;
  const bool va = ta < T, vb = tb < T;
  const int64_t tqa = va ? ta : T - 1, tqb = vb ? tb : T - 1;  // clamped row for loads
  const int spa = va ? min(pos[ta] + 1, kLeft) : 1;
  const int spb = vb ? min(pos[tb] + 1, kLeft) : 1;
  const bf16 *qa_row = q + tqa * ld + h * kHeadDim;
  const bf16 *qb_row = q + tqb * ld + h * kHeadDim;

  float2 acc[2][kLeft];
#pragma unroll
  for (int d = 0; d < kLeft; ++d) acc[0][d] = acc[1][d] = make_float2(0.f, 0.f);
  // q of the next chunk is loaded while the current one is used
  uint4 na0 = __ldg(reinterpret_cast<const uint4 *>(qa_row)), na1 = __ldg(reinterpret_cast<const uint4 *>(qa_row) + 1);
  uint4 nb0 = __ldg(reinterpret_cast<const uint4 *>(qb_row)), nb1 = __ldg(reinterpret_cast<const uint4 *>(qb_row) + 1);
#pragma unroll 1
  for (int cc = 0; cc < kHeadDim / 16; ++cc) {
    float2 qa[8], qb[8];
    {
      const uint4 a0 = na0, a1 = na1, b0 = nb0, b1 = nb1;
      if (cc + 1 < kHeadDim / 16) {
        na0 = __ldg(reinterpret_cast<const uint4 *>(qa_row + (cc + 1) * 16));
        na1 = __ldg(reinterpret_cast<const uint4 *>(qa_row + (cc + 1) * 16) + 1);
        nb0 = __ldg(reinterpret_cast<const uint4 *>(qb_row + (cc + 1) * 16));
        nb1 = __ldg(reinterpret_cast<const uint4 *>(qb_row + (cc + 1) * 16) + 1);
      }
      const uint32_t wa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const uint32_t wb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
      const float4 *qs4 = reinterpret_cast<const float4 *>(Qs + cc * 16);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float4 s = qs4[m];
        const float2 a_lo = bf2(wa[2 * m]), a_hi = bf2(wa[2 * m + 1]);
        const float2 b_lo = bf2(wb[2 * m]), b_hi = bf2(wb[2 * m + 1]);
        qa[2 * m] = make_float2(a_lo.x * s.x, a_lo.y * s.y);
        qa[2 * m + 1] = make_float2(a_hi.x * s.z, a_hi.y * s.w);
        qb[2 * m] = make_float2(b_lo.x * s.x, b_lo.y * s.y);
        qb[2 * m + 1] = make_float2(b_hi.x * s.z, b_hi.y * s.w);
      }
    }
    // key rows 2i .. 2i+12 (local): distance 11-j for query a, 12-j for query b
#pragma unroll
    for (int j = 0; j <= kLeft; ++j) {
      const uint4 c0 = *a2_chunk(buf, 2 * i + j, 2 * cc), c1 = *a2_chunk(buf, 2 * i + j, 2 * cc + 1);
      const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const float2 kk = bf2(w[m]);
        if (j <= kLeft - 1) ffma2(acc[0][kLeft - 1 - j], qa[m], kk);
        if (j >= 1) ffma2(acc[1][kLeft - j], qb[m], kk);
      }
    }
#pragma unroll
    for (int d = 0; d < kLeft; ++d) {
      const float4 *r4 = reinterpret_cast<const float4 *>(Rt + d * kHeadDim + cc * 16);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float4 r = r4[m];
        ffma2(acc[0][d], qa[2 * m], make_float2(r.x, r.y));
        ffma2(acc[0][d], qa[2 * m + 1], make_float2(r.z, r.w));
        ffma2(acc[1][d], qb[2 * m], make_float2(r.x, r.y));
        ffma2(acc[1][d], qb[2 * m + 1], make_float2(r.z, r.w));
      }
    }
  }
  // ---- capped logits and softmax per query
  float p[2][kLeft];
#pragma unroll
  for (int qq = 0; qq < 2; ++qq) {
    const int span = qq == 0 ? spa : spb;
    float mx = -INFINITY;
#pragma unroll
    for (int d = 0; d < kLeft; ++d) {
      const float z = cap * tanhf(k_scale * (acc[qq][d].x + acc[qq][d].y) / cap);
      p[qq][d] = d < span ? z : -INFINITY;
      mx = fmaxf(mx, p[qq][d]);
    }
    float den = 0.f;
#pragma unroll
    for (int d = 0; d < kLeft; ++d) {
      p[qq][d] = d < span ? __expf(p[qq][d] - mx) : 0.f;
      den += p[qq][d];
    }
    const float rd = 1.0f / den;
#pragma unroll
    for (int d = 0; d < kLeft; ++d) p[qq][d] *= rd;
  }
  __syncthreads();  // everyone is done with the k rows
  a2_stage(buf, v, ld, h, t0, T);
  __syncthreads();
  // ---- o = sum_d p_d v_{t-d}
  bf16 *oa_row = out + tqa * ld_out + h * kHeadDim;
  bf16 *ob_row = out + tqb * ld_out + h * kHeadDim;
#pragma unroll 1
  for (int cc = 0; cc < kHeadDim / 16; ++cc) {
    float2 oa[8], ob[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) oa[m] = ob[m] = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j <= kLeft; ++j) {
      const uint4 c0 = *a2_chunk(buf, 2 * i + j, 2 * cc), c1 = *a2_chunk(buf, 2 * i + j, 2 * cc + 1);
      const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      const float pa = j <= kLeft - 1 ? p[0][kLeft - 1 - j] : 0.f;
      const float pb = j >= 1 ? p[1][kLeft - j] : 0.f;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const float2 vv = bf2(w[m]);
        if (j <= kLeft - 1) ffma2(oa[m], make_float2(pa, pa), vv);
        if (j >= 1) ffma2(ob[m], make_float2(pb, pb), vv);
      }
    }
    uint32_t wa[8], wb[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      wa[m] = pack_bf16(clampf(oa[m].x, lo, hi), clampf(oa[m].y, lo, hi));
      wb[m] = pack_bf16(clampf(ob[m].x, lo, hi), clampf(ob[m].y, lo, hi));
    }
    if (va) {
      reinterpret_cast<uint4 *>(oa_row + cc * 16)[0] = make_uint4(wa[0], wa[1], wa[2], wa[3]);
      reinterpret_cast<uint4 *>(oa_row + cc * 16)[1] = make_uint4(wa[4], wa[5], wa[6], wa[7]);
    }
    if (vb) {
      reinterpret_cast<uint4 *>(ob_row + cc * 16)[0] = make_uint4(wb[0], wb[1], wb[2], wb[3]);
      reinterpret_cast<uint4 *>(ob_row + cc * 16)[1] = make_uint4(wb[4], wb[5], wb[6], wb[7]);
    }
  }
}

// ------------------------------------------------------------------ float32 kernel

namespace {
constexpr int kTQ = 128;                 // queries per CTA
constexpr int kRows = kTQ + kLeft - 1;   // staged k/v rows
constexpr int kPitchF = kHeadDim + 4;    // floats per staged row (528 bytes)
}  // namespace

__global__ void __launch_bounds__(kTQ) k_attention_f32(const float *__restrict__ q, const float *__restrict__ k,
                                                       const float *__restrict__ v, int64_t ld,
                                                       const float *__restrict__ R, const float *__restrict__ qscale,
                                                       float k_scale, float cap, const int32_t *__restrict__ pos,
                                                       int64_t T_total, float *__restrict__ out, int64_t ld_out,
                                                       float lo, float hi) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float *Ks = reinterpret_cast<float *>(smem_raw);
  float *Vs = Ks + kRows * kPitchF;
  float *Rs = Vs + kRows * kPitchF;  // [12][128]
  float *Qs = Rs + kLeft * kHeadDim;  // [128]
  const int h = blockIdx.y;
  const int64_t t0 = (int64_t)blockIdx.x * kTQ;
  const int tid = threadIdx.x;
  for (int idx = tid; idx < kRows * (kHeadDim / 4); idx += kTQ) {
    const int r = idx / (kHeadDim / 4), ch = idx % (kHeadDim / 4);
    const int64_t tok = t0 - (kLeft - 1) + r;
    float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
    if (tok >= 0 && tok < T_total) {
      kv = *reinterpret_cast<const float4 *>(k + tok * ld + h * kHeadDim + ch * 4);
      vv = *reinterpret_cast<const float4 *>(v + tok * ld + h * kHeadDim + ch * 4);
    }
    *reinterpret_cast<float4 *>(Ks + r * kPitchF + ch * 4) = kv;
    *reinterpret_cast<float4 *>(Vs + r * kPitchF + ch * 4) = vv;
  }
  for (int x = tid; x < kLeft * kHeadDim; x += kTQ) Rs[x] = R[(x / kHeadDim) * kHidden + h * kHeadDim + x % kHeadDim];
  Qs[tid] = qscale[tid];
  __syncthreads();
  const int64_t t = t0 + tid;
  if (t >= T_total) return;
  const int span = min(pos[t] + 1, kLeft);
  const float *qrow = q + t * ld + h * kHeadDim;
  float d1[kLeft], d2[kLeft];
#pragma unroll
  for (int d = 0; d < kLeft; ++d) d1[d] = d2[d] = 0.f;
#pragma unroll 1
  for (int c = 0; c < kHeadDim / 4; ++c) {
    const float4 q4 = *reinterpret_cast<const float4 *>(qrow + c * 4);
    const float qv[4] = {q4.x * Qs[c * 4], q4.y * Qs[c * 4 + 1], q4.z * Qs[c * 4 + 2], q4.w * Qs[c * 4 + 3]};
#pragma unroll
    for (int d = 0; d < kLeft; ++d) {
      const float4 kk = *reinterpret_cast<const float4 *>(Ks + (tid + kLeft - 1 - d) * kPitchF + c * 4);
      const float4 rr = *reinterpret_cast<const float4 *>(Rs + d * kHeadDim + c * 4);
      d1[d] = fmaf(qv[0], kk.x, fmaf(qv[1], kk.y, fmaf(qv[2], kk.z, fmaf(qv[3], kk.w, d1[d]))));
      d2[d] = fmaf(qv[0], rr.x, fmaf(qv[1], rr.y, fmaf(qv[2], rr.z, fmaf(qv[3], rr.w, d2[d]))));
    }
  }
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
  float *orow = out + t * ld_out + h * kHeadDim;
#pragma unroll 1
  for (int c = 0; c < kHeadDim / 4; ++c) {
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int d = 0; d < kLeft; ++d) {
      const float4 vv = *reinterpret_cast<const float4 *>(Vs + (tid + kLeft - 1 - d) * kPitchF + c * 4);
      const float w = p[d] * rden;
      o.x = fmaf(w, vv.x, o.x);
      o.y = fmaf(w, vv.y, o.y);
      o.z = fmaf(w, vv.z, o.z);
      o.w = fmaf(w, vv.w, o.w);
    }
    *reinterpret_cast<float4 *>(orow + c * 4) =
        make_float4(clampf(o.x, lo, hi), clampf(o.y, lo, hi), clampf(o.z, lo, hi), clampf(o.w, lo, hi));
  }
}

cudaError_t launch_attention(bool is_bf16, const void *q, const void *k, const void *v, int64_t ld, const float *R,
                             const float *qscale, float k_scale, float cap, const int32_t *pos, int64_t T, void *out,
                             int64_t ld_out, float lo, float hi, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  if (is_bf16) {
    static bool attr = false;
    if (!attr) {
      cudaError_t e = cudaFuncSetAttribute(k_attention_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)A2_SMEM);
      if (e != cudaSuccess) return e;
      attr = true;
    }
    dim3 grid((unsigned)((T + A2_TOK - 1) / A2_TOK), kHeads);
    return launch_k(k_attention_bf16, grid, dim3(A2_THREADS), A2_SMEM, s, static_cast<const bf16 *>(q),
                    static_cast<const bf16 *>(k), static_cast<const bf16 *>(v), ld, R, qscale, k_scale, cap, pos, T,
                    static_cast<bf16 *>(out), ld_out, lo, hi);
  }
  const size_t smem = (2 * (size_t)kRows * kPitchF + kLeft * kHeadDim + kHeadDim) * sizeof(float);
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_attention_f32, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  dim3 grid((unsigned)((T + kTQ - 1) / kTQ), kHeads);
  return launch_k(k_attention_f32, grid, dim3(kTQ), smem, s, static_cast<const float *>(q),
                  static_cast<const float *>(k), static_cast<const float *>(v), ld, R, qscale, k_scale, cap, pos, T,
                  static_cast<float *>(out), ld_out, lo, hi);
}

}  // namespace ae
