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

// The first convolution on the tensor cores, the depthwise one from shared
// memory. A work item is a run of up to kLencStemRun consecutive rows t2 of
// one clip (the output of the two convolutions); the item's mel rows are
// staged once. Each step computes two rows t1 of the first convolution, 128
// positions (t1, f1) against the 256 channels, as one tcgen05 product with
// K = 32: position r's A row is its 3 x 3 mel patch split into bf16 parts
// (p_hi, p_hi, p_lo) and channel c's B row the taps as (w_hi, w_lo, w_hi), so
// the product is p_hi w_hi + p_hi w_lo + p_lo w_hi (about 16 bits) in float32.
// Two tensor-memory accumulators alternate, so the next step's product runs
// while the current one is drained: bias, ReLU, bf16, into a ring of three
// rows t1 in shared memory ([row][f1][channel], 16-byte pieces swizzled by
// f1), beside a fourth row of zeros that stands for the first convolution's
// rows outside the clip (the second's zero padding). A step that completes
// rows 2 t2 and 2 t2 + 1 then gives output row t2 from rows 2 t2 - 1 .. 2 t2 + 1.
// The item's first step computes rows 2 a - 2 and 2 a - 1 when it does not
// start the clip.
constexpr int kS1Threads = 512;
constexpr int kS1MelRows = 4 * kLencStemRun + 5;
constexpr int kS1MelPitch = 132;  // floats: zeros at 0..3 (column -1 at index 3), the 128 columns from 4
constexpr uint32_t kS1ABytes = 128 * 128, kS1BBytes = 256 * 128, kS1RingBytes = 64 * 512;
constexpr size_t kS1Smem = 1024 + kS1ABytes + kS1BBytes + 4 * kS1RingBytes +
                           sizeof(float) * (kS1MelRows * kS1MelPitch + kLencStemCh) + 64;
static_assert(kS1Smem <= 227 * 1024, "one CTA per SM");

__device__ __forceinline__ void s1_cp(float *dst, const float *src, int bytes_max, bool valid) {
  const uint32_t d = smem_u32(dst);
  if (bytes_max == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(valid ? 16 : 0) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(d), "l"(src), "r"(valid ? 4 : 0) : "memory");
}

__device__ __forceinline__ uint32_t relu_bf16x2(float a, float b) {
  const __nv_bfloat162 v = __hmax2(__floats2bfloat162_rn(a, b), __float2bfloat162_rn(0.f));
  return *reinterpret_cast<const uint32_t *>(&v);
}

__global__ void __launch_bounds__(kS1Threads, 1) k_lenc_stem01(const float *__restrict__ mel, int mel16,
                                                              const bf16 *__restrict__ w0b,
                                                              const float *__restrict__ b0,
                                                              const float *__restrict__ w1,
                                                              const float *__restrict__ b1, bf16 *__restrict__ y2,
                                                              const LencTablesDev t, int n_items, unsigned *status) {
  extern __shared__ uint8_t s1_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(s1_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem, *sB = smem + kS1ABytes, *ring = sB + kS1BBytes;  // ring slots 0..2, slot 3 all zero
  float *s_mel = reinterpret_cast<float *>(ring + 4 * kS1RingBytes);
  float *s_b0 = s_mel + kS1MelRows * kS1MelPitch;
  uint64_t *bar = reinterpret_cast<uint64_t *>(s_b0 + kLencStemCh);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + 2);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // the taps once (swizzled rows of 128 bytes), A's granules 4..7 zero, the zero row, column -1 zero
  for (int i = tid; i < kLencStemCh * 8; i += kS1Threads) {
    const int n = i >> 3, g = i & 7;
    *reinterpret_cast<uint4 *>(sB + n * 128 + ((g ^ (n & 7)) << 4)) = __ldg(reinterpret_cast<const uint4 *>(w0b) + i);
  }
  if (tid < 128) {
#pragma unroll
    for (int g = 4; g < 8; ++g) *reinterpret_cast<uint4 *>(sA + tid * 128 + ((g ^ (tid & 7)) << 4)) = make_uint4(0, 0, 0, 0);
  }
  for (int i = tid; i < (int)(kS1RingBytes / 16); i += kS1Threads)
    reinterpret_cast<uint4 *>(ring + 3 * kS1RingBytes)[i] = make_uint4(0, 0, 0, 0);
  for (int c = tid; c < kLencStemCh; c += kS1Threads) s_b0[c] = __ldg(b0 + c);
  for (int i = tid; i < kS1MelRows * 4; i += kS1Threads) s_mel[(i >> 2) * kS1MelPitch + (i & 3)] = 0.f;
  const int cp = tid & 127, fq = tid >> 7;  // depthwise: channels 2 cp, 2 cp + 1; outputs f2 = 8 fq .. 8 fq + 7
  float2 wk[9], bias1;
#pragma unroll
  for (int k = 0; k < 9; ++k) wk[k] = make_float2(__ldg(w1 + (2 * cp) * 9 + k), __ldg(w1 + (2 * cp + 1) * 9 + k));
  bias1 = make_float2(__ldg(b1 + 2 * cp), __ldg(b1 + 2 * cp + 1));
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // A rows of the step whose first row is r0: thread m < 128 is position (r0 + m / 64, m mod 64)
  auto build_a = [&](int r0, int mrow0) {
    if (tid >= 128) return;
    const int m = tid, t1 = r0 + (m >> 6), f1 = m & 63;
    const float *src = s_mel + (2 * t1 - 1 - mrow0) * kS1MelPitch + 3 + 2 * f1;
    float kv[32];
#pragma unroll
    for (int dt = 0; dt < 3; ++dt)
#pragma unroll
      for (int df = 0; df < 3; ++df) {
        const float p = src[dt * kS1MelPitch + df];
        const float hi = __bfloat162float(__float2bfloat16_rn(p));
        kv[dt * 3 + df] = hi;
        kv[9 + dt * 3 + df] = hi;
        kv[18 + dt * 3 + df] = p - hi;
      }
#pragma unroll
    for (int k = 27; k < 32; ++k) kv[k] = 0.f;
    uint8_t *row = sA + m * 128;
#pragma unroll
    for (int g = 0; g < 4; ++g)
      *reinterpret_cast<uint4 *>(row + ((g ^ (m & 7)) << 4)) =
          make_uint4(pack_bf16(kv[8 * g], kv[8 * g + 1]), pack_bf16(kv[8 * g + 2], kv[8 * g + 3]),
                     pack_bf16(kv[8 * g + 4], kv[8 * g + 5]), pack_bf16(kv[8 * g + 6], kv[8 * g + 7]));
    fence_async_smem();
  };
  auto issue = [&](int acc) {
    tc_fence_after();
    const uint32_t aa = smem_u32(sA), bb = smem_u32(sB);
#pragma unroll
    for (int k = 0; k < 2; ++k)
      tc_mma_bf16(tmem + (uint32_t)(acc * 256), sw128_desc(aa + k * 32), sw128_desc(bb + k * 32),
                  idesc_bf16_f32(128, 256), k > 0 ? 1u : 0u);
    tc_commit(&bar[acc]);
  };

  int64_t step = 0;
  bool ok = true;
  for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
    const int c = lenc_clip_of(t.s2item_off, t.n_clips, item);
    const int a = (item - t.s2item_off[c]) * kLencStemRun;
    const int T2 = t.s2_off[c + 1] - t.s2_off[c];
    const int b = min(T2, a + kLencStemRun);
    const int F = t.frame_off[c + 1] - t.frame_off[c], T1 = (F + 1) / 2;
    const int mrow0 = 4 * a - 5;  // staged row i is mel row mrow0 + i
    const float *m = mel + (int64_t)t.frame_off[c] * kLencMels;
    {
      const int nrows = 4 * (b - a) + 5, per_row = mel16 ? 32 : 128, w = mel16 ? 4 : 1;
      for (int i = tid; i < nrows * per_row; i += kS1Threads) {
        const int r = i / per_row, q = i % per_row, fr = mrow0 + r;
        const bool valid = fr >= 0 && fr < F;
        s1_cp(s_mel + r * kS1MelPitch + 4 + q * w, valid ? m + (int64_t)fr * kLencMels + q * w : mel, 4 * w, valid);
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      asm volatile("cp.async.wait_all;" ::: "memory");
    }
    __syncthreads();  // mel staged; the previous item is done with the ring and A
    const int first = a > 0 ? 2 * a - 2 : 0;
    const int nsteps = b - a + (a > 0 ? 1 : 0);
    build_a(first, mrow0);
    __syncthreads();
    if (tid == 0) issue((int)(step & 1));
    for (int sidx = 0; sidx < nsteps; ++sidx, ++step) {
      const int r0 = first + 2 * sidx, acc = (int)(step & 1);
      if (!__syncthreads_and(mbar_wait(&bar[acc], (uint32_t)((step >> 1) & 1)))) {
        if (tid == 0) atomicOr(status, kStatusWaitTimeout);
        ok = false;
        break;
      }
      tc_fence_after();
      if (sidx + 1 < nsteps) build_a(r0 + 2, mrow0);  // A is free: this step's product is done
      __syncthreads();  // the next A is built; the previous step's depthwise reads are done
      if (tid == 0 && sidx + 1 < nsteps) issue(acc ^ 1);
      {  // drain: warp w reads lanes 32 (w & 3) .. + 31 (positions), channels 64 (w >> 2) .. + 63
        const int pos = 32 * (warp & 3) + lane, t1 = r0 + (pos >> 6), f1 = pos & 63, ch0 = 64 * (warp >> 2);
        const uint32_t taddr = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(acc * 256 + ch0);
        uint8_t *rrow = ring + (t1 % 3) * kS1RingBytes + f1 * 512;
        const int sw = f1 & 31;
        uint32_t v0[32], v1[32];
        tmem_ld32(taddr, v0);
        tmem_ld32(taddr + 32, v1);
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t *v = h ? v1 : v0;
          const int cb = ch0 + 32 * h;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const float4 bA = *reinterpret_cast<const float4 *>(s_b0 + cb + 8 * g);
            const float4 bB = *reinterpret_cast<const float4 *>(s_b0 + cb + 8 * g + 4);
            const int e = 8 * g;
            const float2 p0 = __fadd2_rn(make_float2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), make_float2(bA.x, bA.y));
            const float2 p1 = __fadd2_rn(make_float2(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3])), make_float2(bA.z, bA.w));
            const float2 p2 = __fadd2_rn(make_float2(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5])), make_float2(bB.x, bB.y));
            const float2 p3 = __fadd2_rn(make_float2(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7])), make_float2(bB.z, bB.w));
            *reinterpret_cast<uint4 *>(rrow + (((cb >> 3) + g) ^ sw) * 16) =
                make_uint4(relu_bf16x2(p0.x, p0.y), relu_bf16x2(p1.x, p1.y), relu_bf16x2(p2.x, p2.y),
                           relu_bf16x2(p3.x, p3.y));
          }
        }
      }
      tc_fence_before();
      __syncthreads();  // ring rows r0, r0 + 1 written
      if ((r0 >> 1) < a) continue;  // the item's first step when it does not start the clip
      {  // output row t2 = r0 / 2 from ring rows 2 t2 - 1 .. 2 t2 + 1 (the zero row outside the clip)
        const int t2 = r0 >> 1;
        const uint8_t *rb[3];
#pragma unroll
        for (int dt = 0; dt < 3; ++dt) {
          const int t1 = 2 * t2 - 1 + dt;
          rb[dt] = ring + (t1 >= 0 && t1 < T1 ? t1 % 3 : 3) * kS1RingBytes + 16 * fq * 512 + (cp & 3) * 4;
        }
        // column 16 fq + k (0 <= k < 16) holds this thread's channels in piece (cp / 4) ^ (16 (fq & 1) + k)
        const int q = (cp >> 2) ^ (16 * (fq & 1));
        auto ld = [&](int dt, int k) {
          const uint32_t v = *reinterpret_cast<const uint32_t *>(rb[dt] + k * 512 + ((q ^ k) << 4));
          return make_float2(bf16lo(v), bf16hi(v));
        };
        float2 left[3];
        {  // column 16 fq - 1: the zero padding for fq = 0
          const int ql = (cp >> 2) ^ ((16 * fq - 1) & 31);
#pragma unroll
          for (int dt = 0; dt < 3; ++dt) {
            const uint32_t v = fq ? *reinterpret_cast<const uint32_t *>(rb[dt] - 512 + (ql << 4)) : 0u;
            left[dt] = make_float2(bf16lo(v), bf16hi(v));
          }
        }
        bf16 *orow = y2 + ((int64_t)(t.s2_off[c] + t2) * 32 + 8 * fq) * kLencStemCh + 2 * cp;
#pragma unroll
        for (int i = 0; i < 8; ++i) {  // f2 = 8 fq + i reads columns 2 i - 1 .. 2 i + 1 of the quarter
          float2 o = bias1;
#pragma unroll
          for (int dt = 0; dt < 3; ++dt) {
            const float2 mid = ld(dt, 2 * i), right = ld(dt, 2 * i + 1);
            ffma2(o, wk[dt * 3 + 0], left[dt]);
            ffma2(o, wk[dt * 3 + 1], mid);
            ffma2(o, wk[dt * 3 + 2], right);
            left[dt] = right;
          }
          *reinterpret_cast<uint32_t *>(orow + i * kLencStemCh) = pack_bf16(o.x, o.y);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
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
  bool trok[3];  // input rows inside the clip
#pragma unroll
  for (int dt = 0; dt < 3; ++dt) trok[dt] = 2 * t3 + dt - 1 >= 0 && 2 * t3 + dt - 1 < T2;
  // two output columns per step: their 18 loads are issued before the sums
#pragma unroll 1
  for (int f3 = 0; f3 < 16; f3 += 2) {
    uint32_t v[2][9];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int dt = 0; dt < 3; ++dt)
#pragma unroll
        for (int df = 0; df < 3; ++df) {
          const int fr = 2 * (f3 + h) + df - 1;
          v[h][dt * 3 + df] =
              trok[dt] && fr >= 0
                  ? *reinterpret_cast<const uint32_t *>(src + ((int64_t)(2 * t3 + dt - 1) * 32 + fr) * kLencStemCh)
                  : 0u;
        }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float2 a = bias;
#pragma unroll
      for (int dt = 0; dt < 3; ++dt) {
        if (!trok[dt]) continue;
#pragma unroll
        for (int df = 0; df < 3; ++df) {
          if (2 * (f3 + h) + df - 1 < 0) continue;
          const uint32_t x = v[h][dt * 3 + df];
          ffma2(a, wk[dt * 3 + df], make_float2(bf16lo(x), bf16hi(x)));
        }
      }
      *reinterpret_cast<uint32_t *>(out + (row * 16 + f3 + h) * (int64_t)kLencStemCh + ch) = pack_bf16(a.x, a.y);
    }
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
// memory (bf16, 16-byte cp.async, zero fill outside the batch) and each
// thread computes two channels of every row. SiLU is y / (1 + 2^(-y log2 e))
// with the hardware's ex2 and reciprocal.
constexpr int kDwRows = 16;

__device__ __forceinline__ float lenc_silu(float y) {
  float e, r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-1.4426950408889634f * y));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + e));
  return y * r;
}

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
  for (int i = threadIdx.x; i < nrows * 64; i += 256) {  // 16-byte chunks: 64 per 512-channel row
    const int rr = i >> 6, q = i & 63;
    const int64_t tr = t0 - lo + rr;
    const bool ok = tr >= 0 && tr < T;
    const uint32_t d = smem_u32(s_g + rr * 256 + 4 * q);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d),
                 "l"(ok ? g + tr * kLencEmbd + 8 * q : g), "r"(ok ? 16 : 0)
                 : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  const int ch = 2 * threadIdx.x;
  float2 wr[KT > 0 ? KT : 1];
  if (KT > 0) {
#pragma unroll
    for (int m = 0; m < (KT > 0 ? KT : 1); ++m) wr[m] = make_float2(__ldg(w + m * kLencEmbd + ch), __ldg(w + m * kLencEmbd + ch + 1));
  }
  const float2 bias = make_float2(db[ch], db[ch + 1]), sc = make_float2(aw[ch], aw[ch + 1]),
               sh = make_float2(ab[ch], ab[ch + 1]);
  int c = lenc_clip_of(tok_off, n_clips, t0 < T ? t0 : T - 1);
  int64_t s0 = tok_off[c], e = tok_off[c + 1];  // the current clip's rows, kept in registers
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
#pragma unroll 1
  for (int r = 0; r < kDwRows; ++r) {
    const int64_t tt = t0 + r;
    if (tt >= T) break;
    while (e <= tt) {  // rows are in order; clips may be empty
      ++c;
      s0 = e;
      e = tok_off[c + 1];
    }
    const int m0 = (int)max((int64_t)0, s0 - (tt - lo)), m1 = (int)min((int64_t)k, e - (tt - lo));
    float2 a = bias;
    if (KT > 0) {
      if (m0 == 0 && m1 == KT) {  // the whole window inside the clip: no per-tap test
#pragma unroll
        for (int m = 0; m < (KT > 0 ? KT : 1); ++m) {
          const uint32_t v = s_g[(r + m) * 256 + threadIdx.x];
          ffma2(a, wr[m], make_float2(bf16lo(v), bf16hi(v)));
        }
      } else {
#pragma unroll
        for (int m = 0; m < (KT > 0 ? KT : 1); ++m)
          if (m >= m0 && m < m1) {
            const uint32_t v = s_g[(r + m) * 256 + threadIdx.x];
            ffma2(a, wr[m], make_float2(bf16lo(v), bf16hi(v)));
          }
      }
    } else {
      for (int m = m0; m < m1; ++m) {
        const uint32_t v = s_g[(r + m) * 256 + threadIdx.x];
        ffma2(a, make_float2(__ldg(w + m * kLencEmbd + ch), __ldg(w + m * kLencEmbd + ch + 1)),
              make_float2(bf16lo(v), bf16hi(v)));
      }
    }
    const float2 y = __ffma2_rn(a, sc, sh);
    *reinterpret_cast<uint32_t *>(out + tt * kLencEmbd + ch) = pack_bf16(lenc_silu(y.x), lenc_silu(y.y));
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

cudaError_t launch_lenc_stem01(const float *mel, const void *w0b, const float *b0, const float *w1, const float *b1,
                               void *y2, const LencTablesDev &t, int64_t s2_items, cudaStream_t s) {
  if (s2_items <= 0) return cudaSuccess;
  static std::atomic<uint64_t> attr{0};
  if (const cudaError_t e = smem_attr(k_lenc_stem01, kS1Smem, attr)) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = (int)(s2_items < sms ? s2_items : sms);
  const int mel16 = (reinterpret_cast<uintptr_t>(mel) & 15) == 0 ? 1 : 0;
  return launch_k(k_lenc_stem01, dim3((unsigned)grid), dim3(kS1Threads), kS1Smem, s, mel, mel16,
                  static_cast<const bf16 *>(w0b), b0, w1, b1, static_cast<bf16 *>(y2), t, (int)s2_items,
                  device_status_word());
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
  // the attribute is set once per device, so the generic form takes the size
  // of the widest kernel it accepts (models of other widths may follow)
  static std::atomic<uint64_t> attr9{0}, attr0{0};
  auto kern = k == 9 ? k_lenc_dwconv<9> : k_lenc_dwconv<0>;
  const size_t smem_max = k == 9 ? smem : (size_t)(kDwRows + kLencMaxConvK - 1) * 256 * 4;
  if (const cudaError_t e = smem_attr(kern, smem_max, k == 9 ? attr9 : attr0)) return e;
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
