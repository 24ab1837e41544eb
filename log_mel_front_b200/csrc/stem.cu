// Subsampling stem (egemma2_audio.rs, AudioTower::subsample): two 3x3
// stride-2 convolutions with zero padding 1 and no bias, each followed by a
// bias-free LayerNorm over the channels (eps 1e-6) and ReLU.
//
// conv0 (1 -> 128 channels): the channel mean of the outputs is linear in
// the 9-sample patch p and their variance is the quadratic form p^T C p of
// the taps' channel covariance C, so one pass gives the normalised outputs:
// y_c = relu(g_c (w'_c . p) / sqrt(p^T C p + eps)) with w'_c the taps minus
// their channel mean (taps times gains, and C, precomputed in float64 at
// model creation). A CTA writes four time rows [64 freq][128 ch] of the
// channels-last output.
//
// The output rows of each clip are laid out with two zero rows in front and
// zero rows after the last real one, up to 2 * tokens + 2 rows per clip, so
// the second convolution's stride-2 windows never need a bounds test in
// time and never read a neighbouring clip.
//
// conv1 (128 -> 32 channels) as an implicit GEMM on the tensor cores: the
// output rows (token, freq) are GEMM rows, K = 9 taps x 128 channels. For
// each tap the A tile (4 tokens x 32 freq x 64 channels) is one TMA box of a
// 5-D view of conv0's output that splits time and frequency into (pair,
// parity), so the stride-2 gather is a plain box; the frequency pad at -1 is
// the TMA's out-of-range zero fill. tcgen05.mma (M=128, N=32) accumulates
// in tensor memory; the epilogue thread of each row holds all 32 channels
// and applies the LayerNorm, ReLU and the frequency-major flatten.
#include "ae_internal.h"
#include "common.cuh"

namespace ae {

// Clip of a packed row index, by binary search over a prefix array [B+1].
__device__ __forceinline__ int clip_of(const int32_t *off, int n_clips, int64_t r) {
  int lo = 0, hi = n_clips;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (off[mid] <= r) lo = mid; else hi = mid;
  }
  return lo;
}

// ------------------------------------------------------------------ conv0 + LN + ReLU

// A CTA writes kConv0Rows stem rows (64 positions each). Phase 1: four
// threads locate the rows' clips; the three mel rows each stem row reads are
// staged in shared memory (coalesced, with a zero band on either side); the
// 45 distinct entries of the symmetric 9x9 covariance C sit in registers;
// each of the 256 positions then gets its 9-sample patch (stored duplicated
// as (p, p) pairs) and 1/sqrt(p^T C p + eps) in shared memory. Phase 2:
// thread (channel quad, position phase) holds its four channels' taps,
// pre-multiplied by the LayerNorm gains at model creation, in registers and
// walks the positions: two packed FMAs per tap cover the four channels;
// relu(r * (w'' . p)) is the normalised output (r > 0). Consecutive threads
// write consecutive channels of one position, so every row is written with
// full coalesced segments. Rows outside a clip's frames (the zero padding)
// come out as zeros.
constexpr int kConv0Rows = 4;

template <typename OutT>
__global__ void __launch_bounds__(128) k_conv0(const float *__restrict__ mel, const float *__restrict__ wg,
                                               const float *__restrict__ cov, OutT *__restrict__ y0,
                                               const ClipTablesDev t, int64_t stem_rows) {
  constexpr int P = kConv0Rows * kF1;  // positions per CTA
  constexpr int MP = kMels + 2;        // staged mel row with a zero band on either side
  __shared__ __align__(16) float2 s_pp[P][10];
  __shared__ float s_r[P];
  __shared__ float s_mel[kConv0Rows][3][MP];
  __shared__ int64_t s_base[kConv0Rows];
  __shared__ int s_ti[kConv0Rows], s_F[kConv0Rows];
  const int64_t row0 = (int64_t)blockIdx.x * kConv0Rows;
  if (threadIdx.x < kConv0Rows) {
    const int64_t row = row0 + threadIdx.x;
    int ti = -1, F = 0;
    int64_t base = 0;
    if (row < stem_rows) {
      const int c = clip_of(t.stem_off, t.n_clips, row);
      F = t.frame_off[c + 1] - t.frame_off[c];
      ti = (int)(row - t.stem_off[c]) - 2;
      if (ti >= (F + 1) / 2) ti = -1;
      base = (int64_t)t.frame_off[c] * kMels;
    }
    s_ti[threadIdx.x] = ti;
    s_F[threadIdx.x] = F;
    s_base[threadIdx.x] = base;
  }
  // C_aa and 2 C_ab (b > a): p^T C p = sum_a p_a (C_aa p_a + sum_{b>a} 2 C_ab p_b)
  float cv[45];
  {
    int n = 0;
#pragma unroll
    for (int a = 0; a < 9; ++a)
#pragma unroll
      for (int b = a; b < 9; ++b) cv[n++] = (b == a ? 1.0f : 2.0f) * __ldg(cov + a * 9 + b);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kConv0Rows * 3 * MP; i += blockDim.x) {
    const int rr = i / (3 * MP), dt = (i / MP) % 3, cc = i % MP;
    const int ti = s_ti[rr], tr = 2 * ti + dt - 1, fr = cc - 1;
    float v = 0.f;
    if (ti >= 0 && tr >= 0 && tr < s_F[rr] && fr >= 0 && fr < kMels) v = __ldg(mel + s_base[rr] + (int64_t)tr * kMels + fr);
    s_mel[rr][dt][cc] = v;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < P; i += blockDim.x) {
    const int rr = i / kF1, f = i % kF1;
    float p[9];
#pragma unroll
    for (int dt = 0; dt < 3; ++dt)
#pragma unroll
      for (int df = 0; df < 3; ++df) p[dt * 3 + df] = s_mel[rr][dt][2 * f + df];  // column 2f + df - 1, shifted by the band
    float var = 0.f;
    int n = 0;
#pragma unroll
    for (int a = 0; a < 9; ++a) {
      float s = 0.f;
#pragma unroll
      for (int b = a; b < 9; ++b) s = fmaf(cv[n++], p[b], s);
      var = fmaf(p[a], s, var);
    }
#pragma unroll
    for (int k = 0; k < 9; ++k) s_pp[i][k] = make_float2(p[k], p[k]);
    s_pp[i][9] = make_float2(0.f, 0.f);
    s_r[i] = rsqrtf(fmaxf(var, 0.f) + 1e-6f);
  }
  __syncthreads();
  const int cq = threadIdx.x & 31, ph = threadIdx.x >> 5;  // channels 4cq .. 4cq+3; positions ph, ph+4, ...
  float2 w01[10], w23[10];
#pragma unroll
  for (int k = 0; k < 9; ++k) {
    w01[k] = make_float2(__ldg(wg + (4 * cq) * 9 + k), __ldg(wg + (4 * cq + 1) * 9 + k));
    w23[k] = make_float2(__ldg(wg + (4 * cq + 2) * 9 + k), __ldg(wg + (4 * cq + 3) * 9 + k));
  }
  w01[9] = w23[9] = make_float2(0.f, 0.f);
  const int64_t left_pos = (stem_rows - row0) * kF1;
  const int n_pos = left_pos < P ? (int)left_pos : P;
  OutT *out = y0 + row0 * (int64_t)(kF1 * kC0) + 4 * cq;
#pragma unroll 2
  for (int i = ph; i < n_pos; i += 4) {
    float2 a = make_float2(0.f, 0.f), b = make_float2(0.f, 0.f);
    const float4 *pp = reinterpret_cast<const float4 *>(&s_pp[i][0]);
#pragma unroll
    for (int m = 0; m < 5; ++m) {
      const float4 q = pp[m];
      ffma2(a, w01[2 * m], make_float2(q.x, q.y));
      ffma2(b, w23[2 * m], make_float2(q.x, q.y));
      ffma2(a, w01[2 * m + 1], make_float2(q.z, q.w));
      ffma2(b, w23[2 * m + 1], make_float2(q.z, q.w));
    }
    const float r = s_r[i];
    const float v[4] = {fmaxf(a.x * r, 0.f), fmaxf(a.y * r, 0.f), fmaxf(b.x * r, 0.f), fmaxf(b.y * r, 0.f)};
    store4(out + (int64_t)i * kC0, v);
  }
}

// ------------------------------------------------------------------ conv0 + LN + ReLU, tensor cores

// The same normalised conv0 as a tcgen05 product, for the bf16 and e4m3
// models: a work item is two stem rows, 128 positions (M = 128), against the
// 128 channels (N = 128). Position r's A row is its 9-sample patch split into
// bf16 parts, (p_hi, p_hi, p_lo) in k = 0..26, and channel c's B row is
// (w_hi, w_lo, w_hi) of its centred, gain-folded taps (built at model
// creation), so the product is p_hi w_hi + p_hi w_lo + p_lo w_hi: the taps
// and the patch to about 16 bits, accumulated in float32 (K = 64, zero beyond
// 27). Thread r builds row r, computes its LayerNorm factor 1/sqrt(p^T C p +
// eps) from the covariance in registers, and after the MMA drains its own
// tensor-memory lane (the 128 channels of its position), scales, applies
// ReLU and stages its 256-byte row in shared memory (128-byte swizzle, as two
// 64-channel halves); two TMA tensor stores write the item's output, one
// contiguous 32 KB block of whole lines. Persistent CTAs, at most four per SM
// (128 tensor-memory columns each); the six mel rows an item reads are copied
// into one of two shared-memory buffers with cp.async while the item before
// it is computed.
namespace {
constexpr uint32_t C0T_TILE = 128 * 128;  // 128 rows x 64 bf16, 128-byte swizzle
constexpr int C0T_MP = 136;               // staged mel row: zero at 3, mel columns 0..127 at 4..131
constexpr size_t C0T_SMEM = 56 * 1024;    // four CTAs per SM at most (4 x 57 KB with the runtime's reserve)
// size bytes from global to shared memory, asynchronously; zeros where !valid
__device__ __forceinline__ void c0_cp_async(void *dst, const void *src, bool valid, int size) {
  const uint32_t d = smem_u32(dst);
  if (size == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(valid ? 16 : 0) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(d), "l"(src), "r"(valid ? 4 : 0) : "memory");
}
__device__ __forceinline__ void c0_cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void c0_cp_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

struct C0Row {  // where a stem row's three mel rows come from
  int64_t base;
  int ti, F;
};
__device__ __forceinline__ C0Row c0_row(const ClipTablesDev &t, int64_t row, int64_t stem_rows) {
  C0Row r{0, -1, 0};
  if (row < stem_rows) {
    const int c = clip_of(t.stem_off, t.n_clips, row);
    r.F = t.frame_off[c + 1] - t.frame_off[c];
    r.ti = (int)(row - t.stem_off[c]) - 2;
    if (r.ti >= (r.F + 1) / 2) r.ti = -1;
    r.base = (int64_t)t.frame_off[c] * kMels;
  }
  return r;
}
}  // namespace

__global__ void __launch_bounds__(128, 4) k_conv0_tc(const __grid_constant__ CUtensorMap tmY, const float *__restrict__ mel,
                                                      bool mel16, const bf16 *__restrict__ bw,
                                                      const float *__restrict__ cov, const ClipTablesDev t,
                                                      int64_t stem_rows, int n_items, unsigned *status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // A, then (once the MMA has read it) the staged channels 0..63; B; the staged channels 64..127
  uint8_t *sA = smem, *sB = smem + C0T_TILE, *sO = smem + 2 * C0T_TILE;
  float *s_mel = reinterpret_cast<float *>(smem + 3 * C0T_TILE);  // [2 buffers][2 stem rows x 3][C0T_MP]
  C0Row *s_row = reinterpret_cast<C0Row *>(s_mel + 2 * 6 * C0T_MP);  // [2 buffers][2]
  uint64_t *bar = reinterpret_cast<uint64_t *>(s_row + 4);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + 1);
  const int tid = threadIdx.x, warp = tid >> 5, r7 = tid & 7;
  // the mel rows of one item into buffer b: 16-byte pieces where the mel
  // array allows (rows are 512 bytes), else 4-byte ones
  auto stage = [&](int b) {
    float *dst = s_mel + b * 6 * C0T_MP;
    const int per_row = mel16 ? 32 : 128, w = mel16 ? 4 : 1;
    for (int i = tid; i < 6 * per_row; i += 128) {
      const int q = i / (3 * per_row), dt = (i / per_row) % 3, sg = i % per_row;
      const C0Row R = s_row[2 * b + q];
      const int tr = 2 * R.ti + dt - 1;
      const bool valid = R.ti >= 0 && tr >= 0 && tr < R.F;
      c0_cp_async(dst + (q * 3 + dt) * C0T_MP + 4 + sg * w, valid ? mel + R.base + (int64_t)tr * kMels + sg * w : mel,
                  valid, 4 * w);
    }
    c0_cp_commit();
  };
  // B (the taps) into shared memory once, swizzled; A's granules 4..7 stay zero
  for (int i = tid; i < 128 * 8; i += 128) {
    const int n = i >> 3, g = i & 7;
    *reinterpret_cast<uint4 *>(sB + n * 128 + ((g ^ (n & 7)) << 4)) = __ldg(reinterpret_cast<const uint4 *>(bw) + i);
  }
#pragma unroll
  for (int g = 4; g < 8; ++g) *reinterpret_cast<uint4 *>(sA + tid * 128 + ((g ^ r7) << 4)) = make_uint4(0, 0, 0, 0);
  for (int i = tid; i < 12; i += 128) s_mel[i * C0T_MP + 3] = 0.f;  // column -1 of every staged row
  float cv[45];  // C_aa and 2 C_ab (b > a)
  {
    int n = 0;
#pragma unroll
    for (int a = 0; a < 9; ++a)
#pragma unroll
      for (int b = a; b < 9; ++b) cv[n++] = (b == a ? 1.0f : 2.0f) * __ldg(cov + a * 9 + b);
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmY);
  }
  if (tid < 2) s_row[tid] = c0_row(t, (int64_t)blockIdx.x * 2 + tid, stem_rows);
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t trow = tmem + ((uint32_t)(32 * warp) << 16);
  const int rr = tid >> 6, f = tid & 63;  // this thread's position: stem row rr of the item, frequency f
  if (blockIdx.x < n_items) stage(0);
  uint32_t phase = 0;
  for (int item = blockIdx.x, it = 0; item < n_items; item += gridDim.x, ++it) {
    const int b = it & 1;
    const int next = item + gridDim.x;
    if (tid < 2 && next < n_items) s_row[2 * (b ^ 1) + tid] = c0_row(t, (int64_t)next * 2 + tid, stem_rows);
    c0_cp_wait_all();
    if (tid == 0) bulk_wait_read<0>();  // the previous item's stores have read A's and sO's staged rows
    __syncthreads();  // this item's rows have landed; the next item's sources are known
    if (next < n_items) stage(b ^ 1);
    const float *m = s_mel + b * 6 * C0T_MP + rr * 3 * C0T_MP + 3 + 2 * f;  // column 2f - 1 of the first row
    float p[9];
#pragma unroll
    for (int dt = 0; dt < 3; ++dt)
#pragma unroll
      for (int df = 0; df < 3; ++df) p[dt * 3 + df] = m[dt * C0T_MP + df];
    float var = 0.f;
    {
      int n = 0;
#pragma unroll
      for (int a = 0; a < 9; ++a) {
        float sa = 0.f;
#pragma unroll
        for (int c = a; c < 9; ++c) sa = fmaf(cv[n++], p[c], sa);
        var = fmaf(p[a], sa, var);
      }
    }
    const float rinv = rsqrtf(fmaxf(var, 0.f) + 1e-6f);
    {
      float kv[32];
#pragma unroll
      for (int k = 0; k < 9; ++k) {
        const float hi = __bfloat162float(__float2bfloat16_rn(p[k]));
        kv[k] = hi;
        kv[9 + k] = hi;
        kv[18 + k] = p[k] - hi;
      }
#pragma unroll
      for (int k = 27; k < 32; ++k) kv[k] = 0.f;
#pragma unroll
      for (int g = 0; g < 4; ++g)
        *reinterpret_cast<uint4 *>(sA + tid * 128 + ((g ^ r7) << 4)) =
            make_uint4(pack_bf16(kv[8 * g], kv[8 * g + 1]), pack_bf16(kv[8 * g + 2], kv[8 * g + 3]),
                       pack_bf16(kv[8 * g + 4], kv[8 * g + 5]), pack_bf16(kv[8 * g + 6], kv[8 * g + 7]));
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t aa = smem_u32(sA), ab = smem_u32(sB);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        tc_mma_bf16(tmem, sw128_desc(aa + k * 32), sw128_desc(ab + k * 32), idesc_bf16_f32(128, 128), k > 0 ? 1u : 0u);
      tc_commit(bar);
    }
    if (!__syncthreads_and(mbar_wait(bar, phase))) {
      if (tid == 0) atomicOr(status, kStatusWaitTimeout);
      break;
    }
    phase ^= 1;
    tc_fence_after();
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {  // channels 32 c .. 32 c + 31: granules 4 (c & 1) .. +3 of a staged half
      uint32_t v[32];
      tmem_ld32(trow + 32 * c, v);
      tmem_ld_wait();
      uint8_t *line = (c < 2 ? sA : sO) + tid * 128;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int g = 4 * (c & 1) + j;
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          w[e] = pack_bf16(fmaxf(__uint_as_float(v[8 * j + 2 * e]) * rinv, 0.f),
                           fmaxf(__uint_as_float(v[8 * j + 2 * e + 1]) * rinv, 0.f));
        *reinterpret_cast<uint4 *>(line + ((g ^ r7) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    tc_fence_before();
    fence_async_smem();
    __syncthreads();  // rows staged; tensor memory is free for the next item
    if (tid == 0) {  // positions beyond the last stem row fall outside the map and are not written
      tma_store_2d(&tmY, sA, 0, item * 128);
      tma_store_2d(&tmY, sO, 64, item * 128);
      bulk_commit();
    }
  }
  if (tid == 0) bulk_wait_all();
  c0_cp_wait_all();  // no copy may still be in flight when the CTA ends
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ------------------------------------------------------------------ conv1, tensor cores (bf16)

namespace {
constexpr int C1_STAGES = 4;
constexpr uint32_t C1_A = 128 * 64 * 2, C1_B = kC1 * 64 * 2, C1_STAGE = C1_A + C1_B;
constexpr size_t C1_SMEM = C1_STAGES * C1_STAGE + 1024 + 256;
constexpr int C1_KB = 9 * kC0 / 64;  // 18 k-blocks of 64
}  // namespace

__global__ void __launch_bounds__(128, 1)
    k_conv1_tc(const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmW,
               const ClipTablesDev t, const float *__restrict__ g1, bf16 *__restrict__ xs, unsigned *status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C1_STAGES * C1_STAGE);
  uint64_t *empty = full + C1_STAGES;
  uint64_t *accb = empty + C1_STAGES;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accb + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  __shared__ float s_g[kC1];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x;
  const int c = clip_of(t.conv1_tile_off, t.n_clips, tile);
  const int tok0 = (tile - t.conv1_tile_off[c]) * kConv1TileTok;
  const int n_tok = t.tok_off[c + 1] - t.tok_off[c];
  const int tp_base = t.stem_off[c] / 2 + tok0;

  if (threadIdx.x < kC1) s_g[threadIdx.x] = g1[threadIdx.x];
  if (threadIdx.x == 0) {
    for (int i = 0; i < C1_STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(accb, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    int issued = 0;
    bool ok = true;
    for (int kb = 0; kb < C1_KB; ++kb) {
      const int s = kb % C1_STAGES;
      const uint32_t ph = (kb / C1_STAGES) & 1;
      if (!mbar_wait(&empty[s], ph ^ 1) || *abort_flag) {
        ok = false;
        break;
      }
      const int tap = kb >> 1, half = kb & 1, dt = tap / 3, df = tap % 3;
      // time row 2t + dt - 1 is stored row base + 2t + dt + 1 = 2 tp + tpar
      const int tpar = (dt == 1) ? 0 : 1, tp = tp_base + (dt == 0 ? 0 : 1);
      // frequency 2f + df - 1 = 2 fp + fpar
      const int fpar = (df == 1) ? 0 : 1, fp = (df == 0) ? -1 : 0;
      uint8_t *sa = smem + s * C1_STAGE;
      mbar_arrive_expect_tx(&full[s], C1_STAGE);
      tma_load_5d(sa, &tmY, half * 64, fpar, fp, tpar, tp, &full[s]);
      tma_load_2d(sa + C1_A, &tmW, kb * 64, 0, &full[s]);
      ++issued;
    }
    if (!ok) {
      atomicOr(status, kStatusWaitTimeout);
      *abort_flag = 1;
    }
    for (int s = 0; s < C1_STAGES; ++s) {
      const int n = issued / C1_STAGES + (s < issued % C1_STAGES ? 1 : 0);
      if (n > 0) mbar_wait(&full[s], (uint32_t)((n - 1) & 1));
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(128, kC1);
    bool ok = true;
    for (int kb = 0; kb < C1_KB; ++kb) {
      const int s = kb % C1_STAGES;
      const uint32_t ph = (kb / C1_STAGES) & 1;
      if (!mbar_wait(&full[s], ph) || *abort_flag) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + s * C1_STAGE), sb = sa + C1_A;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        tc_mma_bf16(tmem, sw128_desc(sa + k * 32), sw128_desc(sb + k * 32), idesc, (kb | k) != 0 ? 1u : 0u);
      tc_commit(&empty[s]);
    }
    if (!ok) {
      atomicOr(status, kStatusWaitTimeout);
      *abort_flag = 1;
    }
    tc_commit(accb);  // arrives when every MMA above has completed (or none was issued)
  }
  __syncwarp();
  // ---- epilogue: row = warp * 32 + lane = (token tok0 + warp, freq lane)
  const bool got = mbar_wait(accb, 0);
  if (__all_sync(0xffffffffu, got)) {
    tc_fence_after();
    uint32_t r[32];
    tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16), r);
    tmem_ld_wait();
    const int tok = tok0 + warp;
    if (tok < n_tok && !*abort_flag) {
      float v[32], mean = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        v[i] = __uint_as_float(r[i]);
        mean += v[i];
      }
      mean *= (1.0f / 32);
      float var = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) var = fmaf(v[i] - mean, v[i] - mean, var);
      const float rs = rsqrtf(var * (1.0f / 32) + 1e-6f);
      uint32_t p[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        p[i] = pack_bf16(fmaxf((v[2 * i] - mean) * rs * s_g[2 * i], 0.f),
                         fmaxf((v[2 * i + 1] - mean) * rs * s_g[2 * i + 1], 0.f));
      uint4 *o = reinterpret_cast<uint4 *>(xs + ((int64_t)t.tok_off[c] + tok) * kHidden + lane * kC1);
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
    }
  } else if (lane == 0) {
    atomicOr(status, kStatusWaitTimeout);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 32);
  }
}

// ------------------------------------------------------------------ conv1, float32 FMA

// One warp per output row (token, freq): lane = output channel.
__global__ void __launch_bounds__(256) k_conv1_f32(const float *__restrict__ y0, const float *__restrict__ w1,
                                                   const float *__restrict__ g1, float *__restrict__ xs,
                                                   const ClipTablesDev t, int64_t T) {
  const int64_t gw = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= T * kF2) return;
  const int64_t tokg = gw / kF2;
  const int f = (int)(gw % kF2);
  const int c = clip_of(t.tok_off, t.n_clips, tokg);
  const int tok = (int)(tokg - t.tok_off[c]);
  const float *w = w1 + (int64_t)lane * 9 * kC0;
  float acc = 0.f;
  for (int dt = 0; dt < 3; ++dt) {
    const int64_t row = (int64_t)t.stem_off[c] + 2 * tok + dt + 1;  // time row 2 tok + dt - 1
    for (int df = 0; df < 3; ++df) {
      const int fr = 2 * f + df - 1;
      if (fr < 0 || fr >= kF1) continue;
      const float *src = y0 + (row * kF1 + fr) * kC0;
      const float *wk = w + (dt * 3 + df) * kC0;
      for (int ci = 0; ci < kC0; ++ci) acc = fmaf(src[ci], wk[ci], acc);
    }
  }
  float s = acc;
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s * (1.0f / 32);
  float d = (acc - mean) * (acc - mean);
  for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
  const float rs = rsqrtf(d * (1.0f / 32) + 1e-6f);
  xs[tokg * kHidden + f * kC1 + lane] = fmaxf((acc - mean) * rs * g1[lane], 0.f);
}

// ------------------------------------------------------------------ launchers

cudaError_t launch_conv0(const ae_model *m, const float *mel, void *y0, const ClipTablesDev &t, int64_t stem_rows,
                         cudaStream_t s) {
  if (stem_rows <= 0) return cudaSuccess;
  const unsigned grid = (unsigned)((stem_rows + kConv0Rows - 1) / kConv0Rows);
  if (m->dtype != AE_F32) {
    static std::atomic<uint64_t> attr{0};
    if (const cudaError_t e = smem_attr(k_conv0_tc, C0T_SMEM, attr)) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t items = (stem_rows + 1) / 2;
    const unsigned g = (unsigned)std::min<int64_t>(items, 4 * (int64_t)(sms > 0 ? sms : 148));
    const bool mel16 = (reinterpret_cast<uintptr_t>(mel) & 15) == 0;
    CUtensorMap tm;  // y0 as [stem rows x 64 positions][128 channels], boxes of 128 positions x 64 channels
    if (!make_tmap_2d_bf16(&tm, y0, kC0, (uint64_t)stem_rows * kF1, kC0 * 2, 64, 128)) return cudaErrorInvalidValue;
    return launch_k(k_conv0_tc, dim3(g), dim3(128), C0T_SMEM, s, tm, mel, mel16, static_cast<const bf16 *>(m->conv0b),
                    (const float *)m->conv0cov, t, stem_rows, (int)items, device_status_word());
  }
  return launch_k(k_conv0<float>, dim3(grid), dim3(128), 0, s, mel, (const float *)m->conv0c,
                  (const float *)m->conv0cov, static_cast<float *>(y0), t, stem_rows);
}

cudaError_t launch_conv1(const ae_model *m, const void *y0, int64_t stem_rows, void *xs, const ClipTablesDev &t,
                         int64_t conv1_tiles, int64_t tokens, cudaStream_t s) {
  if (tokens <= 0) return cudaSuccess;
  if (m->dtype != AE_F32) {
    static std::atomic<uint64_t> attr{0};
    if (const cudaError_t e = smem_attr(k_conv1_tc, C1_SMEM, attr)) return e;
    CUtensorMap tmY;
    if (!make_tmap_stem_y0(&tmY, y0, stem_rows)) return cudaErrorInvalidValue;
    return launch_k(k_conv1_tc, dim3((unsigned)conv1_tiles), dim3(128), C1_SMEM, s, tmY, m->tm_conv1, t,
                    (const float *)m->ln1, static_cast<bf16 *>(xs), device_status_word());
  }
  const int64_t warps = tokens * kF2;
  return launch_k(k_conv1_f32, dim3((unsigned)((warps + 7) / 8)), dim3(256), 0, s, static_cast<const float *>(y0),
                  static_cast<const float *>(m->conv1), (const float *)m->ln1, static_cast<float *>(xs), t, tokens);
}

}  // namespace ae
