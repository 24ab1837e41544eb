// Chunked local attention core (egemma2_audio.rs, AudioTower::attention):
// per head, token t attends to itself and the 11 tokens before it within its
// clip; logits z_d = (q s) . (k_scale k_{t-d}) + (q s) . R[d] with
// s = log2(e)/sqrt(128) * softplus(per_dim_scale), capped as
// cap * tanh(z / cap); natural-exp softmax over the distances; o_t =
// sum_d p_d v_{t-d}.
//
// bf16 kernel (k_attention_tc): both contractions on the tensor cores. The
// 12-wide band of a 128-query tile is a slice of the dense 128 x 144 score
// tile against the tile's keys, so one tcgen05.mma computes all of it (and the
// 12 position terms, as 12 extra B rows); the banded probabilities go back
// through shared memory as the A operand of a second MMA against v. The dense
// tile does 12x the band's multiply-adds, which the tensor cores absorb; what
// is left on the CUDA cores is the softmax of 12 logits per query.
//
// float32 kernel (the float32 model): one query per thread, padded rows.
#include "ae_internal.h"
#include "common.cuh"

namespace ae {

// ------------------------------------------------------------------ tensor-core kernel
//
// Work item = one head x 128 consecutive tokens t0 .. t0+127 (the packed rows
// of any clips); a persistent CTA (one per SM) walks the items. Per item:
//   * TMA loads the q tile [128 x 128], the 144 k rows t0-11 .. t0+132 and the
//     144 v rows (the tensor maps zero-fill rows before 0 and past T);
//   * the eight softmax warps (two per 32-row quarter of the tile, each on
//     half of the 128 head dims) scale q by s and split the product into two bf16
//     tiles, hi = bf16(q s) and lo = bf16(q s - hi), so the score MMA sees q s
//     to about 16 bits (a single bf16 rounding of q s costs more accuracy
//     than everything else in the kernel together); they also write the
//     head's R[d] / k_scale as rows 144..155 under the k rows;
//   * tcgen05.mma (M=128, N=160, K=128, issued for hi and then for lo into
//     the same accumulator) gives S = (q s) [k ; R/k_scale]^T in tensor
//     memory: row r holds q_t.k_{t0-11+c} at column c and the position term
//     q_t.R[d]/k_scale at column 144+d;
//   * in the first warp of each pair, the thread of row r (t = t0 + r) reads
//     columns 32w .. 32w+47 of its warp's
//     32 rows and shifts them left by its lane (five select stages), so that
//     column r + 11 - d, the key t - d, lands at index 11 - d; it caps and
//     softmaxes the 12 logits (distances past the clip start masked by pos) and
//     writes them as bf16 into its row of a banded P [128 x 144] whose other
//     entries stay zero;
//   * tcgen05.mma (M=128, N=128, K=144, v read MN-major) gives O = P V;
//   * both warps of the pair drain their row's half of O (64 dims each), clamp
//     it, and TMA stores leave through a shared-memory box per warp.
// Buffers are single: the next item's q/k load starts when the score MMA has
// read them, its v load when the PV MMA has, so loads overlap the softmax.
namespace {
constexpr int AT_Q = 128;                                 // queries per item
constexpr int AT_KEYS = 144;                              // key rows per item (139 used)
constexpr int AT_BROWS = AT_KEYS + 16;                    // score MMA B rows: keys, R rows, zero rows
constexpr uint32_t AT_Q_REGION = AT_Q * 128;              // 64 head dims of q: 16 KB
constexpr uint32_t AT_KR_REGION = AT_BROWS * 128;         // 20 KB
constexpr uint32_t AT_V_REGION = AT_KEYS * 128;           // 18 KB
constexpr uint32_t AT_P_REGION = AT_Q * 128;              // 64 keys of P: 16 KB
constexpr uint32_t AT_O_BOX = 32 * 128;                   // store box: 32 rows x 64 dims
constexpr uint32_t OFF_Q = 0;                             // hi part of q s (the TMA lands q here)
constexpr uint32_t OFF_QL = OFF_Q + 2 * AT_Q_REGION;      // lo part of q s
constexpr uint32_t OFF_KR = OFF_QL + 2 * AT_Q_REGION;
constexpr uint32_t OFF_V = OFF_KR + 2 * AT_KR_REGION;
constexpr uint32_t OFF_P = OFF_V + 2 * AT_V_REGION;
constexpr uint32_t OFF_O = OFF_P + 3 * AT_P_REGION;
constexpr uint32_t OFF_BAR = OFF_O + 4 * 2 * AT_O_BOX;
constexpr size_t AT_SMEM = OFF_BAR + 1024 + 1024;          // barriers + q scales, alignment slack
constexpr int AT_THREADS = 320;                           // producer warp, MMA warp, 8 softmax warps
constexpr uint32_t AT_TMEM_COLS = 512;                    // S at column 0, O at column 256
constexpr uint32_t AT_O_COL = 256;
constexpr uint32_t AT_QK_BYTES = 2 * AT_Q_REGION + 2 * AT_KEYS * 128;
constexpr uint32_t AT_V_BYTES = 2 * AT_V_REGION;
static_assert(AT_SMEM <= 227 * 1024, "shared memory");
static_assert(OFF_KR % 1024 == 0 && OFF_V % 1024 == 0 && OFF_P % 1024 == 0 && OFF_O % 1024 == 0, "swizzle atoms");
static_assert(AT_KR_REGION % 1024 == 0 && AT_V_REGION % 1024 == 0, "swizzle atoms");
}  // namespace

__global__ void __launch_bounds__(AT_THREADS, 1)
    k_attention_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const float *__restrict__ R, const float *__restrict__ qscale, float k_scale, float cap,
                   const int32_t *__restrict__ pos, int T, float lo, float hi, unsigned *status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem + OFF_Q, *sQL = smem + OFF_QL, *sKR = smem + OFF_KR, *sV = smem + OFF_V, *sP = smem + OFF_P, *sO = smem + OFF_O;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint64_t *qk_full = bars, *v_full = bars + 1, *q_ready = bars + 2, *s_full = bars + 3, *p_full = bars + 4,
           *o_full = bars + 5, *o_empty = bars + 6;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 7);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  float *s_qs = reinterpret_cast<float *>(smem + OFF_BAR + 128);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = ((T + AT_Q - 1) / AT_Q) * kHeads;
  if (threadIdx.x == 0) {
    mbar_init(qk_full, 1);
    mbar_init(v_full, 1);
    mbar_init(q_ready, 256);
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(o_full, 1);
    mbar_init(o_empty, 256);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
  }
  if (threadIdx.x >= 64 && threadIdx.x < 64 + kHeadDim) s_qs[threadIdx.x - 64] = qscale[threadIdx.x - 64];
  if (warp == 1) {
    tmem_alloc(tmem_slot, AT_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    int n_qk = 0, n_v = 0;
    bool ok = true;
    for (int item = blockIdx.x, it = 0; item < n_items; item += gridDim.x, ++it) {
      const int t0 = (item >> 3) * AT_Q, x = (item & 7) * kHeadDim;
      if (it > 0 && !mbar_wait(s_full, (it - 1) & 1)) { ok = false; break; }  // q/k buffers read
      if (*abort_flag) break;
      mbar_arrive_expect_tx(qk_full, AT_QK_BYTES);
      tma_load_2d(sQ, &tmQ, x, t0, qk_full);
      tma_load_2d(sQ + AT_Q_REGION, &tmQ, x + 64, t0, qk_full);
      tma_load_2d(sKR, &tmK, x, t0 - (kLeft - 1), qk_full);
      tma_load_2d(sKR + AT_KR_REGION, &tmK, x + 64, t0 - (kLeft - 1), qk_full);
      ++n_qk;
      if (it > 0 && !mbar_wait(o_full, (it - 1) & 1)) { ok = false; break; }  // v buffer read
      if (*abort_flag) break;
      mbar_arrive_expect_tx(v_full, AT_V_BYTES);
      tma_load_2d(sV, &tmV, x, t0 - (kLeft - 1), v_full);
      tma_load_2d(sV + AT_V_REGION, &tmV, x + 64, t0 - (kLeft - 1), v_full);
      ++n_v;
    }
    if (!ok) {
      atomicOr(status, kStatusWaitTimeout);
      *abort_flag = 1;
    }
    // every load issued must land before the CTA may end
    if (n_qk > 0) mbar_wait(qk_full, (n_qk - 1) & 1);
    if (n_v > 0) mbar_wait(v_full, (n_v - 1) & 1);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    constexpr uint32_t idesc_s = idesc_bf16_f32(AT_Q, AT_BROWS);
    constexpr uint32_t idesc_o = idesc_bf16_f32_bmn(AT_Q, kHeadDim);
    const uint32_t aq = smem_u32(sQ), aql = smem_u32(sQL), akr = smem_u32(sKR), ap = smem_u32(sP),
                   av = smem_u32(sV);
    bool ok = true;
    for (int item = blockIdx.x, it = 0; item < n_items; item += gridDim.x, ++it) {
      if (!mbar_wait(q_ready, it & 1) || *abort_flag) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < 2 * kHeadDim / 16; ++ks) {
        const int kk = ks & 7;
        tc_mma_bf16(tmem, sw128_desc((ks < 8 ? aq : aql) + (kk >> 2) * AT_Q_REGION + (kk & 3) * 32),
                    sw128_desc(akr + (kk >> 2) * AT_KR_REGION + (kk & 3) * 32), idesc_s, ks > 0 ? 1u : 0u);
      }
      tc_commit(s_full);
      if (!mbar_wait(p_full, it & 1) || !mbar_wait(v_full, it & 1) ||
          (it > 0 && !mbar_wait(o_empty, (it - 1) & 1)) || *abort_flag) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < AT_KEYS / 16; ++ks)
        tc_mma_bf16(tmem + AT_O_COL, sw128_desc(ap + (ks >> 2) * AT_P_REGION + (ks & 3) * 32),
                    sw128_desc_mn(av + ks * 2048, AT_V_REGION), idesc_o, ks > 0 ? 1u : 0u);
      tc_commit(o_full);
    }
    if (!ok) {
      atomicOr(status, kStatusWaitTimeout);
      *abort_flag = 1;
    }
  } else if (warp >= 2) {
    // ---------------- softmax warps: two per TMEM lane quarter, thread = tile row r;
    // warp half hw takes head dims 64 hw .. +63 of q and of the output, and the
    // hw = 0 warps the softmax of their rows
    const int qw = warp & 3, hw = (warp - 2) >> 2, r = 32 * qw + lane, r7 = r & 7, tid = threadIdx.x - 64;
    uint8_t *box = sO + (qw * 2 + hw) * AT_O_BOX;
    // P outside the band and the zero rows 156..159 of the B operand stay zero
    for (int i = tid; i < (int)(3 * AT_P_REGION / 16); i += 256) reinterpret_cast<uint4 *>(sP)[i] = make_uint4(0, 0, 0, 0);
    if (tid < 64) {
      const int rr = AT_KEYS + 12 + (tid >> 4), g = tid & 15;
      *reinterpret_cast<uint4 *>(sKR + (g >> 3) * AT_KR_REGION + rr * 128 + (((g & 7) ^ (rr & 7)) << 4)) =
          make_uint4(0, 0, 0, 0);
    }
    const float zs = k_scale / cap, inv_ks = 1.0f / k_scale;
    const uint32_t trow = tmem + ((uint32_t)(32 * qw) << 16);
    bool ok = true;
    for (int item = blockIdx.x, it = 0; item < n_items; item += gridDim.x, ++it) {
      const int t0 = (item >> 3) * AT_Q, h = item & 7, t = t0 + r;
      // ---- q s as hi + lo bf16 tiles, and R / k_scale under the k rows
      if (!__all_sync(0xffffffffu, mbar_wait(qk_full, it & 1))) { ok = false; break; }
#pragma unroll 4
      for (int j = 8 * hw; j < 8 * hw + 8; ++j) {
        const uint32_t off = (j >> 3) * AT_Q_REGION + r * 128 + (((j & 7) ^ r7) << 4);
        const uint4 w = *reinterpret_cast<const uint4 *>(sQ + off);
        const float4 s0 = reinterpret_cast<const float4 *>(s_qs)[2 * j], s1 = reinterpret_cast<const float4 *>(s_qs)[2 * j + 1];
        const float f[8] = {bf16lo(w.x) * s0.x, bf16hi(w.x) * s0.y, bf16lo(w.y) * s0.z, bf16hi(w.y) * s0.w,
                            bf16lo(w.z) * s1.x, bf16hi(w.z) * s1.y, bf16lo(w.w) * s1.z, bf16hi(w.w) * s1.w};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          hi[e] = pack_bf16(f[2 * e], f[2 * e + 1]);
          lo[e] = pack_bf16(f[2 * e] - bf16lo(hi[e]), f[2 * e + 1] - bf16hi(hi[e]));
        }
        *reinterpret_cast<uint4 *>(sQ + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4 *>(sQL + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      for (int rr = tid >> 4; rr < kLeft; rr += 16) {
        const int g = tid & 15, row = AT_KEYS + rr;
        const float4 a = *reinterpret_cast<const float4 *>(R + (size_t)rr * kHidden + h * kHeadDim + g * 8);
        const float4 b = *reinterpret_cast<const float4 *>(R + (size_t)rr * kHidden + h * kHeadDim + g * 8 + 4);
        *reinterpret_cast<uint4 *>(sKR + (g >> 3) * AT_KR_REGION + row * 128 + (((g & 7) ^ (row & 7)) << 4)) =
            make_uint4(pack_bf16(a.x * inv_ks, a.y * inv_ks), pack_bf16(a.z * inv_ks, a.w * inv_ks),
                       pack_bf16(b.x * inv_ks, b.y * inv_ks), pack_bf16(b.z * inv_ks, b.w * inv_ks));
      }
      fence_async_smem();
      mbar_arrive(q_ready);
      // ---- scores -> probabilities -> banded P (warps of half 0)
      if (hw == 0) {
      if (!__all_sync(0xffffffffu, mbar_wait(s_full, it & 1))) { ok = false; break; }
      tc_fence_after();
      uint32_t a32[32], a16[16], u16[16];
      tmem_ld32(trow + 32 * qw, a32);
      tmem_ld16(trow + 32 * qw + 32, a16);
      tmem_ld16(trow + AT_KEYS, u16);
      tmem_ld_wait();
      float sc[48];
#pragma unroll
      for (int i = 0; i < 32; ++i) sc[i] = __uint_as_float(a32[i]);
#pragma unroll
      for (int i = 0; i < 16; ++i) sc[32 + i] = __uint_as_float(a16[i]);
      // shift left by lane: afterwards sc[i] holds column r + i
#pragma unroll
      for (int i = 0; i < 42; ++i) sc[i] = (lane & 1) ? sc[i + 1] : sc[i];
#pragma unroll
      for (int i = 0; i < 40; ++i) sc[i] = (lane & 2) ? sc[i + 2] : sc[i];
#pragma unroll
      for (int i = 0; i < 36; ++i) sc[i] = (lane & 4) ? sc[i + 4] : sc[i];
#pragma unroll
      for (int i = 0; i < 28; ++i) sc[i] = (lane & 8) ? sc[i + 8] : sc[i];
#pragma unroll
      for (int i = 0; i < 12; ++i) sc[i] = (lane & 16) ? sc[i + 16] : sc[i];
      const int span = t < T ? min(pos[t] + 1, kLeft) : 0;
      float pr[kLeft], mx = -INFINITY;
#pragma unroll
      for (int d = 0; d < kLeft; ++d) {
        const float z = cap * tanhf(zs * (sc[kLeft - 1 - d] + __uint_as_float(u16[d])));
        pr[d] = d < span ? z : -INFINITY;
        mx = fmaxf(mx, pr[d]);
      }
      float den = 0.f;
#pragma unroll
      for (int d = 0; d < kLeft; ++d) {
        pr[d] = d < span ? __expf(pr[d] - mx) : 0.f;
        den += pr[d];
      }
      const float rd = span > 0 ? 1.0f / den : 0.f;
      // band of row r: column r + i holds p_{11-i}; written as the three
      // granules (8 columns each) from column r & ~7, zeros around the band
      float a[24];
#pragma unroll
      for (int j = 0; j < 24; ++j) a[j] = j < kLeft ? pr[kLeft - 1 - j] * rd : 0.f;
#pragma unroll
      for (int j = 23; j >= 0; --j) a[j] = (r7 & 4) ? (j >= 4 ? a[j - 4] : 0.f) : a[j];
#pragma unroll
      for (int j = 23; j >= 0; --j) a[j] = (r7 & 2) ? (j >= 2 ? a[j - 2] : 0.f) : a[j];
#pragma unroll
      for (int j = 23; j >= 0; --j) a[j] = (r7 & 1) ? (j >= 1 ? a[j - 1] : 0.f) : a[j];
#pragma unroll
      for (int gg = 0; gg < 3; ++gg) {
        const int G = (r >> 3) + gg;
        *reinterpret_cast<uint4 *>(sP + (G >> 3) * AT_P_REGION + r * 128 + (((G & 7) ^ r7) << 4)) =
            make_uint4(pack_bf16(a[8 * gg], a[8 * gg + 1]), pack_bf16(a[8 * gg + 2], a[8 * gg + 3]),
                       pack_bf16(a[8 * gg + 4], a[8 * gg + 5]), pack_bf16(a[8 * gg + 6], a[8 * gg + 7]));
      }
      tc_fence_before();
      fence_async_smem();
      mbar_arrive(p_full);
      }
      // ---- O rows out: head dims 64 hw .. +63
      if (!__all_sync(0xffffffffu, mbar_wait(o_full, it & 1))) { ok = false; break; }
      tc_fence_after();
      if (lane == 0) bulk_wait_read<0>();  // the previous item's stores are done with the boxes
      __syncwarp();
#pragma unroll 1
      for (int c = 2 * hw; c < 2 * hw + 2; ++c) {
        uint32_t o[32];
        tmem_ld32(trow + AT_O_COL + 32 * c, o);
        tmem_ld_wait();
        uint8_t *line = box + lane * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int g = (c & 1) * 4 + j;
          *reinterpret_cast<uint4 *>(line + ((g ^ (lane & 7)) << 4)) = make_uint4(
              pack_bf16(clampf(__uint_as_float(o[8 * j]), lo, hi), clampf(__uint_as_float(o[8 * j + 1]), lo, hi)),
              pack_bf16(clampf(__uint_as_float(o[8 * j + 2]), lo, hi), clampf(__uint_as_float(o[8 * j + 3]), lo, hi)),
              pack_bf16(clampf(__uint_as_float(o[8 * j + 4]), lo, hi), clampf(__uint_as_float(o[8 * j + 5]), lo, hi)),
              pack_bf16(clampf(__uint_as_float(o[8 * j + 6]), lo, hi), clampf(__uint_as_float(o[8 * j + 7]), lo, hi)));
        }
      }
      tc_fence_before();
      mbar_arrive(o_empty);
      fence_async_smem();
      __syncwarp();
      if (lane == 0 && t0 + 32 * qw < T) {
        tma_store_2d(&tmO, box, h * kHeadDim + 64 * hw, t0 + 32 * qw);
        bulk_commit();
      }
    }
    if (lane == 0) bulk_wait_all();
    if (!ok && lane == 0) {
      atomicOr(status, kStatusWaitTimeout);
      *abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, AT_TMEM_COLS);
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
    static std::atomic<uint64_t> attr{0};
    if (const cudaError_t e = smem_attr(k_attention_tc, AT_SMEM, attr)) return e;
    CUtensorMap tq, tk, tv, to;
    const uint64_t rb = (uint64_t)ld * 2, ob = (uint64_t)ld_out * 2;
    if (!make_tmap_2d_bf16(&tq, q, kHidden, (uint64_t)T, rb, 64, AT_Q) ||
        !make_tmap_2d_bf16(&tk, k, kHidden, (uint64_t)T, rb, 64, AT_KEYS) ||
        !make_tmap_2d_bf16(&tv, v, kHidden, (uint64_t)T, rb, 64, AT_KEYS) ||
        !make_tmap_2d_bf16(&to, out, kHidden, (uint64_t)T, ob, 64, 32))
      return cudaErrorInvalidValue;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t items = (T + AT_Q - 1) / AT_Q * kHeads;
    const unsigned grid = (unsigned)(items < sms ? items : (sms > 0 ? sms : 1));
    return launch_k(k_attention_tc, dim3(grid), dim3(AT_THREADS), AT_SMEM, s, tq, tk, tv, to, R, qscale, k_scale,
                    cap, pos, (int)T, lo, hi, device_status_word());
  }
  const size_t smem = (2 * (size_t)kRows * kPitchF + kLeft * kHeadDim + kHeadDim) * sizeof(float);
  static std::atomic<uint64_t> attr{0};
  if (const cudaError_t e = smem_attr(k_attention_f32, smem, attr)) return e;
  dim3 grid((unsigned)((T + kTQ - 1) / kTQ), kHeads);
  return launch_k(k_attention_f32, grid, dim3(kTQ), smem, s, static_cast<const float *>(q),
                  static_cast<const float *>(k), static_cast<const float *>(v), ld, R, qscale, k_scale, cap, pos, T,
                  static_cast<float *>(out), ld_out, lo, hi);
}

}  // namespace ae
