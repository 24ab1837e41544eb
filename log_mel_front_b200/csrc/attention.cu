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
//   * TMA loads the q tile [128 x 128] and the 144 k rows t0-11 .. t0+132 into
//     one of two shared-memory stages, and the 144 v rows into one buffer (the
//     tensor maps zero-fill rows before 0 and past T);
//   * four q warps (one per 32-row quarter) scale q by s and split the product
//     into two bf16 parts, hi = bf16(q s), written over the q tile, and lo =
//     bf16(q s - hi), written to a tile of its own, so the score MMA sees q s
//     to about 16 bits (a single bf16 rounding of q s costs more accuracy than
//     everything else in the kernel together); they also write the head's
//     R[d] / k_scale as rows 144..155 under the k rows;
//   * tcgen05.mma (M=128, N=160, K=128 for hi and again for lo into the same
//     accumulator, both operands in shared memory) gives S = (q s)
//     [k ; R/k_scale]^T in tensor memory: row r holds q_t.k_{t0-11+c} at
//     column c and the position term q_t.R[d]/k_scale at column 144+d;
//   * four softmax warps: the thread of row r (t = t0 + r) reads columns
//     32w .. 32w+47 of its warp's 32 rows and shifts them left by its lane
//     (five select stages), so that column r + 11 - d, the key t - d, lands at
//     index 11 - d; it caps (cap tanh(z / cap), tanh from the exponential) and
//     softmaxes the 12 logits (distances past the clip start masked by pos) and
//     writes its row of the banded P [128 x 160] (bf16) into tensor memory: the
//     64-key window of its warp, the band shifted right by its lane, zeros
//     around it (the columns outside every warp's window stay zero from the
//     start);
//   * tcgen05.mma (A = P from tensor memory, M=128, N=128, K=144, v read
//     MN-major) gives O = P V in one of two tensor-memory accumulators;
//   * the softmax warps (head dims 64..127) and the q warps (0..63) drain O,
//     clamp it and store it from registers, whole 32-byte sectors per row
//     where the output's alignment allows.
// The stages overlap across items: the q warps split item i+1 as soon as the
// score MMA of item i has read the previous split, while the softmax warps
// work on item i; the MMA warp issues item i's P V as soon as its P is
// written, then item i+1's score MMA; item i's O is drained while item i+1
// runs. A stage's q/k are reloaded once the score MMA that read them
// completes, v once the P V MMA has.
namespace {
constexpr int AT_Q = 128;                                  // queries per item
constexpr int AT_KEYS = 144;                               // key rows per item (139 used)
constexpr int AT_BROWS = AT_KEYS + 16;                     // score MMA B rows: keys, R rows, zero rows
constexpr uint32_t AT_Q_REGION = AT_Q * 128;               // 64 head dims of q: 16 KB
constexpr uint32_t AT_KR_REGION = AT_BROWS * 128;          // 20 KB
constexpr uint32_t AT_V_REGION = AT_KEYS * 128;            // 18 KB
constexpr uint32_t OFF_Q = 0;                              // offsets within a stage: q (then hi), k rows
constexpr uint32_t OFF_KR = OFF_Q + 2 * AT_Q_REGION;
constexpr uint32_t AT_STAGE = OFF_KR + 2 * AT_KR_REGION;   // 72 KB
constexpr uint32_t OFF_QL = 2 * AT_STAGE;                  // lo part of q s
constexpr uint32_t OFF_V = OFF_QL + 2 * AT_Q_REGION;
constexpr uint32_t OFF_BAR = OFF_V + 2 * AT_V_REGION;
constexpr size_t AT_SMEM = OFF_BAR + 1024 + 1024;          // barriers + q scales, alignment slack
constexpr int AT_THREADS = 320;                            // producer, MMA, 4 softmax warps, 4 q warps
constexpr int AT_DRAIN_THREADS = 256;                      // both warp groups drain half of O
constexpr uint32_t AT_TMEM_COLS = 512;
constexpr uint32_t COL_S = 0;                              // scores, 160 f32 columns
constexpr uint32_t COL_P = 160;                            // banded P, 160 bf16 = 80 columns
constexpr uint32_t COL_O = 256;                            // two P V accumulators, 128 f32 columns each
constexpr uint32_t AT_QK_BYTES = 2 * AT_Q_REGION + 2 * AT_KEYS * 128;
constexpr uint32_t AT_V_BYTES = 2 * AT_V_REGION;
static_assert(AT_SMEM <= 227 * 1024, "shared memory");
static_assert(AT_STAGE % 1024 == 0 && OFF_KR % 1024 == 0 && OFF_QL % 1024 == 0 && OFF_V % 1024 == 0, "swizzle atoms");
static_assert(AT_KR_REGION % 1024 == 0 && AT_V_REGION % 1024 == 0, "swizzle atoms");
static_assert(COL_P + 80 <= COL_O && COL_O + 256 <= AT_TMEM_COLS, "tensor-memory map");

// D[tmem] (+)= A[tmem] * B[smem]^T, bf16 inputs, f32 accumulate: A's row m is
// tensor-memory lane m, two bf16 per 32-bit column (the lower k in the low
// half), K = 16 per instruction over 8 columns. One thread issues.
__device__ __forceinline__ void at_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 (16) consecutive 32-bit columns from registers into tensor
// memory (thread i of the warp writes row lane-base + i), and the wait for them.
__device__ __forceinline__ void at_tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void at_tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void at_tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void at_st32B(void *p, uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint32_t e,
                                         uint32_t f, uint32_t g, uint32_t h) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d),
               "r"(e), "r"(f), "r"(g), "r"(h)
               : "memory");
}
__device__ __forceinline__ float at_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float at_rcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
}  // namespace

__global__ void __launch_bounds__(AT_THREADS, 1)
    k_attention_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, bf16 *__restrict__ out, int64_t ld_out, bool out_v8,
                   const float *__restrict__ R, const float *__restrict__ qscale, float k_scale, float cap,
                   const int32_t *__restrict__ pos, int T, float lo, float hi, unsigned *status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint64_t *qk_full = bars, *qk_free = bars + 2;                      // per stage
  uint64_t *o_full = bars + 4, *o_empty = bars + 6;                   // per accumulator
  uint64_t *v_full = bars + 8, *v_free = bars + 9, *q_ready = bars + 10, *s_full = bars + 11, *s_free = bars + 12,
           *p_full = bars + 13;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 14);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  float *s_qs = reinterpret_cast<float *>(smem + OFF_BAR + 128);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = ((T + AT_Q - 1) / AT_Q) * kHeads;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(bars + i, 1);   // qk_full, qk_free
    for (int i = 0; i < 2; ++i) {
      mbar_init(&o_full[i], 1);
      mbar_init(&o_empty[i], AT_DRAIN_THREADS);
    }
    mbar_init(v_full, 1);
    mbar_init(v_free, 1);
    mbar_init(q_ready, 128);
    mbar_init(s_full, 1);
    mbar_init(s_free, 128);
    mbar_init(p_full, 128);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
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
  // O rows of item j (the j-th of this CTA), head dims 64 hw .. 64 hw + 63, out by
  // the warp of lane quarter warp & 3
  auto drain_half = [&](int j, int jitem, int hw) -> bool {
    const int b = j & 1;
    if (!__all_sync(0xffffffffu, mbar_wait(&o_full[b], (j >> 1) & 1))) return false;
    tc_fence_after();
    const int qw = warp & 3, r = 32 * qw + lane;
    const uint32_t trow = tmem + ((uint32_t)(32 * qw) << 16);
    const int t = (jitem >> 3) * AT_Q + r, h = jitem & 7;
    bf16 *orow = out + (int64_t)t * ld_out + h * kHeadDim + 64 * hw;
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      uint32_t o[32];
      tmem_ld32(trow + COL_O + 128 * b + 64 * hw + 32 * c, o);
      tmem_ld_wait();
      uint32_t w[16];
#pragma unroll
      for (int j2 = 0; j2 < 16; ++j2)
        w[j2] = pack_bf16(clampf(__uint_as_float(o[2 * j2]), lo, hi), clampf(__uint_as_float(o[2 * j2 + 1]), lo, hi));
      if (t < T) {
        if (out_v8) {
          at_st32B(orow + 32 * c, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
          at_st32B(orow + 32 * c + 16, w[8], w[9], w[10], w[11], w[12], w[13], w[14], w[15]);
        } else {
#pragma unroll
          for (int g = 0; g < 4; ++g)
            *reinterpret_cast<uint4 *>(orow + 32 * c + 8 * g) = make_uint4(w[4 * g], w[4 * g + 1], w[4 * g + 2], w[4 * g + 3]);
        }
      }
    }
    tc_fence_before();
    mbar_arrive(&o_empty[b]);
    return true;
  };

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer: q, k of item i into stage i & 1 once the
    // score MMA of item i - 2 has read it; v of item i once the P V of item i - 1 has
    int n_qk = 0, n_v = 0;
    bool ok = true;
    for (int item = blockIdx.x, it = 0; item < n_items; item += gridDim.x, ++it) {
      const int st = it & 1, u = it >> 1;
      uint8_t *stage = smem + st * AT_STAGE;
      const int t0 = (item >> 3) * AT_Q, x = (item & 7) * kHeadDim;
      if (u > 0 && !mbar_wait(&qk_free[st], (u - 1) & 1)) { ok = false; break; }
      if (*abort_flag) break;
      mbar_arrive_expect_tx(&qk_full[st], AT_QK_BYTES);
      tma_load_2d(stage + OFF_Q, &tmQ, x, t0, &qk_full[st]);
      tma_load_2d(stage + OFF_Q + AT_Q_REGION, &tmQ, x + 64, t0, &qk_full[st]);
      tma_load_2d(stage + OFF_KR, &tmK, x, t0 - (kLeft - 1), &qk_full[st]);
      tma_load_2d(stage + OFF_KR + AT_KR_REGION, &tmK, x + 64, t0 - (kLeft - 1), &qk_full[st]);
      ++n_qk;
      if (it > 0 && !mbar_wait(v_free, (it - 1) & 1)) { ok = false; break; }
      if (*abort_flag) break;
      mbar_arrive_expect_tx(v_full, AT_V_BYTES);
      tma_load_2d(smem + OFF_V, &tmV, x, t0 - (kLeft - 1), v_full);
      tma_load_2d(smem + OFF_V + AT_V_REGION, &tmV, x + 64, t0 - (kLeft - 1), v_full);
      ++n_v;
    }
    if (!ok) {
      atomicOr(status, kStatusWaitTimeout);
      *abort_flag = 1;
    }
    // every load issued must land before the CTA may end
#pragma unroll
    for (int st = 0; st < 2; ++st) {
      const int uq = (n_qk + 1 - st) / 2;  // uses of stage st
      if (uq > 0) mbar_wait(&qk_full[st], (uq - 1) & 1);
    }
    if (n_v > 0) mbar_wait(v_full, (n_v - 1) & 1);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer: the score MMA of item i, then (once P is written) its P V MMA
    constexpr uint32_t idesc_s = idesc_bf16_f32(AT_Q, AT_BROWS);
    constexpr uint32_t idesc_o = idesc_bf16_f32_bmn(AT_Q, kHeadDim);
    const uint32_t aql = smem_u32(smem + OFF_QL), av = smem_u32(smem + OFF_V);
    bool ok = true;
    for (int item = blockIdx.x, it = 0; item < n_items; item += gridDim.x, ++it) {
      const int st = it & 1, b = it & 1;
      const uint32_t aq = smem_u32(smem + st * AT_STAGE + OFF_Q), akr = smem_u32(smem + st * AT_STAGE + OFF_KR);
      // q s of this item is split, and the softmax has read the previous scores
      if (!mbar_wait(q_ready, it & 1) || (it > 0 && !mbar_wait(s_free, (it - 1) & 1)) || *abort_flag) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < 2 * kHeadDim / 16; ++ks) {
        const int kk = ks & 7;  // hi part for ks < 8, lo part after: the same k rows
        tc_mma_bf16(tmem + COL_S, sw128_desc((ks < 8 ? aq : aql) + (kk >> 2) * AT_Q_REGION + (kk & 3) * 32),
                    sw128_desc(akr + (kk >> 2) * AT_KR_REGION + (kk & 3) * 32), idesc_s, ks > 0 ? 1u : 0u);
      }
      tc_commit(&qk_free[st]);
      tc_commit(s_full);
      // P is written, v has landed, and this accumulator's previous item is drained
      if (!mbar_wait(p_full, it & 1) || !mbar_wait(v_full, it & 1) ||
          (it >= 2 && !mbar_wait(&o_empty[b], ((it >> 1) - 1) & 1)) || *abort_flag) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < AT_KEYS / 16; ++ks)
        at_mma_ts(tmem + COL_O + 128 * b, tmem + COL_P + 8 * ks, sw128_desc_mn(av + ks * 2048, AT_V_REGION),
                  idesc_o, ks > 0 ? 1u : 0u);
      tc_commit(v_free);
      tc_commit(&o_full[b]);
    }
    if (!ok) {
      atomicOr(status, kStatusWaitTimeout);
      *abort_flag = 1;
    }
  } else if (warp >= 2 && warp < 6) {
    // ---------------- softmax warps: TMEM lane quarter qw, thread = tile row r
    const int qw = warp & 3, r = 32 * qw + lane;
    const uint32_t trow = tmem + ((uint32_t)(32 * qw) << 16);
    {  // P's columns outside the warps' windows stay zero
      uint32_t z[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) z[i] = 0u;
      at_tmem_st32(trow + COL_P, z);
      at_tmem_st32(trow + COL_P + 32, z);
      uint32_t z16[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) z16[i] = 0u;
      at_tmem_st16(trow + COL_P + 64, z16);
      at_tmem_st_wait();
    }
    // z = cap tanh(zs x) = cap (1 - 2 / (1 + 2^(e2 x))), e2 = 2 log2(e) zs: the
    // exponential and reciprocal to about 2^-22 give z to about 1e-6 cap
    const float zs = k_scale / cap, e2 = 2.0f * 1.4426950408889634f * zs;
    bool ok = true;
    for (int item = blockIdx.x, it = 0; item < n_items; item += gridDim.x, ++it) {
      const int t = (item >> 3) * AT_Q + r;
      const int pos_t = t < T ? pos[t] : -1;  // issued before the wait, used after it
      if (!__all_sync(0xffffffffu, mbar_wait(s_full, it & 1))) { ok = false; break; }
      tc_fence_after();
      uint32_t a32[32], a16[16], u16[16];
      tmem_ld32(trow + COL_S + 32 * qw, a32);
      tmem_ld16(trow + COL_S + 32 * qw + 32, a16);
      tmem_ld16(trow + COL_S + AT_KEYS, u16);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(s_free);  // the scores are in registers
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
      const int span = min(pos_t + 1, kLeft);
      float pr[kLeft], mx = -INFINITY;
#pragma unroll
      for (int d = 0; d < kLeft; ++d) {
        const float x = sc[kLeft - 1 - d] + __uint_as_float(u16[d]);
        const float z = cap * fmaf(-2.0f, at_rcp(1.0f + at_ex2(e2 * x)), 1.0f);
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
      // the warp's window holds keys 32 qw .. 32 qw + 63 (32 columns of bf16
      // pairs); row r's band, key r + i = p_{11-i}, sits at window index
      // lane + i: shift by the lane's low bit in floats, pair up, then shift
      // the pairs by lane >> 1
      float c[14];
#pragma unroll
      for (int j = 0; j < 14; ++j) {
        const float cur = j < kLeft ? pr[kLeft - 1 - j] * rd : 0.f;
        const float prev = (j >= 1 && j - 1 < kLeft) ? pr[kLeft - j] * rd : 0.f;
        c[j] = (lane & 1) ? prev : cur;
      }
      uint32_t w[22];
#pragma unroll
      for (int k = 0; k < 22; ++k) w[k] = k < 7 ? pack_bf16(c[2 * k], c[2 * k + 1]) : 0u;
      const int hs = lane >> 1;
#pragma unroll
      for (int k = 21; k >= 0; --k) w[k] = (hs & 8) ? (k >= 8 ? w[k - 8] : 0u) : w[k];
#pragma unroll
      for (int k = 21; k >= 0; --k) w[k] = (hs & 4) ? (k >= 4 ? w[k - 4] : 0u) : w[k];
#pragma unroll
      for (int k = 21; k >= 0; --k) w[k] = (hs & 2) ? (k >= 2 ? w[k - 2] : 0u) : w[k];
#pragma unroll
      for (int k = 21; k >= 0; --k) w[k] = (hs & 1) ? (k >= 1 ? w[k - 1] : 0u) : w[k];
      uint32_t pw[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) pw[k] = k < 22 ? w[k] : 0u;
      // the previous item's P V has read P: these warps waited for it before draining it
      at_tmem_st32(trow + COL_P + 16 * qw, pw);
      at_tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);
      if (!drain_half(it, item, 1)) { ok = false; break; }
    }
    if (!ok && lane == 0) {
      atomicOr(status, kStatusWaitTimeout);
      *abort_flag = 1;
    }
  } else if (warp >= 6) {
    // ---------------- q warps: split item i's q s (hi over q, lo into its tile), then drain item i - 1
    const int qw = warp & 3, r = 32 * qw + lane, r7 = r & 7, tid = threadIdx.x - 192;
    // rows 156..159 of both stages' B operand stay zero
    {
      const int s = tid >> 6, rr = AT_KEYS + 12 + ((tid >> 4) & 3), g = tid & 15;
      *reinterpret_cast<uint4 *>(smem + s * AT_STAGE + OFF_KR + (g >> 3) * AT_KR_REGION + rr * 128 +
                                 (((g & 7) ^ (rr & 7)) << 4)) = make_uint4(0, 0, 0, 0);
    }
    uint8_t *sQL = smem + OFF_QL;
    const float inv_ks = 1.0f / k_scale;
    bool ok = true;
    int it = 0, prev_item = -1;
    int r_head0 = -1, r_head1 = -1;  // the head whose R rows each stage holds (one head per stage
                                     // when the grid is a multiple of 4, as on 148 SMs)
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it) {
      const int st = it & 1, u = it >> 1;
      uint8_t *sQ = smem + st * AT_STAGE + OFF_Q, *sKR = smem + st * AT_STAGE + OFF_KR;
      const int h = item & 7;
      // this item's q and k have landed, and the previous score MMA has read the lo tile
      if (!__all_sync(0xffffffffu, mbar_wait(&qk_full[st], u & 1)) ||
          (it > 0 && !__all_sync(0xffffffffu, mbar_wait(s_full, (it - 1) & 1)))) {
        ok = false;
        break;
      }
#pragma unroll 4
      for (int j = 0; j < 16; ++j) {  // head dims 8 j .. 8 j + 7 of row r
        const uint32_t off = (j >> 3) * AT_Q_REGION + r * 128 + (((j & 7) ^ r7) << 4);
        const uint4 wv = *reinterpret_cast<const uint4 *>(sQ + off);
        const float4 s0 = reinterpret_cast<const float4 *>(s_qs)[2 * j], s1 = reinterpret_cast<const float4 *>(s_qs)[2 * j + 1];
        const float f[8] = {bf16lo(wv.x) * s0.x, bf16hi(wv.x) * s0.y, bf16lo(wv.y) * s0.z, bf16hi(wv.y) * s0.w,
                            bf16lo(wv.z) * s1.x, bf16hi(wv.z) * s1.y, bf16lo(wv.w) * s1.z, bf16hi(wv.w) * s1.w};
        uint32_t hv[4], lv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          hv[e] = pack_bf16(f[2 * e], f[2 * e + 1]);
          lv[e] = pack_bf16(f[2 * e] - bf16lo(hv[e]), f[2 * e + 1] - bf16hi(hv[e]));
        }
        *reinterpret_cast<uint4 *>(sQ + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        *reinterpret_cast<uint4 *>(sQL + off) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
      }
      if ((st ? r_head1 : r_head0) != h) {  // the TMA never writes rows 144.., so they keep the stage's last head
        if (st) r_head1 = h; else r_head0 = h;
        for (int rr = tid >> 4; rr < kLeft; rr += 8) {
          const int g = tid & 15, row = AT_KEYS + rr;
          const float4 a = *reinterpret_cast<const float4 *>(R + (size_t)rr * kHidden + h * kHeadDim + g * 8);
          const float4 b = *reinterpret_cast<const float4 *>(R + (size_t)rr * kHidden + h * kHeadDim + g * 8 + 4);
          *reinterpret_cast<uint4 *>(sKR + (g >> 3) * AT_KR_REGION + row * 128 + (((g & 7) ^ (row & 7)) << 4)) =
              make_uint4(pack_bf16(a.x * inv_ks, a.y * inv_ks), pack_bf16(a.z * inv_ks, a.w * inv_ks),
                         pack_bf16(b.x * inv_ks, b.y * inv_ks), pack_bf16(b.z * inv_ks, b.w * inv_ks));
        }
      }
      fence_async_smem();
      mbar_arrive(q_ready);
      if (it > 0 && !drain_half(it - 1, prev_item, 0)) { ok = false; break; }
      prev_item = item;
    }
    if (ok && it > 0 && !drain_half(it - 1, prev_item, 0)) ok = false;
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
    CUtensorMap tq, tk, tv;
    const uint64_t rb = (uint64_t)ld * 2;
    if (!make_tmap_2d_bf16(&tq, q, kHidden, (uint64_t)T, rb, 64, AT_Q) ||
        !make_tmap_2d_bf16(&tk, k, kHidden, (uint64_t)T, rb, 64, AT_KEYS) ||
        !make_tmap_2d_bf16(&tv, v, kHidden, (uint64_t)T, rb, 64, AT_KEYS))
      return cudaErrorInvalidValue;
    // rows leave as 32-byte sectors when the output and its stride allow it, else as 16-byte pieces
    const bool v8 = (reinterpret_cast<uintptr_t>(out) % 32) == 0 && (ld_out % 16) == 0;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t items = (T + AT_Q - 1) / AT_Q * kHeads;
    const unsigned grid = (unsigned)(items < sms ? items : (sms > 0 ? sms : 1));
    return launch_k(k_attention_tc, dim3(grid), dim3(AT_THREADS), AT_SMEM, s, tq, tk, tv, static_cast<bf16 *>(out),
                    ld_out, v8, R, qscale, k_scale, cap, pos, (int)T, lo, hi, device_status_word());
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
