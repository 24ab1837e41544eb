// Self-attention with a Transformer-XL relative-position bias, over whole
// clips (cera 0.5.3, audio_encoder_gpu.rs: the `xl_attention` op of the LFM2A
// Conformer): per head, score(i, j) = ((q_i + u) . k_j + (q_i + v) .
// p_{i - j}) / sqrt(64), softmax over the keys j of the clip, out_i =
// sum_j softmax * v_j. p_r is the projected position row of relative
// distance r; the table holds r = t_max - 1 .. -(t_max - 1) top to bottom,
// so row (t_max - 1 - r) is distance r.
//
// One CTA per (clip, 128-query block, head); warp 0 loads tiles with TMA,
// warp 1 issues tcgen05.mma, and two row warps per 32-row quarter of the tile
// own a query row per thread, each warp half of the keys (64 of a block's 128)
// and half of the output dims; the two exchange their rows' block maxima and
// final sums through shared memory (64-arrival mbarriers per quarter). Per
// 128-key block:
//   * TMA: the 128 key rows and the 256 position rows of the distances the
//     block spans (r = i - j from i0 - j0 - 127 to i0 - j0 + 127; rows outside
//     the table are zero-filled) into one of two stages, loaded while the
//     block before is processed, and the 128 value rows (one buffer, loaded
//     once the previous block's P V has read it);
//   * S = (q + u) K^T (M=128, N=128) and T = (q + v) Pband^T (M=128, N=256)
//     into tensor memory; (q + u) and (q + v) are written once, as bf16, by
//     the row threads;
//   * the row thread of query li needs T[li][127 - li + lj] for key lj: a
//     window that starts one column earlier per row. It loads the two 32-column
//     chunks of T that cover its window for 32 keys, writes them into its row
//     of a per-warp scratch (row pitch 66 floats) and reads them back from
//     offset 31 - lane (conflict-free: 65 lane + const); then adds S, scales
//     and masks keys past the clip end, 32 keys at a time (two such chunks per
//     warp and block);
//   * online softmax over the key blocks: the row thread keeps its row's
//     running maximum and sum, writes the block's probabilities (relative to
//     the new maximum) as bf16 into tensor memory, and, when the maximum grew,
//     first rescales its part of the row's P V accumulator there (one
//     tcgen05.ld and one tcgen05.st); tcgen05.mma then accumulates P V (A = P
//     from tensor memory, M=128, N=64, K=128, V read MN-major) into it. The
//     row thread reads the accumulator once at the end and divides by the sum.
// Every wait is bounded and reports through the library's status word.
#include "ae_internal.h"
#include "common.cuh"

namespace ae {

namespace {
constexpr int XA_Q = 128, XA_K = 128, XA_HD = 64;
constexpr uint32_t XA_TILE = 128 * 128;               // 128 rows x 64 bf16
constexpr uint32_t OFF_QU = 0, OFF_QV = OFF_QU + XA_TILE, OFF_V = OFF_QV + XA_TILE;
constexpr uint32_t OFF_K = OFF_V + XA_TILE;              // [2 stages] 128 key rows
constexpr uint32_t OFF_PB = OFF_K + 2 * XA_TILE;         // [2 stages] 256 position rows
constexpr uint32_t OFF_SCR = OFF_PB + 4 * XA_TILE;       // skew scratch, 8 warps x 32 rows x 66 floats
constexpr int SCR_PITCH = 66;
constexpr uint32_t OFF_X = OFF_SCR + 8 * 32 * SCR_PITCH * 4;  // [2 block parities][2 key halves][128] maxima, [2][128] sums
constexpr uint32_t OFF_BAR = OFF_X + (2 * 2 * 128 + 2 * 128) * 4;
constexpr size_t XA_SMEM = OFF_BAR + 256 + 1024;
constexpr int XA_THREADS = 320;
constexpr int XA_ROW_THREADS = 256;
constexpr uint32_t XA_TMEM_COLS = 512, COL_S = 0, COL_T = 128, COL_O = 384, COL_P = 448;  // P: 128 bf16 keys
constexpr uint32_t XA_KP_BYTES = 3 * XA_TILE;            // K and two position boxes
static_assert(XA_SMEM <= 227 * 1024, "shared memory");
static_assert(OFF_K % 1024 == 0 && OFF_PB % 1024 == 0 && OFF_SCR % 16 == 0, "swizzle atoms");

// D[tmem] (+)= A[tmem] * B[smem]^T, bf16, f32 accumulate: A's row m is lane m,
// two bf16 per 32-bit column (the lower k in the low half), K = 16 per
// instruction over 8 columns. One thread issues.
__device__ __forceinline__ void xa_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
}  // namespace

// 32 lanes x 32 consecutive 32-bit columns from registers into tensor memory
// (thread i of the warp writes row lane-base + i), and the wait for them.
__device__ __forceinline__ void xa_tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
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
// 2^x with the hardware's base-2 exponential (0 for x = -inf); the
// probabilities it gives are rounded to bf16 for the P V product
__device__ __forceinline__ float xa_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void xa_tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__global__ void __launch_bounds__(XA_THREADS, 1)
    k_lenc_xlattn(const __grid_constant__ CUtensorMap tmQKV, const __grid_constant__ CUtensorMap tmP,
                  const float *__restrict__ bias_u, const float *__restrict__ bias_v,
                  const int32_t *__restrict__ tok_off, const int32_t *__restrict__ qblk_off, int n_clips,
                  int t_max, int p_col, bf16 *__restrict__ out, int ld_out, unsigned *status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQu = smem + OFF_QU, *sQv = smem + OFF_QV, *sV = smem + OFF_V;
  float *scr = reinterpret_cast<float *>(smem + OFF_SCR);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint64_t *q_full = bars, *q_ready = bars + 1, *v_full = bars + 2, *s_full = bars + 3, *s_free = bars + 4,
           *p_full = bars + 5, *o_full = bars + 6;
  uint64_t *kp_full = bars + 20, *kp_free = bars + 22;  // per stage: K and position rows landed / read
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 7);
  // per lane quarter: the two row warps' exchanges (q tiles read, block maxima, final sums)
  uint64_t *xq = bars + 8, *xm = bars + 12, *xs = bars + 16;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // item -> (clip, query block, head)
  const int head = blockIdx.x % kLencHeads, qitem = blockIdx.x / kLencHeads;
  // the last clip whose first query block is <= qitem: for up to 1024 clips each
  // warp counts the offsets <= qitem with independent loads (one round trip;
  // the offsets are non-decreasing), else a binary search
  int c = 0;
  if (n_clips <= 1024) {
    int cnt = 0;
    for (int i = lane; i < n_clips; i += 32) cnt += qblk_off[i] <= qitem ? 1 : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    c = cnt - 1;
  } else {
    int lo = 0, hi = n_clips;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (qblk_off[mid] <= qitem) lo = mid; else hi = mid;
    }
    c = lo;
  }
  const int tok0 = tok_off[c], t_c = tok_off[c + 1] - tok0;
  const int i0 = (qitem - qblk_off[c]) * XA_Q;
  const int n_kb = (t_c + XA_K - 1) / XA_K;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_ready, XA_ROW_THREADS);
    mbar_init(v_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kp_full[i], 1);
      mbar_init(&kp_free[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, XA_ROW_THREADS);
    mbar_init(p_full, XA_ROW_THREADS);
    mbar_init(o_full, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&xq[i], 64);
      mbar_init(&xm[i], 64);
      mbar_init(&xs[i], 64);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQKV);
    tma_prefetch_desc(&tmP);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, XA_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer: K and position rows of block kb into stage kb & 1
    // (once the score MMAs of block kb - 2 have read it), V of block kb into its
    // buffer (once the P V of block kb - 1 has read it)
    bool ok = true;
    mbar_arrive_expect_tx(q_full, XA_TILE);
    tma_load_2d(sQu, &tmQKV, head * XA_HD, tok0 + i0, q_full);
    int n_kp = 0, n_v = 0;
    auto load_kp = [&](int kb) -> bool {
      const int st = kb & 1;
      if (kb >= 2 && !mbar_wait(&kp_free[st], ((kb >> 1) - 1) & 1)) return false;
      if (*abort_flag) return false;
      const int j0 = kb * XA_K;
      const int prow = t_max - 128 - i0 + j0;  // table row of distance i0 - j0 + 127
      mbar_arrive_expect_tx(&kp_full[st], XA_KP_BYTES);
      tma_load_2d(smem + OFF_K + st * XA_TILE, &tmQKV, kLencEmbd + head * XA_HD, tok0 + j0, &kp_full[st]);
      tma_load_2d(smem + OFF_PB + st * 2 * XA_TILE, &tmP, p_col + head * XA_HD, prow, &kp_full[st]);
      tma_load_2d(smem + OFF_PB + st * 2 * XA_TILE + XA_TILE, &tmP, p_col + head * XA_HD, prow + 128, &kp_full[st]);
      ++n_kp;
      return true;
    };
    auto load_v = [&](int kb) -> bool {
      if (kb >= 1 && !mbar_wait(o_full, (kb - 1) & 1)) return false;
      if (*abort_flag) return false;
      mbar_arrive_expect_tx(v_full, XA_TILE);
      tma_load_2d(sV, &tmQKV, 2 * kLencEmbd + head * XA_HD, tok0 + kb * XA_K, v_full);
      ++n_v;
      return true;
    };
    if (n_kb > 0) ok = load_kp(0) && load_v(0);
    for (int kb = 1; kb < n_kb && ok; ++kb) ok = load_kp(kb) && load_v(kb);
    if (!ok) {
      atomicOr(status, kStatusWaitTimeout);
      *abort_flag = 1;
    }
    mbar_wait(q_full, 0);  // every load lands before the CTA ends
#pragma unroll
    for (int st = 0; st < 2; ++st) {
      const int u = (n_kp + 1 - st) / 2;  // uses of stage st
      if (u > 0) mbar_wait(&kp_full[st], (u - 1) & 1);
    }
    if (n_v > 0) mbar_wait(v_full, (n_v - 1) & 1);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    constexpr uint32_t idesc_s = idesc_bf16_f32(XA_Q, XA_K);
    constexpr uint32_t idesc_t = idesc_bf16_f32(XA_Q, 2 * XA_K);
    constexpr uint32_t idesc_o = idesc_bf16_f32_bmn(XA_Q, XA_HD);
    const uint32_t aqu = smem_u32(sQu), aqv = smem_u32(sQv), av = smem_u32(sV);
    // the score products of block kb + 1 go out as soon as the row threads have
    // read block kb's, so they run during block kb's softmax; P V of block kb
    // follows once its probabilities are in tensor memory
    auto scores = [&](int kb) -> bool {
      const int st = kb & 1;
      const uint32_t ak = smem_u32(smem + OFF_K + st * XA_TILE), apb = smem_u32(smem + OFF_PB + st * 2 * XA_TILE);
      if (!mbar_wait(&kp_full[st], (kb >> 1) & 1) || (kb > 0 && !mbar_wait(s_free, (kb - 1) & 1)) || *abort_flag)
        return false;
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < XA_HD / 16; ++k)
        tc_mma_bf16(tmem + COL_S, sw128_desc(aqu + k * 32), sw128_desc(ak + k * 32), idesc_s, k > 0 ? 1u : 0u);
#pragma unroll
      for (int k = 0; k < XA_HD / 16; ++k)
        tc_mma_bf16(tmem + COL_T, sw128_desc(aqv + k * 32), sw128_desc(apb + k * 32), idesc_t, k > 0 ? 1u : 0u);
      tc_commit(&kp_free[st]);
      tc_commit(s_full);
      return true;
    };
    bool ok = mbar_wait(q_ready, 0) && (n_kb == 0 || scores(0));
    for (int kb = 0; kb < n_kb && ok; ++kb) {
      if (kb + 1 < n_kb && !scores(kb + 1)) {
        ok = false;
        break;
      }
      if (!mbar_wait(p_full, kb & 1) || !mbar_wait(v_full, kb & 1) || *abort_flag) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < XA_K / 16; ++ks)
        xa_mma_ts(tmem + COL_O, tmem + COL_P + 8 * ks, sw128_desc_mn(av + ks * 2048, XA_TILE), idesc_o,
                  (kb | ks) != 0 ? 1u : 0u);
      tc_commit(o_full);
    }
    if (!ok) {
      atomicOr(status, kStatusWaitTimeout);
      *abort_flag = 1;
    }
  } else if (warp >= 2) {
    // ---------------- row threads: TMEM lane quarter qw, query row li = 32 qw + lane;
    // warp half kh: keys 64 kh .. 64 kh + 63 of each block, output dims 32 kh .. 32 kh + 31
    const int qw = warp & 3, kh = (warp - 2) >> 2, li = 32 * qw + lane, r7 = li & 7;
    const uint32_t trow = tmem + ((uint32_t)(32 * qw) << 16);
    float *my = scr + (size_t)((kh * 4 + qw) * 32 + lane) * SCR_PITCH;
    float *xmax = reinterpret_cast<float *>(smem + OFF_X), *xsum = xmax + 2 * 2 * 128;
    // the two warps of a quarter meet at an mbarrier of 64 arrivals (bounded wait)
    auto pair_sync = [&](uint64_t *b, uint32_t parity) -> bool {
      mbar_arrive(b);
      return __all_sync(0xffffffffu, mbar_wait(b, parity));
    };
    bool ok = true;
    // ---- q + u (warp half 0) and q + v (half 1) as bf16 operand tiles, in place
    // of / beside the raw q rows, once both halves have read them
    if (!__all_sync(0xffffffffu, mbar_wait(q_full, 0))) ok = false;
    {
      uint4 w[8];
#pragma unroll
      for (int g = 0; g < 8; ++g) w[g] = *reinterpret_cast<const uint4 *>(sQu + li * 128 + ((g ^ r7) << 4));
      if (!pair_sync(&xq[qw], 0)) ok = false;
      if (ok) {
        const float *bias = (kh == 0 ? bias_u : bias_v) + head * XA_HD;
        uint8_t *dst = kh == 0 ? sQu : sQv;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const float q[8] = {bf16lo(w[g].x), bf16hi(w[g].x), bf16lo(w[g].y), bf16hi(w[g].y),
                              bf16lo(w[g].z), bf16hi(w[g].z), bf16lo(w[g].w), bf16hi(w[g].w)};
          const float4 b0 = *reinterpret_cast<const float4 *>(bias + 8 * g);
          const float4 b1 = *reinterpret_cast<const float4 *>(bias + 8 * g + 4);
          *reinterpret_cast<uint4 *>(dst + li * 128 + ((g ^ r7) << 4)) =
              make_uint4(pack_bf16(q[0] + b0.x, q[1] + b0.y), pack_bf16(q[2] + b0.z, q[3] + b0.w),
                         pack_bf16(q[4] + b1.x, q[5] + b1.y), pack_bf16(q[6] + b1.z, q[7] + b1.w));
        }
        fence_async_smem();
      }
    }
    mbar_arrive(q_ready);
    constexpr float kScale = 0.125f * 1.4426950408889634f;  // 1/sqrt(64), in base 2
    float m_run = -INFINITY, l_run = 0.f;  // l_run: this warp half's keys only
    for (int kb = 0; kb < n_kb && ok; ++kb) {
      const int j0 = kb * XA_K + 64 * kh;
      if (!__all_sync(0xffffffffu, mbar_wait(s_full, kb & 1))) { ok = false; break; }
      tc_fence_after();
      // ---- this half's 64 logits: S plus the skewed window of T
      float z[64];
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const int q = 2 * kh + qq;  // 32-key chunk of the block
        uint32_t a[32], b[32];
        const int ca = 3 - qw + q;  // chunk of T holding column 127 - li + 32 q (or the next one)
        tmem_ld32(trow + COL_T + 32 * ca, a);
        tmem_ld32(trow + COL_T + 32 * (ca + 1), b);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          *reinterpret_cast<float2 *>(my + 2 * e) = make_float2(__uint_as_float(a[2 * e]), __uint_as_float(a[2 * e + 1]));
          *reinterpret_cast<float2 *>(my + 32 + 2 * e) =
              make_float2(__uint_as_float(b[2 * e]), __uint_as_float(b[2 * e + 1]));
        }
        tmem_ld32(trow + COL_S + 32 * q, a);
        tmem_ld_wait();
        __syncwarp();
        if (j0 + 32 * qq + 32 <= t_c) {  // every key of the chunk lies in the clip
#pragma unroll
          for (int x = 0; x < 32; ++x) z[32 * qq + x] = (__uint_as_float(a[x]) + my[31 - lane + x]) * kScale;
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            const int j = j0 + 32 * qq + x;
            z[32 * qq + x] = j < t_c ? (__uint_as_float(a[x]) + my[31 - lane + x]) * kScale : -INFINITY;
          }
        }
        __syncwarp();
      }
      tc_fence_before();
      mbar_arrive(s_free);  // this block's scores are read
      float bm = -INFINITY;
#pragma unroll
      for (int x = 0; x < 64; ++x) bm = fmaxf(bm, z[x]);
      xmax[((kb & 1) * 2 + kh) * 128 + li] = bm;
      if (!pair_sync(&xm[qw], kb & 1)) { ok = false; break; }
      // finite: every block holds a key of the clip, in one half or the other
      const float m_new = fmaxf(m_run, fmaxf(bm, xmax[((kb & 1) * 2 + (kh ^ 1)) * 128 + li]));
      const float alpha = xa_ex2(m_run - m_new);  // 0 on the first block
      // the previous block's P V is done: the probabilities' buffer is free and
      // the accumulator holds every earlier block
      if (kb > 0 && !__all_sync(0xffffffffu, mbar_wait(o_full, (kb - 1) & 1))) { ok = false; break; }
      tc_fence_after();
      float ls = 0.f;
      uint32_t pw[32];  // keys 64 kh .. 64 kh + 63 as bf16 pairs: tensor-memory columns COL_P + 32 kh ..
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        const float p0 = xa_ex2(z[2 * x] - m_new), p1 = xa_ex2(z[2 * x + 1] - m_new);
        ls += p0 + p1;
        pw[x] = pack_bf16(p0, p1);
      }
      xa_tmem_st32(trow + COL_P + 32 * kh, pw);
      l_run = l_run * alpha + ls;
      m_run = m_new;
      if (kb > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
        // rescale this warp's 32 columns of the row's accumulator to the new maximum
        uint32_t o[32];
        tmem_ld32(trow + COL_O + 32 * kh, o);
        tmem_ld_wait();
#pragma unroll
        for (int d = 0; d < 32; ++d) o[d] = __float_as_uint(__uint_as_float(o[d]) * alpha);
        xa_tmem_st32(trow + COL_O + 32 * kh, o);
      }
      xa_tmem_st_wait();  // P (and the rescaled accumulator) are in tensor memory
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && !__all_sync(0xffffffffu, mbar_wait(o_full, (n_kb - 1) & 1))) ok = false;
    // both halves' sums (also after a failure; the wait is bounded either way)
    xsum[kh * 128 + li] = l_run;
    if (!pair_sync(&xs[qw], 0)) ok = false;
    if (ok) {
      tc_fence_after();
      const float inv = 1.0f / (l_run + xsum[(kh ^ 1) * 128 + li]);
      uint32_t o0[32];
      tmem_ld32(trow + COL_O + 32 * kh, o0);
      tmem_ld_wait();
      if (i0 + li < t_c) {
        bf16 *orow = out + (int64_t)(tok0 + i0 + li) * ld_out + head * XA_HD + 32 * kh;
#pragma unroll
        for (int g = 0; g < 4; ++g)
          *reinterpret_cast<uint4 *>(orow + 8 * g) = make_uint4(
              pack_bf16(__uint_as_float(o0[8 * g]) * inv, __uint_as_float(o0[8 * g + 1]) * inv),
              pack_bf16(__uint_as_float(o0[8 * g + 2]) * inv, __uint_as_float(o0[8 * g + 3]) * inv),
              pack_bf16(__uint_as_float(o0[8 * g + 4]) * inv, __uint_as_float(o0[8 * g + 5]) * inv),
              pack_bf16(__uint_as_float(o0[8 * g + 6]) * inv, __uint_as_float(o0[8 * g + 7]) * inv));
      }
    }
    if (!ok && lane == 0) {
      atomicOr(status, kStatusWaitTimeout);
      *abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, XA_TMEM_COLS);
  }
}

cudaError_t launch_lenc_xlattn(const void *qkv, int64_t T, const void *ptab, int64_t p_rows, int64_t p_cols, int p_col,
                               const float *bias_u, const float *bias_v, const int32_t *tok_off,
                               const int32_t *qblk_off, int n_clips, int n_qblk, int t_max, void *out,
                               cudaStream_t s) {
  if (n_qblk <= 0 || T <= 0) return cudaSuccess;
  static std::atomic<uint64_t> attr{0};
  if (const cudaError_t e = smem_attr(k_lenc_xlattn, XA_SMEM, attr)) return e;
  CUtensorMap tq, tp;
  if (!make_tmap_2d_bf16(&tq, qkv, 3 * kLencEmbd, (uint64_t)T, 3 * kLencEmbd * 2, 64, 128) ||
      !make_tmap_2d_bf16(&tp, ptab, (uint64_t)p_cols, (uint64_t)p_rows, (uint64_t)p_cols * 2, 64, 128))
    return cudaErrorInvalidValue;
  return launch_k(k_lenc_xlattn, dim3((unsigned)(n_qblk * kLencHeads)), dim3(XA_THREADS), XA_SMEM, s, tq, tp, bias_u,
                  bias_v, tok_off, qblk_off, n_clips, t_max, p_col, static_cast<bf16 *>(out), kLencEmbd,
                  device_status_word());
}

}  // namespace ae
