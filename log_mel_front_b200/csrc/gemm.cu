// Projections of the tower: y = epilogue(x W^T) with x [M][K] (packed token
// rows, M ragged) and W [N][K] (the checkpoint's [out][in] layout).
//
// Tensor-core path: a persistent tcgen05 kernel on CTA pairs (clusters of two
// SMs), warp-specialised. Per k-block (one 128-byte swizzle atom per row: 64
// bf16 or 128 e4m3 elements), each CTA's warp 0 streams its half of the pair
// tile (128 rows of x, 128 rows of W) into a shared-memory ring with TMA (no
// multicast): 6 stages for the epilogues that store from registers, 4 for the
// float32 ones, which also need staging boxes. The leader CTA's warp 1 issues
// tcgen05.mma.cta_group::2 (M=256, N=256; kind::f16 with K=16 for bf16,
// kind::f8f6f4 with K=32 for e4m3, f32 accumulate), which reads the operand
// halves from both SMs, into one of two 256-column accumulators in each CTA's
// tensor memory. Warps 2-9 of each CTA drain the other accumulator with
// tcgen05.ld and apply the epilogue: the e4m3 column factors, the ClipLin output
// clamp, SiLU (and the next projection's input clamp, or its e4m3 codes), GLU,
// bias or the residual add. bf16 and e4m3 results leave each lane's row as
// 32-byte sectors from registers; float32 results go through a swizzled
// shared-memory box and coalesced row stores. Pairing halves the W bytes each
// SM stages per flop. Tiles are walked m-major, so the pairs in flight share
// rows of x in L2 while W stays L2-resident.
//
// f32 path: a plain 64x64-tile FMA kernel with the same epilogues.
#include <cudaTypedefs.h>

#include "ae_internal.h"
#include "common.cuh"

namespace ae {

__device__ unsigned g_status_word = 0;

unsigned read_and_clear_status() {
  unsigned v = 0, z = 0;
  if (cudaMemcpyFromSymbol(&v, g_status_word, sizeof(v)) != cudaSuccess) return ~0u;
  cudaMemcpyToSymbol(g_status_word, &z, sizeof(z));
  return v;
}

unsigned *device_status_word() {
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
  return static_cast<unsigned *>(p);
}

// The failure path of the bounded waits, exercised without a fault: thread 0
// initialises an mbarrier of one arrival and waits on its first phase, which
// completes only if `arrive` (then the wait succeeds at once); otherwise the
// wait gives up after limit_ns and records the timeout as the kernels do.
__global__ void k_wait_probe(unsigned long long limit_ns, int arrive, unsigned *status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  if (arrive) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&bar)) : "memory");
  if (!mbar_wait_for(&bar, 0, limit_ns)) atomicOr(status, kStatusWaitTimeout);
}

cudaError_t launch_wait_probe(unsigned long long limit_ns, int arrive, cudaStream_t s) {
  return launch_k(k_wait_probe, dim3(1), dim3(32), 0, s, limit_ns, arrive, device_status_word());
}

// ------------------------------------------------------------------ epilogue

// 128-byte line of the staging buffer: the 16-byte granule g of row r sits at
// granule g ^ (r & 7) (the TMA's 128-byte swizzle), so the 32 rows of a warp
// write a granule column without bank conflicts.
__device__ __forceinline__ void st_granule(uint8_t *line, int r7, int g, uint4 v) {
  *reinterpret_cast<uint4 *>(line + ((g ^ r7) << 4)) = v;
}

// e4m3 projections: accumulator column j times cs[j] (the weight row's scale
// over the input's code scale). Every lane reads the same 32 factors.
__device__ __forceinline__ void scale_cols(const float *cs, float (&v)[32]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float4 c = __ldg(reinterpret_cast<const float4 *>(cs) + j);
    const float2 a = __fmul2_rn(make_float2(v[4 * j], v[4 * j + 1]), make_float2(c.x, c.y));
    const float2 b = __fmul2_rn(make_float2(v[4 * j + 2], v[4 * j + 3]), make_float2(c.z, c.w));
    v[4 * j] = a.x;
    v[4 * j + 1] = a.y;
    v[4 * j + 2] = b.x;
    v[4 * j + 3] = b.y;
  }
}

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

// c * sigmoid(g) = c / (1 + 2^(-g log2 e)) for two lanes: the power of two and
// the reciprocal from the special-function unit's approximations, the
// multiplies and the add on the packed two-lane pipe. Limits: g -> -inf gives
// 0 (the reciprocal of +inf), g -> +inf gives c.
__device__ __forceinline__ float2 mul_sigmoid2(float2 c, float2 g) {
  constexpr float kNegLog2e = -1.4426950408889634f;
  const float2 t = __fmul2_rn(g, make_float2(kNegLog2e, kNegLog2e));
  const float2 d = __fadd2_rn(make_float2(ex2_approx(t.x), ex2_approx(t.y)), make_float2(1.0f, 1.0f));
  return __fmul2_rn(c, make_float2(rcp_approx(d.x), rcp_approx(d.y)));
}

// Float32 epilogue (EPI_F32, EPI_ADD_F32) of 32 accumulator columns [col,
// col + 32) of one row: clamp (after the bias for EPI_F32), written as the 8
// granules g0 .. g0 + 7 of the row's staging line.
template <bool SC>
__device__ __forceinline__ void epi_stage_f32(const EpiArgs &ep, bool bias, float alpha, int col,
                                              const uint32_t (&r)[32], uint8_t *line, int r7, int g0) {
  float lo = ep.lo, hi = ep.hi;
  if (ep.seg_w > 0) {
    const int sg = col / ep.seg_w;  // selects, not a runtime index into the parameter array
    lo = sg == 0 ? ep.seg_lo[0] : (sg == 1 ? ep.seg_lo[1] : ep.seg_lo[2]);
    hi = sg == 0 ? ep.seg_hi[0] : (sg == 1 ? ep.seg_hi[1] : ep.seg_hi[2]);
  }
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  if (SC) scale_cols(ep.cs + col, v);
  if (bias) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] += __ldg(ep.bias + col + i);
  }
  if (alpha != 1.0f) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] *= alpha;
  }
#pragma unroll
  for (int j = 0; j < 8; ++j)
    st_granule(line, r7, g0 + j,
               make_uint4(__float_as_uint(clampf(v[4 * j], lo, hi)), __float_as_uint(clampf(v[4 * j + 1], lo, hi)),
                          __float_as_uint(clampf(v[4 * j + 2], lo, hi)),
                          __float_as_uint(clampf(v[4 * j + 3], lo, hi))));
}

__device__ __forceinline__ void st_global_32B(void *p, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t a4,
                                              uint32_t a5, uint32_t a6, uint32_t a7) {
  // no memory clobber: nothing in the kernel reads the outputs, so the next
  // chunk's loads may be scheduled ahead of these stores
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a0), "r"(a1), "r"(a2),
               "r"(a3), "r"(a4), "r"(a5), "r"(a6), "r"(a7));
}

// Epilogue of 32 accumulator columns of one row, stored from registers as
// whole 32-byte sectors (bf16 and e4m3 outputs; float32 outputs go through
// epi_stage_f32).
template <int MODE, bool SC>
__device__ __forceinline__ void epi_store32(const EpiArgs &ep, int row, int col, const uint32_t (&r)[32]) {
  float lo = ep.lo, hi = ep.hi;
  if (ep.seg_w > 0) {
    const int sg = col / ep.seg_w;
    lo = sg == 0 ? ep.seg_lo[0] : (sg == 1 ? ep.seg_lo[1] : ep.seg_lo[2]);
    hi = sg == 0 ? ep.seg_hi[0] : (sg == 1 ? ep.seg_hi[1] : ep.seg_hi[2]);
  }
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  if (SC) scale_cols(ep.cs + col, v);
  static_assert(MODE != EPI_F32 && MODE != EPI_ADD_F32 && MODE != EPI_BIAS_ADD_F32,
                "float32 outputs go through the staging boxes");
  // the bias modes add the column bias, then take the path of their plain mode
  // (GELU has its own)
  constexpr bool BIAS = MODE == EPI_BIAS_BF16 || MODE == EPI_BIAS_SILU || MODE == EPI_BIAS_GLU || MODE == EPI_BIAS_GELU;
  constexpr int BASE = MODE == EPI_BIAS_BF16 ? EPI_BF16
                       : MODE == EPI_BIAS_SILU ? EPI_SILU
                       : MODE == EPI_BIAS_GLU  ? EPI_GLU
                                               : MODE;
  if (BIAS) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 b = __ldg(reinterpret_cast<const float4 *>(ep.bias + col) + j);
      v[4 * j] += b.x;
      v[4 * j + 1] += b.y;
      v[4 * j + 2] += b.z;
      v[4 * j + 3] += b.w;
    }
  }
  if (BASE == EPI_BIAS_GELU) {  // x (1 + erf(x / sqrt 2)) / 2
    uint32_t p[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float a = v[2 * j], b = v[2 * j + 1];
      p[j] = pack_bf16(0.5f * a * (1.0f + erff(a * 0.70710678118654752f)),
                       0.5f * b * (1.0f + erff(b * 0.70710678118654752f)));
    }
    bf16 *o = static_cast<bf16 *>(ep.out) + (int64_t)row * ep.ld + col;
    st_global_32B(o, p[0], p[1], p[2], p[3], p[4], p[5], p[6], p[7]);
    st_global_32B(o + 16, p[8], p[9], p[10], p[11], p[12], p[13], p[14], p[15]);
  } else if (BASE == EPI_GLU) {
    uint32_t p[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {  // columns (4j, 4j+1, 4j+2, 4j+3) = (a, b, a, b)
      const float2 a = make_float2(clampf(v[4 * j], lo, hi), clampf(v[4 * j + 2], lo, hi));
      const float2 b = make_float2(clampf(v[4 * j + 1], lo, hi), clampf(v[4 * j + 3], lo, hi));
      const float2 y = mul_sigmoid2(a, b);
      p[j] = pack_bf16(y.x, y.y);
    }
    bf16 *o = static_cast<bf16 *>(ep.out) + (int64_t)row * ep.ld + col / 2;
    st_global_32B(o, p[0], p[1], p[2], p[3], p[4], p[5], p[6], p[7]);
  } else if (BASE == EPI_SILU || BASE == EPI_SILU_Q8) {
    float2 y[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float2 c = make_float2(clampf(v[2 * j], lo, hi), clampf(v[2 * j + 1], lo, hi));
      y[j] = mul_sigmoid2(c, c);
    }
    if (ep.clamp2) {  // the host clears it when the second clamp cannot bind
#pragma unroll
      for (int j = 0; j < 16; ++j) y[j] = make_float2(clampf(y[j].x, ep.lo2, ep.hi2), clampf(y[j].y, ep.lo2, ep.hi2));
    }
    if (MODE == EPI_SILU_Q8) {  // the next projection's e4m3 operand: 32 codes, one 32-byte sector
      uint32_t p[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float2 a = __fmul2_rn(y[2 * j], make_float2(ep.q8, ep.q8));
        const float2 b = __fmul2_rn(y[2 * j + 1], make_float2(ep.q8, ep.q8));
        p[j] = pack_e4m3x4(a.x, a.y, b.x, b.y);
      }
      uint8_t *o = static_cast<uint8_t *>(ep.out) + (int64_t)row * ep.ld + col;
      st_global_32B(o, p[0], p[1], p[2], p[3], p[4], p[5], p[6], p[7]);
    } else {
      uint32_t p[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) p[j] = pack_bf16(y[j].x, y[j].y);
      bf16 *o = static_cast<bf16 *>(ep.out) + (int64_t)row * ep.ld + col;
      st_global_32B(o, p[0], p[1], p[2], p[3], p[4], p[5], p[6], p[7]);
      st_global_32B(o + 16, p[8], p[9], p[10], p[11], p[12], p[13], p[14], p[15]);
    }
  } else {  // EPI_BF16
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = clampf(v[i], lo, hi);
    uint32_t p[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) p[j] = pack_bf16(v[2 * j], v[2 * j + 1]);
    bf16 *o = static_cast<bf16 *>(ep.out) + (int64_t)row * ep.ld + col;
    st_global_32B(o, p[0], p[1], p[2], p[3], p[4], p[5], p[6], p[7]);
    st_global_32B(o + 16, p[8], p[9], p[10], p[11], p[12], p[13], p[14], p[15]);
  }
}

// ------------------------------------------------------------------ tcgen05 pair kernel

namespace {
constexpr int BM = 128;                 // rows of x per CTA (256 per pair)
constexpr int BK = 64;                  // one 128-byte swizzle atom of bf16
constexpr int BN = 256;                 // columns per pair tile (128 rows of W per CTA)
constexpr uint32_t A_BYTES = BM * BK * 2, B_BYTES = (BN / 2) * BK * 2, STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t TMEM_COLS = 2 * BN;  // two 128 x 256 f32 accumulators per CTA
constexpr int EPI_WARPS = 8;
constexpr uint32_t LINE_BYTES = 32 * 128;  // one staging box: 32 rows x 128 bytes
constexpr uint32_t EPI_BYTES = EPI_WARPS * LINE_BYTES;  // one box per epilogue warp
constexpr int GEMM_THREADS = 64 + 32 * EPI_WARPS;
// float32 outputs go through the staging boxes, which leave room for a
// 4-stage ring; the other epilogues store from registers and take 6 stages,
// which keeps more loads in flight (the e4m3 mainloop consumes a stage in half
// the time of a bf16 one).
__host__ __device__ constexpr bool f32_out(int mode) {
  return mode == EPI_F32 || mode == EPI_ADD_F32 || mode == EPI_BIAS_ADD_F32;
}
__host__ __device__ constexpr int stages_of(int mode) { return f32_out(mode) ? 4 : 6; }
__host__ __device__ constexpr size_t smem_of(int mode) {
  return stages_of(mode) * STAGE_BYTES + (f32_out(mode) ? EPI_BYTES : 0) + 1024 + 256;
}
}  // namespace

// Persistent pair kernel (cluster of 2 CTAs on 2 SMs). Pair tile 256 x 256:
// CTA r of the pair loads rows [m0 + 128 r, +128) of x and rows
// [n0 + 128 r, +128) of W for every 64-wide k-block; the leader (even) CTA
// issues tcgen05.mma.cta_group::2 (M=256, N=256, K=16), which reads the A and
// B halves from both CTAs' shared memory and accumulates rows 128 r .. +127
// in CTA r's tensor memory. Each CTA's epilogue drains its own 128 rows.
template <int MODE, bool F8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GEMM_THREADS, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const EpiArgs ep, const int M, const int N, const int K,
              unsigned *status) {
  constexpr int STAGES = stages_of(MODE);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *epi_smem = smem + STAGES * STAGE_BYTES;                                 // store boxes (f32 outputs)
  uint64_t *full = reinterpret_cast<uint64_t *>(epi_smem + (f32_out(MODE) ? EPI_BYTES : 0));  // used in the leader
  uint64_t *empty = full + STAGES;                                              // per CTA
  uint64_t *tfull = empty + STAGES;                                             // per CTA
  uint64_t *tempty = tfull + 2;                                                 // used in the leader
  uint64_t *done = tempty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  // one k-block is a 128-byte swizzle atom per row: 64 bf16 or 128 e4m3 elements
  constexpr int BKE = F8 ? 2 * BK : BK;
  const int m_blocks = (M + 2 * BM - 1) / (2 * BM), n_blocks = N / BN, kb_n = K / BKE;
  const int num_tiles = m_blocks * n_blocks;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 2 * EPI_WARPS);  // one arrival per epilogue warp of both CTAs
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers are initialised before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer (both CTAs)
    int stage = 0;
    uint32_t phase = 0;
    long issued = 0;
    bool ok = true;
    for (int tile = pair; tile < num_tiles && ok; tile += n_pairs) {
      const int mb = tile / n_blocks, nb = tile % n_blocks;
      const int arow = mb * 2 * BM + (int)rank * BM, brow = nb * BN + (int)rank * (BN / 2);
      for (int kb = 0; kb < kb_n; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1) || *abort_flag) {
          ok = false;
          break;
        }
        uint8_t *sa = smem + stage * STAGE_BYTES;
        if (leader) mbar_arrive_expect_tx(&full[stage], 2 * STAGE_BYTES);
        tma_load_2d_pair(sa, &tmA, kb * BKE, arow, &full[stage]);
        tma_load_2d_pair(sa + A_BYTES, &tmB, kb * BKE, brow, &full[stage]);
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (!ok) {
      atomicOr(status, kStatusWaitTimeout);
      *abort_flag = 1;
    }
    if (leader) {  // every load issued by the pair must land before the leader may exit
      for (int s = 0; s < STAGES; ++s) {
        const long n = issued / STAGES + (s < issued % STAGES ? 1 : 0);
        if (n > 0) mbar_wait(&full[s], (uint32_t)((n - 1) & 1));
      }
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ---------------- MMA issuer (leader CTA only)
    constexpr uint32_t idesc = F8 ? idesc_e4m3_f32(2 * BM, BN) : idesc_bf16_f32(2 * BM, BN);
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true;
    for (int tile = pair; tile < num_tiles && ok; tile += n_pairs) {
      if (!mbar_wait(&tempty[acc], acc_phase ^ 1) || *abort_flag) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      for (int kb = 0; kb < kb_n; ++kb) {
        if (!mbar_wait(&full[stage], phase)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
        const uint32_t sb = sa + A_BYTES;
#pragma unroll
        for (int k = 0; k < 4; ++k) {  // 32 bytes of k per instruction: K = 16 bf16 or 32 e4m3
          if (F8)
            tc_mma_f8_pair(d_tmem, sw128_desc(sa + k * 32), sw128_desc(sb + k * 32), idesc, (kb | k) != 0 ? 1u : 0u);
          else
            tc_mma_bf16_pair(d_tmem, sw128_desc(sa + k * 32), sw128_desc(sb + k * 32), idesc,
                             (kb | k) != 0 ? 1u : 0u);
        }
        tc_commit_pair_both(&empty[stage]);  // frees the stage in both CTAs
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      tc_commit_pair_both(&tfull[acc]);  // accumulator ready in both CTAs
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if (!ok) {
      atomicOr(status, kStatusWaitTimeout);
      *abort_flag = 1;
    }
    tc_commit_pair_local(done);  // arrives once every MMA issued above has completed
    mbar_wait(done, 0);
  } else if (warp >= 2) {
    // ---------------- epilogue (both CTAs): warp w reads TMEM lanes 32*(w%4) .. +31
    // (rows of the tile) and one half of the tile's 256 columns. bf16 results
    // leave each lane's row as whole 32-byte sectors. f32 results are written
    // by each lane into a 32-row x 128-byte box in shared memory (128-byte
    // swizzle: conflict-free), which the warp reads back row by row to write 4
    // full 128-byte row segments per store instruction (measured faster for
    // f32, slower for bf16, than the direct sector stores).
    constexpr bool F32_OUT = f32_out(MODE);
    // float32 staging: one 32-column TMEM load fills a box row (128 bytes)
    constexpr int LOADS_PER_BOX = 1, OUT_COLS_PER_BOX = 32, GRANULES_PER_LOAD = 8, ES = 4;
    const int q = warp & 3, half = (warp - 2) >> 2;
    uint8_t *box = epi_smem + (warp - 2) * LINE_BYTES;
    const uint32_t tempty_leader = map_to_rank(&tempty[0], 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int tile = pair; tile < num_tiles; tile += n_pairs) {
      const int mb = tile / n_blocks, nb = tile % n_blocks;
      const bool got = mbar_wait(&tfull[acc], acc_phase);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int row0 = mb * 2 * BM + (int)rank * BM + q * 32;
      const int col0 = nb * BN + half * (BN / 2);
      const int ocol0 = (MODE == EPI_GLU || MODE == EPI_BIAS_GLU) ? col0 / 2 : col0;
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + half * (BN / 2));
      auto stage = [&](int c, const uint32_t(&r)[32]) {
        if constexpr (!F32_OUT) {  // bf16 / e4m3 rows: 32-byte stores straight from registers
          if (row0 + lane < M) epi_store32<MODE, F8>(ep, row0 + lane, col0 + c * 32, r);
        } else {
          const int j = c % LOADS_PER_BOX;
          epi_stage_f32<F8>(ep, (MODE == EPI_F32 || MODE == EPI_BIAS_ADD_F32) && ep.bias,
                            MODE == EPI_BIAS_ADD_F32 ? ep.alpha : 1.0f, col0 + c * 32, r, box + lane * 128, lane & 7,
                            j * GRANULES_PER_LOAD);
          if (j == LOADS_PER_BOX - 1) {
            __syncwarp();
            // lane l moves granule l % 8 of rows l / 8, l / 8 + 4, ...
            const int g = lane & 7;
            uint8_t *dst = static_cast<uint8_t *>(ep.out) +
                           ((int64_t)ocol0 + (c / LOADS_PER_BOX) * OUT_COLS_PER_BOX) * ES + g * 16;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int rr = (lane >> 3) + 4 * i;
              const uint4 v = *reinterpret_cast<const uint4 *>(box + rr * 128 + ((g ^ (rr & 7)) << 4));
              if (row0 + rr < M) {
                uint8_t *p = dst + (int64_t)(row0 + rr) * ep.ld * ES;
                if (MODE == EPI_ADD_F32 || MODE == EPI_BIAS_ADD_F32)  // one vector add per 4 elements; no other thread touches them
                  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(__uint_as_float(v.x)),
                               "f"(__uint_as_float(v.y)), "f"(__uint_as_float(v.z)), "f"(__uint_as_float(v.w))
                               : "memory");
                else
                  *reinterpret_cast<uint4 *>(p) = v;
              }
            }
            __syncwarp();
          }
        }
      };
      // two register buffers: the next chunk's tcgen05.ld is in flight during the math
      uint32_t ra[32], rb[32];
      tmem_ld32(tbase, ra);
      tmem_ld_wait();
#pragma unroll 1
      for (int c = 0; c < BN / 64; c += 2) {
        tmem_ld32(tbase + (c + 1) * 32, rb);
        stage(c, ra);
        tmem_ld_wait();
        if (c + 2 < BN / 64) tmem_ld32(tbase + (c + 2) * 32, ra);
        stage(c + 1, rb);
        tmem_ld_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(tempty_leader + (uint32_t)(acc * sizeof(uint64_t)));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if (!ok && lane == 0) {
      atomicOr(status, kStatusWaitTimeout);
      *abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA of the pair leaves while the other may still touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ f32 FMA kernel

template <int MODE>
__global__ void __launch_bounds__(256) k_gemm_f32(const float *__restrict__ A, const float *__restrict__ B,
                                                  const EpiArgs ep, int M, int N, int K) {
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  const int lr = threadIdx.x >> 2, lc = (threadIdx.x & 3) * 4;
  for (int k0 = 0; k0 < K; k0 += 16) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    if (m0 + lr < M) a = *reinterpret_cast<const float4 *>(A + (int64_t)(m0 + lr) * K + k0 + lc);
    const float4 b = *reinterpret_cast<const float4 *>(B + (int64_t)(n0 + lr) * K + k0 + lc);
    As[lc + 0][lr] = a.x; As[lc + 1][lr] = a.y; As[lc + 2][lr] = a.z; As[lc + 3][lr] = a.w;
    Bs[lc + 0][lr] = b.x; Bs[lc + 1][lr] = b.y; Bs[lc + 2][lr] = b.z; Bs[lc + 3][lr] = b.w;
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a4[4], b4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a4[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b4[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a4[i], b4[j], acc[i][j]);
    }
    __syncthreads();
  }
  const int col = n0 + tx * 4;
  float lo = ep.lo, hi = ep.hi;
  if (ep.seg_w > 0) {
    const int sg = col / ep.seg_w;  // selects, not a runtime index into the parameter array
    lo = sg == 0 ? ep.seg_lo[0] : (sg == 1 ? ep.seg_lo[1] : ep.seg_lo[2]);
    hi = sg == 0 ? ep.seg_hi[0] : (sg == 1 ? ep.seg_hi[1] : ep.seg_hi[2]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = m0 + ty * 4 + i;
    if (row >= M) continue;
    float v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float x = acc[i][j];
      if (MODE == EPI_F32 && ep.bias) x += ep.bias[col + j];
      x = clampf(x, lo, hi);
      if (MODE == EPI_SILU) x = clampf(x / (1.0f + expf(-x)), ep.lo2, ep.hi2);
      v[j] = x;
    }
    float *o = static_cast<float *>(ep.out) + (int64_t)row * ep.ld;
    if (MODE == EPI_GLU) {
      o[col / 2] = v[0] / (1.0f + expf(-v[1]));
      o[col / 2 + 1] = v[2] / (1.0f + expf(-v[3]));
    } else if (MODE == EPI_ADD_F32) {
      float4 *p = reinterpret_cast<float4 *>(o + col);
      const float4 h = *p;
      *p = make_float4(h.x + v[0], h.y + v[1], h.z + v[2], h.w + v[3]);
    } else {
      *reinterpret_cast<float4 *>(o + col) = make_float4(v[0], v[1], v[2], v[3]);
    }
  }
}

// ------------------------------------------------------------------ host side

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool make_tmap_2d_bf16(CUtensorMap *tm, const void *base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                       uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_2d_u8(CUtensorMap *tm, const void *base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                     uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Stem conv0 output viewed as 5-D for the implicit GEMM of conv1:
// (c 128, fpar 2, fp 32, tpar 2, tp rows/2), boxes (64, 1, 32, 1, 4).
bool make_tmap_stem_y0(CUtensorMap *tm, const void *y0, int64_t stem_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[5] = {(cuuint64_t)kC0, 2, (cuuint64_t)kF1 / 2, 2, (cuuint64_t)(stem_rows / 2)};
  cuuint64_t strides[4] = {(cuuint64_t)kC0 * 2, (cuuint64_t)kC0 * 2 * 2, (cuuint64_t)kF1 * kC0 * 2,
                           (cuuint64_t)kF1 * kC0 * 2 * 2};
  cuuint32_t box[5] = {64, 1, 32, 1, (cuuint32_t)kConv1TileTok};
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(y0), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int num_sms() {
  static std::atomic<int> n[64];
  int dev = 0;
  cudaGetDevice(&dev);
  int v = 0;
  if (dev >= 0 && dev < 64) v = n[dev].load(std::memory_order_relaxed);
  if (!v) {
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    if (dev >= 0 && dev < 64 && v > 0) n[dev].store(v, std::memory_order_relaxed);
  }
  return v > 0 ? v : 1;
}

template <int MODE, bool F8 = false>
static cudaError_t launch_tc(const CUtensorMap &tA, const CUtensorMap &tB, const EpiArgs &ep, int M, int N, int K,
                             cudaStream_t s) {
  static std::atomic<uint64_t> attr{0};
  if (const cudaError_t e = smem_attr(k_gemm_tc<MODE, F8>, smem_of(MODE), attr)) return e;
  const int tiles = ((M + 2 * BM - 1) / (2 * BM)) * (N / BN);
  const int pairs = tiles < num_sms() / 2 ? tiles : num_sms() / 2;
  return launch_k(k_gemm_tc<MODE, F8>, dim3(2 * pairs), dim3(GEMM_THREADS), smem_of(MODE), s, tA, tB, ep, M, N, K,
                  device_status_word());
}

template <int MODE>
static cudaError_t launch_f32(const float *x, const float *w, const EpiArgs &ep, int M, int N, int K,
                              cudaStream_t s) {
  dim3 grid(N / 64, (M + 63) / 64);
  return launch_k(k_gemm_f32<MODE>, grid, dim3(256), 0, s, x, w, ep, M, N, K);
}

cudaError_t gemm(const ae_model *m, const void *x, int64_t M, int K, const void *w, const CUtensorMap *tmW, int N,
                 int mode, const EpiArgs &ep, cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  if (m->dtype != AE_F32) {
    CUtensorMap tA, tB;
    if (!make_tmap_2d_bf16(&tA, x, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, BK, BM)) return cudaErrorInvalidValue;
    if (!tmW) {
      if (!make_tmap_2d_bf16(&tB, w, (uint64_t)K, (uint64_t)N, (uint64_t)K * 2, BK, BN / 2))
        return cudaErrorInvalidValue;
      tmW = &tB;
    }
    switch (mode) {
      case EPI_F32: return launch_tc<EPI_F32>(tA, *tmW, ep, (int)M, N, K, s);
      case EPI_ADD_F32: return launch_tc<EPI_ADD_F32>(tA, *tmW, ep, (int)M, N, K, s);
      case EPI_BF16: return launch_tc<EPI_BF16>(tA, *tmW, ep, (int)M, N, K, s);
      case EPI_SILU: return launch_tc<EPI_SILU>(tA, *tmW, ep, (int)M, N, K, s);
      case EPI_GLU: return launch_tc<EPI_GLU>(tA, *tmW, ep, (int)M, N, K, s);
    }
    return cudaErrorInvalidValue;
  }
  const float *xf = static_cast<const float *>(x);
  const float *wf = static_cast<const float *>(w);
  switch (mode) {
    case EPI_F32: return launch_f32<EPI_F32>(xf, wf, ep, (int)M, N, K, s);
    case EPI_ADD_F32: return launch_f32<EPI_ADD_F32>(xf, wf, ep, (int)M, N, K, s);
    case EPI_BF16: return launch_f32<EPI_BF16>(xf, wf, ep, (int)M, N, K, s);
    case EPI_SILU: return launch_f32<EPI_SILU>(xf, wf, ep, (int)M, N, K, s);
    case EPI_GLU: return launch_f32<EPI_GLU>(xf, wf, ep, (int)M, N, K, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t gemm_bf16(const void *x, int64_t M, int K, const CUtensorMap &tmW, int N, int mode, const EpiArgs &ep,
                      cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  if (K % BK || N % BN || M > INT32_MAX) return cudaErrorInvalidValue;
  CUtensorMap tA;
  if (!make_tmap_2d_bf16(&tA, x, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, BK, BM)) return cudaErrorInvalidValue;
  switch (mode) {
    case EPI_F32: return launch_tc<EPI_F32>(tA, tmW, ep, (int)M, N, K, s);
    case EPI_BF16: return launch_tc<EPI_BF16>(tA, tmW, ep, (int)M, N, K, s);
    case EPI_BIAS_BF16: return launch_tc<EPI_BIAS_BF16>(tA, tmW, ep, (int)M, N, K, s);
    case EPI_BIAS_SILU: return launch_tc<EPI_BIAS_SILU>(tA, tmW, ep, (int)M, N, K, s);
    case EPI_BIAS_GLU: return launch_tc<EPI_BIAS_GLU>(tA, tmW, ep, (int)M, N, K, s);
    case EPI_BIAS_GELU: return launch_tc<EPI_BIAS_GELU>(tA, tmW, ep, (int)M, N, K, s);
    case EPI_BIAS_ADD_F32: return launch_tc<EPI_BIAS_ADD_F32>(tA, tmW, ep, (int)M, N, K, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t gemm_e4m3(const void *x, int64_t M, int K, const CUtensorMap &tmW, int N, int mode, const EpiArgs &ep,
                      cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  if (K % (2 * BK) || N % BN || !ep.cs) return cudaErrorInvalidValue;
  CUtensorMap tA;
  if (!make_tmap_2d_u8(&tA, x, (uint64_t)K, (uint64_t)M, (uint64_t)K, 2 * BK, BM)) return cudaErrorInvalidValue;
  switch (mode) {
    case EPI_BF16: return launch_tc<EPI_BF16, true>(tA, tmW, ep, (int)M, N, K, s);
    case EPI_GLU: return launch_tc<EPI_GLU, true>(tA, tmW, ep, (int)M, N, K, s);
    case EPI_SILU_Q8: return launch_tc<EPI_SILU_Q8, true>(tA, tmW, ep, (int)M, N, K, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace ae
