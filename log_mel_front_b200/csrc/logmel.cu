// Log-mel front-end (egemma2_audio.rs, MelFrontend::log_mel), fused in one
// kernel: framing with the 160-sample semicausal pad, periodic Hann window,
// 512-point real FFT, magnitude, 128-band HTK mel projection and
// ln(mel + 0.001).
//
// Work item: 32 consecutive frames of one clip; one CTA of 256 threads per
// item at a time, two CTAs per SM, persistent over the items. Per item:
//
//  1. Staging. The contiguous waveform span of the 32 frames (33 x 160
//     samples) is copied into shared memory with cp.async, zero fill outside
//     the clip (the semicausal pad and the clip end), into one of two buffers:
//     the next item's copy is issued when an item starts, so it is in flight
//     during the whole item. The copies are 16 bytes wide where the span
//     starts on a 16-byte boundary (every item of a clip whose first sample
//     does), else 4 bytes wide.
//  2. Spectra: 16 groups of 16 threads, two frames per group. A frame's 320
//     windowed samples are packed as 160 complex values z[n] = x[2n] +
//     i x[2n+1] and transformed by a 256-point complex FFT in the four-step
//     form 16 x 16: thread j does the DFT-16 over n1 of z[16 n1 + j] in
//     registers (10 of its 16 inputs are nonzero), multiplies by W256^(j k1),
//     the group transposes through a padded shared-memory tile, and thread j
//     does the DFT-16 that yields Z[j + 16 k2]. The real spectrum follows from
//     X[k] = A - i W512^k B and X[256 - k] = conj(A + i W512^k B), with
//     A = Z[k] + conj Z[256 - k], B = Z[k] - conj Z[256 - k]: thread j takes
//     the pairs of its k2 < 8, Z[256 - k] coming from thread 16 - j by one
//     shuffle per pair (threads 0 and 8 hold both members); the W512^k come
//     from a per-CTA table. The window carries the split's factor 1/2. The 257
//     magnitudes (the hardware square root of |X|^2) go to a [frame][bin] tile.
//  3. Bands: one frame per lane. Warp w computes the bands [kWarpBand[w],
//     kWarpBand[w+1]) of the 32 frames as straight-line code with the HTK
//     weights as literals (htk_bank.h, 506 multiply-adds per frame, split
//     evenly over the warps), reading the magnitudes from the tile (odd row
//     pitch: lane f reads row f without bank conflicts), then the log.
//  4. Store: the [32][128] result leaves as whole contiguous rows, thread t
//     storing column t mod 128 of every other row.
//
// Per-thread constants (the window values and FFT twiddles it uses) are
// computed once at kernel start in float32 (sincospif / cospif, within an
// ulp or so of the float64 values). The log is ln(2) log2(x) with the
// hardware's base-2 logarithm, within 1e-5 of ln(x) for the values that
// occur (x >= 0.001).
#include "ae_internal.h"
#include "common.cuh"
#include "fft16.cuh"

namespace ae {

// ln(acc + 0.001) for acc >= 0: the hardware's base-2 logarithm (within a few
// ulp of the result for the arguments that occur, x >= 0.001), times ln 2.
__device__ __forceinline__ float log_floor_sum(float acc) {
  float l2;
  asm("lg2.approx.f32 %0, %1;" : "=f"(l2) : "f"(acc + 1e-3f));
  return l2 * 0.69314718055994531f;
}

}  // namespace ae

#include "htk_bank.h"

namespace ae {

namespace {
constexpr int kItem = kMelTile;                // frames per work item (32)
constexpr int kThreads = 256;
constexpr int kGroups = kThreads / 16;         // 16-thread FFT groups
constexpr int kSpan = kItem * kHop + kHop;     // staged samples per item
constexpr int kPitch = 17;                     // padded row of the 16 x 16 transpose (float2)
constexpr int kMagPitch = 273;                 // odd: the band phase reads column k of 32 rows conflict-free
constexpr int kOutPitch = 129;
constexpr int kBins = kFft / 2 + 1;

static_assert(kItem == 32 && kGroups * 2 == kItem, "one frame per lane in the band phase, two per FFT group");

// Where an item's samples come from and its rows go: resolved for a run of the
// CTA's items at once (one clip search per thread, in parallel), so that no
// item waits on a chain of dependent table loads.
struct TileRec {
  long long first;    // index in the wave array of the item's local sample 0 (before the clip for frame 0)
  int out_row;        // output row of the item's first frame
  unsigned short hi;  // local samples [lo, hi) lie inside the clip
  unsigned char pad;  // 1: the item starts at frame 0, lo = kHop (the semicausal pad); 0: lo = 0
  unsigned char nf;   // frames in the item
};
constexpr int kRecs = 128;

struct LogmelSmem {
  float wave[2][kSpan];                        // this item's samples and the next one's (in flight)
  union {
    float2 xs[kGroups][16 * kPitch];           // per-group transpose tiles (spectra phase)
    float out[kItem][kOutPitch];               // log-mel rows (band and store phases)
  } u;
  float mag[kItem][kMagPitch];
  float2 wk[8][16];                            // W512^(j + 16 k2) at [k2][j]: the split's twiddles
  TileRec rec[kRecs];                          // the CTA's items kRecs at a time
};
static_assert(sizeof(TileRec) == 16, "tile record");
static_assert(2 * (sizeof(LogmelSmem) + 1024) <= 228 * 1024, "two CTAs per SM");

__device__ __forceinline__ void cp_async4(float *dst, const float *src, bool valid) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  const int n = valid ? 4 : 0;  // src-size 0: 4 zero bytes
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(d), "l"(src), "r"(n) : "memory");
}

// 16-byte copy of which the first nbytes come from src and the rest are zero
__device__ __forceinline__ void cp_async16(float *dst, const float *src, int nbytes) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(nbytes) : "memory");
}

// |X| from |X|^2 >= 0: the hardware square root (0 for 0)
__device__ __forceinline__ float magnitude(float sq) {
  float r;
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(sq));
  return r;
}

struct Item {
  int clip, f0, nf;
};

__device__ __forceinline__ Item item_of(const ClipTablesDev &t, int tile) {
  int lo = 0, hi = t.n_clips;  // last clip c with mel_tile_off[c] <= tile
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (t.mel_tile_off[mid] <= tile) lo = mid; else hi = mid;
  }
  Item it;
  it.clip = lo;
  it.f0 = (tile - t.mel_tile_off[lo]) * kItem;
  it.nf = min(kItem, t.frame_off[lo + 1] - t.frame_off[lo] - it.f0);
  return it;
}

template <int W>
__device__ __forceinline__ void band_phase(const LogmelSmem &S, LogmelSmem &D, int f) {
  htk::bands<W>(S.mag[f], D.u.out[f]);
}
}  // namespace

__global__ void __launch_bounds__(kThreads, 2)
    k_logmel(const float *__restrict__ wave, float *__restrict__ mel, const ClipTablesDev t, int n_tiles) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  LogmelSmem &S = *reinterpret_cast<LogmelSmem *>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = tid >> 4, j = tid & 15;
  const unsigned gmask = 0xFFFFu << (16 * (g & 1));

  // ---- per-thread constants
  float2 win[10];  // Hann / 2 at samples 32 n1 + 2 j and + 1 (the split's 1/2 folded in)
#pragma unroll
  for (int n1 = 0; n1 < 10; ++n1) {
    const int m = 32 * n1 + 2 * j;
    win[n1] = make_float2(0.25f - 0.25f * cospif((float)m / 160.0f), 0.25f - 0.25f * cospif((float)(m + 1) / 160.0f));
  }
  float2 tw1[16];  // W256^(j k1) = W512^(2 j k1)
#pragma unroll
  for (int k1 = 0; k1 < 16; ++k1) {
    float s, c;
    sincospif((float)((2 * j * k1) & (kFft - 1)) / 256.0f, &s, &c);
    tw1[k1] = make_float2(c, -s);
  }
  for (int e = tid; e < 8 * 16; e += kThreads) {  // W512^(j + 16 k2), e = 16 k2 + j
    float s, c;
    sincospif((float)((e & 15) + 16 * (e >> 4)) / 256.0f, &s, &c);
    S.wk[e >> 4][e & 15] = make_float2(c, -s);
  }

  // this CTA's items are tiles blockIdx.x + k gridDim.x, k < my_tiles
  const int my_tiles = (int)blockIdx.x < n_tiles ? (n_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  auto fill = [&](int base) {  // records of items base .. base + kRecs - 1
    for (int k = tid; k < kRecs && base + k < my_tiles; k += kThreads) {
      const Item x = item_of(t, (int)blockIdx.x + (base + k) * (int)gridDim.x);
      const int64_t s_begin = t.sample_off[x.clip];
      const int64_t n_samp = min(t.sample_off[x.clip + 1] - s_begin, (int64_t)kMaxSamples);
      const int64_t first = (int64_t)(x.f0 - 1) * kHop;  // local sample i is clip sample first + i
      const int64_t span = x.nf * kHop + kHop;
      TileRec r;
      r.first = s_begin + first;
      r.out_row = t.frame_off[x.clip] + x.f0;
      r.hi = (unsigned short)max((int64_t)0, min(span, n_samp - first));
      r.pad = first < 0 ? 1 : 0;
      r.nf = (unsigned char)x.nf;
      S.rec[k] = r;
    }
  };
  // ---- stage an item: its waveform span, zero outside the clip
  auto stage = [&](const TileRec &r, int buf) {
    const int span = r.nf * kHop + kHop, lo = r.pad ? kHop : 0, hi = r.hi;
    const float *src = wave + r.first;
    float *dst = S.wave[buf];
    if ((reinterpret_cast<uintptr_t>(src) & 15) == 0) {
      // span and lo are multiples of 4: a chunk is outside [lo, hi), inside, or cut by hi
      const float *any = src + lo;  // an aligned address for the chunks that read nothing
#pragma unroll 2
      for (int i = 4 * tid; i < span; i += 4 * kThreads) {
        const int nb = i < lo ? 0 : 4 * max(0, min(4, hi - i));
        cp_async16(dst + i, nb ? src + i : any, nb);
      }
    } else {
      for (int i = tid; i < span; i += kThreads) {
        const bool ok = i >= lo && i < hi;
        cp_async4(dst + i, ok ? src + i : wave, ok);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  fill(0);
  __syncthreads();
  if (my_tiles > 0) stage(S.rec[0], 0);

  for (int k = 0; k < my_tiles; ++k) {
    const int buf = k & 1;
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();  // this item's wave visible; the previous item's output rows are stored
    const int cur_nf = S.rec[k % kRecs].nf, cur_row = S.rec[k % kRecs].out_row;
    // ---- the next item's samples load during this whole item
    if (k + 1 < my_tiles) {
      if ((k + 1) % kRecs == 0) {  // the next run of records (uniform across the CTA)
        __syncthreads();
        fill(k + 1);
        __syncthreads();
      }
      stage(S.rec[(k + 1) % kRecs], buf ^ 1);
    }

    // ---- spectra: frames g and g + 16 of the item
    float2 *xs = S.u.xs[g];
#pragma unroll 1
    for (int fi = g; fi < cur_nf; fi += kGroups) {
      const float *wv = S.wave[buf] + fi * kHop;
      float2 x[16];
#pragma unroll
      for (int n1 = 0; n1 < 16; ++n1) {
        if (n1 < 10) {
          const float2 a = *reinterpret_cast<const float2 *>(wv + 32 * n1 + 2 * j);
          x[n1] = __fmul2_rn(a, win[n1]);
        } else {
          x[n1] = make_float2(0.f, 0.f);
        }
      }
      dft16(x);
#pragma unroll
      for (int k1 = 1; k1 < 16; ++k1) x[k1] = cmul(x[k1], tw1[k1]);
#pragma unroll
      for (int k1 = 0; k1 < 16; ++k1) xs[k1 * kPitch + j] = x[k1];
      __syncwarp(gmask);
#pragma unroll
      for (int n2 = 0; n2 < 16; ++n2) x[n2] = xs[j * kPitch + n2];
      dft16(x);  // x[k2] = Z[j + 16 k2]
      // ---- real split: pairs (k, 256 - k), k = j + 16 k2, k2 < 8
      float *mg = S.mag[fi];
      const int partner = (lane & 16) | ((16 - j) & 15);
#pragma unroll
      for (int k2 = 0; k2 < 8; ++k2) {
        const float2 o = x[k2];
        float2 mr;
        mr.x = __shfl_sync(gmask, x[15 - k2].x, partner);
        mr.y = __shfl_sync(gmask, x[15 - k2].y, partner);
        if (j == 0) mr = x[(16 - k2) & 15];  // thread 0 pairs 16 k2 with 16 (16 - k2), k2 = 0 with itself
        const float2 mc = make_float2(mr.x, -mr.y);  // conj Z[256 - k]
        const float2 A = cadd(o, mc), B = csub(o, mc);
        const float2 wb = cmul(B, S.wk[k2][j]);  // W512^(j + 16 k2) B
        // P = i W B = (-Im, Re)
        const float2 P = make_float2(-wb.y, wb.x);
        const float2 x1 = csub(A, P), x2 = cadd(A, P);  // X[k], conj X[256 - k]
        const float2 q1 = __fmul2_rn(x1, x1), q2 = __fmul2_rn(x2, x2);
        const float m1 = q1.x + q1.y, m2 = q2.x + q2.y;
        const int k = j + 16 * k2;
        mg[k] = magnitude(m1);
        mg[kFft / 2 - k] = magnitude(m2);
      }
      if (j == 0) {
        // k = 128 is its own partner: |X[128]| = 2 |Z[128]|
        mg[kFft / 4] = 2.0f * magnitude(fmaf(x[8].x, x[8].x, x[8].y * x[8].y));
      }
      __syncwarp(gmask);  // the tile is free for the next frame
    }
    __syncthreads();  // magnitudes complete

    // ---- bands: lane = frame
    if (lane < cur_nf) {
      switch (warp) {
        case 0: band_phase<0>(S, S, lane); break;
        case 1: band_phase<1>(S, S, lane); break;
        case 2: band_phase<2>(S, S, lane); break;
        case 3: band_phase<3>(S, S, lane); break;
        case 4: band_phase<4>(S, S, lane); break;
        case 5: band_phase<5>(S, S, lane); break;
        case 6: band_phase<6>(S, S, lane); break;
        default: band_phase<7>(S, S, lane); break;
      }
    }
    __syncthreads();  // rows complete
    float *orow = mel + (int64_t)cur_row * kMels + (tid & (kMels - 1));
    const int r0 = tid >> 7;
#pragma unroll
    for (int q = 0; q < kItem; q += kThreads / kMels)
      if (r0 + q < cur_nf) orow[(r0 + q) * kMels] = S.u.out[r0 + q][tid & (kMels - 1)];
  }
}

cudaError_t launch_logmel(const float *wave, float *mel, const ClipTablesDev &t, int64_t mel_tiles,
                          cudaStream_t s) {
  if (mel_tiles <= 0) return cudaSuccess;
  const size_t smem = sizeof(LogmelSmem);
  static std::atomic<uint64_t> attr{0};
  if (const cudaError_t e = smem_attr(k_logmel, smem, attr)) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = mel_tiles < 2 * sms ? mel_tiles : 2 * sms;
  return launch_k(k_logmel, dim3((unsigned)grid), dim3(kThreads), smem, s, wave, mel, t, (int)mel_tiles);
}

}  // namespace ae
