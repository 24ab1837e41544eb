// Second log-mel front-end: the LFM2A audio encoder's, as the page of its GPU
// port lays it out (log_mel_spectrogram_gpu: stft_frames, power_spec,
// mel_project, mel_norm). Frames of 512 samples every `hop` samples with 256
// samples of zero padding per side, pre-emphasis y[n] = x[n] - p x[n-1] on the
// clip (x[-1] = 0), a periodic Hann window of `win_length` centred in the
// 512-wide frame, the power spectrum |X_k|^2 (k = 0..256), a Slaney mel
// filterbank, ln(max(mel, floor)), then per band (v - mean) / sqrt(var + eps)
// with the statistics of the frames whose centre lies in the clip and zeros
// for the others.
//
// k_lfm_spec: persistent CTAs of 256 threads, two per SM; the work item is 32
// consecutive frames of one clip. Per item:
//
//  1. Staging. The raw samples the frames cover, and the one before them,
//     are copied into shared memory with cp.async (16 bytes at a time, placed
//     so that 16-byte source chunks land on 16-byte boundaries; 4-byte copies
//     for the chunks cut by a clip boundary, zeros outside the clip). The next
//     item's copy is issued as soon as the current item's spectra are done, so
//     it is in flight during the band, statistics and store phases.
//  2. Spectra: 16 groups of 16 threads, two frames per group. The pre-emphasis
//     is applied as the frame is read (the one sample just past the clip end,
//     which would see the last sample as its predecessor, is masked), then the
//     512 windowed values are packed as 256 complex values z[n] = v[2n] +
//     i v[2n+1] and transformed by the four-step 16 x 16 FFT (fft16.cuh); the
//     real spectrum follows from X[k] = A - i W512^k B, X[256 - k] =
//     conj(A + i W512^k B), A = Z[k] + conj Z[256 - k], B = Z[k] - conj
//     Z[256 - k], the partner Z coming from the mirror thread by one shuffle
//     (the window carries the 1/2). The 257 powers go to a [frame][bin] tile.
//  3. Bands: one frame per lane; warp w takes a contiguous run of bands
//     (balanced by work on the host), each band its nonzero bins from a
//     packed table (weights read as warp-wide broadcasts), then the floored
//     log with the hardware's base-2 logarithm.
//  4. Statistics and store: thread b sums band b over the item's frames that
//     count (float64, frame order) and adds the sums, rounded to multiples of
//     2^-24, into the clip's 64-bit integer accumulators: integer addition is
//     associative, so the totals do not depend on the order in which the
//     items finish. The rows leave as whole contiguous rows.
//
// k_lfm_norm: one CTA per item of 32 rows; thread b loads its column of the
// rows, turns the clip's accumulators into the mean and biased variance of
// band b (float64) and rewrites the rows in place, zeros for the frames past
// the statistics.
#include <cstddef>

#include "ae_internal.h"
#include "common.cuh"
#include "fft16.cuh"

namespace ae {

namespace {
constexpr int kLfmFft = 512;
constexpr int kLfmGroups = 16;              // 16-thread FFT groups
constexpr int kLfmThreads = kLfmGroups * 16;
constexpr int kLfmPitch = 17;               // padded row of the 16 x 16 transpose (float2)
constexpr int kLfmBins = kLfmFft / 2 + 1;   // 257: odd row pitch of the power tile
constexpr int kLfmOutPitch = kLfmMaxMels + 1;
constexpr int kLfmRecs = 64;
constexpr double kMomentScale = 16777216.0;  // 2^24: the accumulators' unit is 2^-24

static_assert(kLfmTile == 2 * kLfmGroups && kLfmTile == 32, "two frames per FFT group, one per lane in the bands");
static_assert(kLfmWarps * 32 == kLfmThreads, "band phase warps");

// Where an item's samples come from and its rows go, resolved for a run of the
// CTA's items at once.
struct LfmRec {
  long long first;       // wave index of the item's local sample 0 (padded position f0 hop, clip sample f0 hop - 256)
  int out_row;           // output row of the item's first frame
  int clip;
  unsigned short lo, hi;  // local samples [lo, hi) lie inside the clip (hi at most the item's span)
  unsigned char nf;      // frames in the item
  unsigned char nstat;   // of those, the ones that count for the statistics (a prefix)
};

struct LfmSmem {
  union {
    float2 xs[kLfmGroups][16 * kLfmPitch];    // per-group transpose tiles (spectra phase)
    float out[kLfmTile][kLfmOutPitch];        // log-mel rows (band, statistics and store phases)
  } u;
  float pw[kLfmTile][kLfmBins];               // power spectra
  float win[kLfmFft];                         // padded periodic Hann / 2
  float2 wk[8][16];                           // W512^(j + 16 k2) at [k2][j]
  int blo[kLfmMaxMels], bcnt[kLfmMaxMels], boff[kLfmMaxMels];
  int wband[kLfmWarps + 4];                   // the warps' band runs (padded to 16 bytes)
  LfmRec rec[kLfmRecs];
  // dynamic tail: staged samples (wave_floats), then the packed weights (nnz)
};
static_assert(sizeof(LfmSmem) % 16 == 0 && offsetof(LfmSmem, win) % 8 == 0, "tail and window alignment");

__device__ __forceinline__ void lfm_cp4(float *dst, const float *src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d), "l"(src) : "memory");
}

__device__ __forceinline__ void lfm_cp16(float *dst, const float *src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}

// ln(max(x, floor)) with the hardware's base-2 logarithm
__device__ __forceinline__ float lfm_log(float x, float floor) {
  float l2;
  asm("lg2.approx.f32 %0, %1;" : "=f"(l2) : "f"(fmaxf(x, floor)));
  return l2 * 0.69314718055994531f;
}
}  // namespace

size_t lfm_smem_bytes(const LfmParams &prm) {
  return sizeof(LfmSmem) + sizeof(float) * ((size_t)prm.wave_floats + (size_t)prm.nnz);
}

__global__ void __launch_bounds__(kLfmThreads, 2)
    k_lfm_spec(const float *__restrict__ wave, float *__restrict__ out, const LfmTablesDev t, const LfmParams prm) {
  extern __shared__ __align__(16) uint8_t lfm_smem_raw[];
  LfmSmem &S = *reinterpret_cast<LfmSmem *>(lfm_smem_raw);
  float *sw = reinterpret_cast<float *>(lfm_smem_raw + sizeof(LfmSmem));  // staged samples
  float *bw = sw + prm.wave_floats;                                       // packed band weights
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = tid >> 4, j = tid & 15;
  const unsigned gmask = 0xFFFFu << (16 * (g & 1));
  const int hop = prm.hop;

  // ---- per-CTA tables
  for (int m = tid; m < kLfmFft; m += kLfmThreads) {
    const int lo = (kLfmFft - prm.win_length) / 2, i = m - lo;
    S.win[m] = (i >= 0 && i < prm.win_length) ? (float)(0.25 - 0.25 * cospi(2.0 * i / prm.win_length)) : 0.f;
  }
  for (int e = tid; e < 8 * 16; e += kLfmThreads) {  // e = 16 k2 + j
    double s, c;
    sincospi((double)((e & 15) + 16 * (e >> 4)) / 256.0, &s, &c);
    S.wk[e >> 4][e & 15] = make_float2((float)c, (float)-s);
  }
  for (int b = tid; b < kLfmMaxMels; b += kLfmThreads) {
    const bool live = b < prm.n_mels;
    S.blo[b] = live ? t.bank_lo[b] : 0;
    S.bcnt[b] = live ? t.bank_cnt[b] : 0;
    S.boff[b] = live ? t.bank_off[b] : 0;
  }
  for (int q = tid; q < prm.nnz; q += kLfmThreads) bw[q] = t.bank_w[q];
  if (tid == 0) {
#pragma unroll
    for (int w = 0; w <= kLfmWarps; ++w) S.wband[w] = prm.wband[w];
  }
  float2 tw1[16];  // W256^(j k1) = W512^(2 j k1), float32 (within an ulp or so)
#pragma unroll
  for (int k1 = 0; k1 < 16; ++k1) {
    float s, c;
    sincospif((float)((2 * j * k1) & (kLfmFft - 1)) / 256.0f, &s, &c);
    tw1[k1] = make_float2(c, -s);
  }

  // this CTA's items are tiles blockIdx.x + k gridDim.x, k < my_tiles
  const int my_tiles = (int)blockIdx.x < t.n_tiles ? (t.n_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  auto fill = [&](int base) {  // records of items base .. base + kLfmRecs - 1
    for (int k = tid; k < kLfmRecs && base + k < my_tiles; k += kLfmThreads) {
      const int tile = (int)blockIdx.x + (base + k) * (int)gridDim.x;
      int lo = 0, hi = t.n_clips;  // last clip whose first tile is <= tile
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (t.tile_off[mid] <= tile) lo = mid; else hi = mid;
      }
      const int f0 = (tile - t.tile_off[lo]) * kLfmTile;
      const int nf = min(kLfmTile, t.frame_off[lo + 1] - t.frame_off[lo] - f0);
      const int64_t s0 = t.sample_off[lo], n = t.sample_off[lo + 1] - s0;
      const int64_t rel = (int64_t)f0 * hop - kLfmFft / 2;  // clip sample of local sample 0
      const int64_t span = (int64_t)(nf - 1) * hop + kLfmFft;
      LfmRec r;
      r.first = s0 + rel;
      r.out_row = t.frame_off[lo] + f0;
      r.clip = lo;
      r.lo = (unsigned short)min(span, max((int64_t)0, -rel));
      r.hi = (unsigned short)min(span, max((int64_t)0, n - rel));
      r.nf = (unsigned char)nf;
      r.nstat = (unsigned char)max(0, min(nf, t.eff[lo] - f0));
      S.rec[k] = r;
    }
  };
  // ---- stage an item: smem index u holds wave index a0 + u, a0 = first - 1 - d
  // rounded down to a multiple of 4, so local sample i (and its predecessor at
  // i - 1) sits at u = i + 1 + d; zeros outside the clip
  auto stage = [&](const LfmRec &r) {
    const int span = (r.nf - 1) * hop + kLfmFft;
    const int d = (int)((r.first - 1) & 3);
    const int ext = span + 1 + d;
    const float *src = wave + (r.first - 1 - d);  // dereferenced only inside the clip
    const int ulo = r.lo + 1 + d, uhi = r.hi + 1 + d;
    if (prm.vec16) {
      for (int u = 4 * tid; u < ext; u += 4 * kLfmThreads) {
        if (u >= ulo && u + 4 <= uhi) {
          lfm_cp16(sw + u, src + u);
        } else if (u + 4 <= ulo || u >= uhi) {
          *reinterpret_cast<float4 *>(sw + u) = make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (u + e >= ulo && u + e < uhi) lfm_cp4(sw + u + e, src + u + e);
            else sw[u + e] = 0.f;
          }
        }
      }
    } else {
      for (int u = tid; u < ext; u += kLfmThreads) {
        if (u >= ulo && u < uhi) lfm_cp4(sw + u, src + u);
        else sw[u] = 0.f;
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  fill(0);
  __syncthreads();
  if (my_tiles > 0) stage(S.rec[0]);

  for (int k = 0; k < my_tiles; ++k) {
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();  // this item's samples visible; the previous item's rows are stored
    const LfmRec cur = S.rec[k % kLfmRecs];
    const int nf = cur.nf;
    const int d = (int)((cur.first - 1) & 3);

    // ---- spectra: frames g and g + 16 of the item
    float2 *xs = S.u.xs[g];
    for (int fi = g; fi < nf; fi += kLfmGroups) {
      const float *wv = sw + fi * hop + d + 2 * j;  // wv[m] = x(local fi hop + 2 j + m - 1)
      const float p = prm.preemph;
      float2 xv[16];
#pragma unroll
      for (int n1 = 0; n1 < 16; ++n1) {
        const float xm = wv[32 * n1], x0 = wv[32 * n1 + 1], x1 = wv[32 * n1 + 2];
        const float2 w = *reinterpret_cast<const float2 *>(S.win + 32 * n1 + 2 * j);
        xv[n1] = make_float2(fmaf(-p, xm, x0) * w.x, fmaf(-p, x0, x1) * w.y);
      }
      // the sample just past the clip end is zero padding, not x - p x_prev (when
      // the clip goes on past the item, hi is the span, which no frame reaches)
      const int rel = (int)cur.hi - fi * hop;
      if (rel >= 0 && rel < kLfmFft) {  // uniform across the group
#pragma unroll
        for (int n1 = 0; n1 < 16; ++n1) {
          const int m = 32 * n1 + 2 * j;
          if (m == rel) xv[n1].x = 0.f;
          if (m + 1 == rel) xv[n1].y = 0.f;
        }
      }
      dft16(xv);
#pragma unroll
      for (int k1 = 1; k1 < 16; ++k1) xv[k1] = cmul(xv[k1], tw1[k1]);
#pragma unroll
      for (int k1 = 0; k1 < 16; ++k1) xs[k1 * kLfmPitch + j] = xv[k1];
      __syncwarp(gmask);
#pragma unroll
      for (int n2 = 0; n2 < 16; ++n2) xv[n2] = xs[j * kLfmPitch + n2];
      dft16(xv);  // xv[k2] = Z[j + 16 k2]
      float *pr = S.pw[fi];
      const int partner = (lane & 16) | ((16 - j) & 15);
#pragma unroll
      for (int k2 = 0; k2 < 8; ++k2) {
        const float2 o = xv[k2];
        float2 mr;
        mr.x = __shfl_sync(gmask, xv[15 - k2].x, partner);
        mr.y = __shfl_sync(gmask, xv[15 - k2].y, partner);
        if (j == 0) mr = xv[(16 - k2) & 15];  // thread 0 pairs 16 k2 with 16 (16 - k2), k2 = 0 with itself
        const float2 mc = make_float2(mr.x, -mr.y);  // conj Z[256 - k]
        const float2 A = cadd(o, mc), B = csub(o, mc);
        const float2 wb = cmul(B, S.wk[k2][j]);      // W512^(j + 16 k2) B
        const float2 P = make_float2(-wb.y, wb.x);   // i W B
        const float2 x1 = csub(A, P), x2 = cadd(A, P);  // X[k], conj X[256 - k]
        const float2 q1 = __fmul2_rn(x1, x1), q2 = __fmul2_rn(x2, x2);
        const int kk = j + 16 * k2;
        pr[kk] = q1.x + q1.y;
        pr[kLfmFft / 2 - kk] = q2.x + q2.y;
      }
      if (j == 0) pr[kLfmFft / 4] = 4.0f * fmaf(xv[8].x, xv[8].x, xv[8].y * xv[8].y);  // |X[128]| = 2 |Z[128]|
      __syncwarp(gmask);  // the tile is free for the next frame
    }
    __syncthreads();  // powers complete; the staged samples are free

    // ---- the next item's samples load during the rest of this item
    if (k + 1 < my_tiles) {
      if ((k + 1) % kLfmRecs == 0) {  // the next run of records (uniform across the CTA)
        fill(k + 1);
        __syncthreads();
      }
      stage(S.rec[(k + 1) % kLfmRecs]);
    }

    // ---- bands: lane = frame
    if (lane < nf) {
      const float *prow = S.pw[lane];
      float *orow = S.u.out[lane];
      const int b1 = S.wband[warp + 1];
      for (int b = S.wband[warp]; b < b1; ++b) {
        const float *p = prow + S.blo[b];
        const float *w = bw + S.boff[b];
        const int cnt = S.bcnt[b];
        float acc = 0.f;
#pragma unroll 4
        for (int q = 0; q < cnt; ++q) acc = fmaf(w[q], p[q], acc);
        orow[b] = lfm_log(acc, prm.log_floor);
      }
    }
    __syncthreads();  // rows complete

    // ---- statistics of the frames that count, then the rows
    if (tid < prm.n_mels && cur.nstat > 0) {
      double s1 = 0.0, s2 = 0.0;
      for (int f = 0; f < cur.nstat; ++f) {
        const double v = (double)S.u.out[f][tid];
        s1 += v;
        s2 = fma(v, v, s2);
      }
      unsigned long long *a = t.moments + 2 * ((size_t)cur.clip * kLfmMaxMels + tid);
      atomicAdd(a, (unsigned long long)__double2ll_rn(s1 * kMomentScale));
      atomicAdd(a + 1, (unsigned long long)__double2ll_rn(s2 * kMomentScale));
    }
    const int c = tid & (kLfmMaxMels - 1), r0 = tid >> 7;
    if (c < prm.n_mels) {
      float *orow = out + (int64_t)cur.out_row * prm.n_mels + c;
#pragma unroll
      for (int q = 0; q < kLfmTile; q += kLfmThreads / kLfmMaxMels)
        if (r0 + q < nf) orow[(int64_t)(r0 + q) * prm.n_mels] = S.u.out[r0 + q][c];
    }
  }
}

__global__ void __launch_bounds__(256, 4) k_lfm_norm(float *__restrict__ out, const LfmTablesDev t, const LfmParams prm) {
  const int tile = blockIdx.x;
  const int c = threadIdx.x & (kLfmMaxMels - 1), r0 = threadIdx.x >> 7;
  if (c >= prm.n_mels) return;
  int lo = 0, hi = t.n_clips;  // last clip whose first tile is <= tile
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (t.tile_off[mid] <= tile) lo = mid; else hi = mid;
  }
  const int f0 = (tile - t.tile_off[lo]) * kLfmTile;
  const int nf = min(kLfmTile, t.frame_off[lo + 1] - t.frame_off[lo] - f0);
  float *p = out + ((int64_t)t.frame_off[lo] + f0) * prm.n_mels + c;
  float v[kLfmTile / 2];
#pragma unroll
  for (int q = 0; q < kLfmTile / 2; ++q) {
    const int f = r0 + 2 * q;
    v[q] = f < nf ? p[(int64_t)f * prm.n_mels] : 0.f;
  }
  const int eff = t.eff[lo];
  const unsigned long long *a = t.moments + 2 * ((size_t)lo * kLfmMaxMels + c);
  const double n = eff > 0 ? (double)eff : 1.0;
  const double mean = (double)(long long)a[0] / kMomentScale / n;
  const double var = fmax(0.0, (double)(long long)a[1] / kMomentScale / n - mean * mean);
  const double inv = 1.0 / sqrt(var + (double)prm.var_eps);
#pragma unroll
  for (int q = 0; q < kLfmTile / 2; ++q) {
    const int f = r0 + 2 * q;
    if (f < nf) p[(int64_t)f * prm.n_mels] = f0 + f < eff ? (float)(((double)v[q] - mean) * inv) : 0.f;
  }
}

cudaError_t launch_lfm(const float *wave, float *out, const LfmTablesDev &t, const LfmParams &prm, cudaStream_t s) {
  if (t.n_tiles <= 0) return cudaSuccess;
  const size_t smem = lfm_smem_bytes(prm);
  cudaError_t e = cudaFuncSetAttribute(k_lfm_spec, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_lfm_spec, kLfmThreads, smem)) != cudaSuccess)
    return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int64_t slots = (int64_t)per_sm * sms;
  const int grid = (int)(t.n_tiles < slots ? t.n_tiles : slots);
  if ((e = cudaMemsetAsync(t.moments, 0, sizeof(unsigned long long) * 2 * kLfmMaxMels * (size_t)t.n_clips, s)) !=
      cudaSuccess)
    return e;
  if ((e = launch_k(k_lfm_spec, dim3((unsigned)grid), dim3(kLfmThreads), smem, s, wave, out, t, prm)) != cudaSuccess)
    return e;
  return launch_k(k_lfm_norm, dim3((unsigned)t.n_tiles), dim3(256), 0, s, out, t, prm);
}

}  // namespace ae
