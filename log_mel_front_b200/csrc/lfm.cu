// Second log-mel front-end: the LFM2A audio encoder's, as the page of its GPU
// port lays it out (log_mel_spectrogram_gpu: stft_frames, power_spec,
// mel_project, mel_norm). Frames of 512 samples every `hop` samples with 256
// samples of zero padding per side, pre-emphasis y[n] = x[n] - p x[n-1], a
// periodic Hann window of `win_length` centred in the 512-wide frame, the
// power spectrum |X_k|^2 (k = 0..256), a Slaney mel filterbank, ln(max(mel,
// floor)), then per band (v - mean) / sqrt(var + eps) with the statistics of
// the frames whose centre lies in the clip and zeros for the others.
//
// k_lfm_spec: the work item is 32 consecutive frames of one clip. The CTA
// stages the pre-emphasised samples those frames cover (zero outside the clip)
// in shared memory; 16 groups of 16 threads take one frame each. Per frame
// the 512 windowed samples are packed as 256 complex values z[n] = v[2n] +
// i v[2n+1] and transformed by the four-step 16 x 16 FFT (fft16.cuh); the
// real spectrum follows from the split X[k] = E[k] - i W512^k O[k] (the 1/2
// of E and O folded into the window), and each band sums only its nonzero
// bins (at most 32, listed by the host). CTAs are persistent.
//
// k_lfm_norm: one CTA per (clip, 32 bands): lane = band, the eight warps
// stride over frames; the sum and the sum of squares are accumulated in
// float64 in one pass and a fixed order (deterministic), giving the mean and
// the biased variance, and the clip's rows are rewritten in place.
#include <cstddef>

#include "ae_internal.h"
#include "common.cuh"
#include "fft16.cuh"

namespace ae {

namespace {
constexpr int kLfmFft = 512;
constexpr int kLfmGroups = 16;              // frames in flight per CTA
constexpr int kLfmThreads = kLfmGroups * 16;
constexpr int kLfmPitch = 17;
}  // namespace

struct LfmSmem {
  float2 tw[kLfmFft];                        // W512^m = (cos, -sin)(2 pi m / 512)
  float win[kLfmFft];                        // padded periodic Hann / 2
  float wts[kLfmMaxMels][kLfmMaxBins + 1];   // sparse bank (odd row pitch against bank conflicts)
  int band_lo[kLfmMaxMels];
  float2 xs[kLfmGroups][kLfmPitch * 16];
  float pw[kLfmGroups][kLfmFft / 2 + 1 + kLfmMaxBins];  // power spectrum, zero tail for the padded band loop
  int tile_clip, tile_f0, tile_nf;
  alignas(16) float wave[4];                 // staged span ((kLfmTile - 1) hop + 512 samples), sized at launch
};
static_assert(offsetof(LfmSmem, wave) % 16 == 0 && offsetof(LfmSmem, win) % 8 == 0,
              "the frame loop reads float2 pairs from the staged samples and the window");

size_t lfm_smem_bytes(int hop) {
  return sizeof(LfmSmem) + sizeof(float) * ((size_t)(kLfmTile - 1) * hop + kLfmFft);
}

__global__ void __launch_bounds__(kLfmThreads, 2)
    k_lfm_spec(const float *__restrict__ wave, float *__restrict__ out, const LfmTablesDev t, const LfmParams prm) {
  extern __shared__ __align__(16) uint8_t lfm_smem_raw[];
  LfmSmem &S = *reinterpret_cast<LfmSmem *>(lfm_smem_raw);
  const int tid = threadIdx.x;
  for (int m = tid; m < kLfmFft; m += kLfmThreads) {
    double s, c;
    sincospi((double)m / 256.0, &s, &c);  // angle 2 pi m / 512
    S.tw[m] = make_float2((float)c, (float)-s);
    const int lo = (kLfmFft - prm.win_length) / 2, i = m - lo;
    S.win[m] = (i >= 0 && i < prm.win_length) ? (float)(0.25 - 0.25 * cospi(2.0 * i / prm.win_length)) : 0.f;
  }
  for (int i = tid; i < kLfmMaxMels * (kLfmMaxBins + 1); i += kLfmThreads) {
    const int b = i / (kLfmMaxBins + 1), q = i % (kLfmMaxBins + 1);
    S.wts[b][q] = (b < prm.n_mels && q < kLfmMaxBins) ? t.bank_w[b * kLfmMaxBins + q] : 0.f;
  }
  for (int b = tid; b < kLfmMaxMels; b += kLfmThreads) S.band_lo[b] = b < prm.n_mels ? t.bank_lo[b] : 0;
  for (int x = tid; x < kLfmGroups * kLfmMaxBins; x += kLfmThreads)
    S.pw[x / kLfmMaxBins][kLfmFft / 2 + 1 + x % kLfmMaxBins] = 0.f;
  __syncthreads();

  const int g = tid >> 4, j = tid & 15;
  const unsigned gmask = 0xFFFFu << (16 * (g & 1));
  float2 tw1[16];  // W256^(j k1)
#pragma unroll
  for (int k1 = 0; k1 < 16; ++k1) tw1[k1] = S.tw[(2 * j * k1) & (kLfmFft - 1)];
  float2 *xs = S.xs[g];
  float *pw = S.pw[g];
  const int hop = prm.hop;

  for (int tile = blockIdx.x; tile < t.n_tiles; tile += gridDim.x) {
    __syncthreads();  // the previous item is done with the staged samples
    if (tid == 0) {
      int lo = 0, hi = t.n_clips;  // last clip whose first tile is <= tile
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (t.tile_off[mid] <= tile) lo = mid; else hi = mid;
      }
      S.tile_clip = lo;
      S.tile_f0 = (tile - t.tile_off[lo]) * kLfmTile;
      S.tile_nf = min(kLfmTile, t.frame_off[lo + 1] - t.frame_off[lo] - S.tile_f0);
    }
    __syncthreads();
    const int c = S.tile_clip, f0 = S.tile_f0, nf = S.tile_nf;
    const int64_t s0 = t.sample_off[c], n = t.sample_off[c + 1] - s0;
    const float *x = wave + s0;
    // local sample i is padded position f0 hop + i, clip sample f0 hop + i - 256
    const int64_t first = (int64_t)f0 * hop - kLfmFft / 2;
    const int span = (nf - 1) * hop + kLfmFft;
#pragma unroll 4
    for (int i = tid; i < span; i += kLfmThreads) {
      const int64_t sidx = first + i;
      float v = 0.f;
      if (sidx >= 0 && sidx < n) {
        const float prev = sidx > 0 ? __ldg(x + sidx - 1) : 0.f;
        v = fmaf(-prm.preemph, prev, __ldg(x + sidx));
      }
      S.wave[i] = v;
    }
    __syncthreads();

    for (int fi = g; fi < nf; fi += kLfmGroups) {
      const float *wv = S.wave + fi * hop;  // hop is even: 8-byte aligned pairs
      float2 xv[16];
#pragma unroll
      for (int n1 = 0; n1 < 16; ++n1) {
        const int m = 32 * n1 + 2 * j;
        const float2 a = *reinterpret_cast<const float2 *>(wv + m);
        const float2 w = *reinterpret_cast<const float2 *>(S.win + m);
        xv[n1] = make_float2(a.x * w.x, a.y * w.y);
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
      __syncwarp(gmask);
#pragma unroll
      for (int k2 = 0; k2 < 16; ++k2) xs[k2 * kLfmPitch + j] = xv[k2];
      __syncwarp(gmask);
      // X[k] = (Z_k + conj Z_k') - i W512^k (Z_k - conj Z_k'), k' = 256 - k (halves in the window)
#pragma unroll
      for (int k2 = 0; k2 < 16; ++k2) {
        const int k = j + 16 * k2;
        const float2 b = j == 0 ? xs[((16 - k2) & 15) * kLfmPitch] : xs[(15 - k2) * kLfmPitch + (16 - j)];
        const float2 a = xv[k2];
        const float2 A = make_float2(a.x + b.x, a.y - b.y);
        const float2 B = make_float2(a.x - b.x, a.y + b.y);
        const float2 w = S.tw[k];
        const float wbr = fmaf(w.x, B.x, -w.y * B.y);
        const float wbi = fmaf(w.x, B.y, w.y * B.x);
        const float re = A.x + wbi, im = A.y - wbr;
        pw[k] = fmaf(re, re, im * im);
        if (k == 0) {
          const float ny = 2.0f * (a.x - a.y);  // X[256] = Re Z0 - Im Z0 (Z halved)
          pw[kLfmFft / 2] = ny * ny;
        }
      }
      __syncwarp(gmask);
      float *orow = out + ((int64_t)t.frame_off[c] + f0 + fi) * prm.n_mels;
      for (int b = j; b < prm.n_mels; b += 16) {
        const float *p = pw + S.band_lo[b];
        float acc = 0.f;
#pragma unroll 4
        for (int q = 0; q < prm.bins; ++q) acc = fmaf(S.wts[b][q], p[q], acc);
        orow[b] = logf(fmaxf(acc, prm.log_floor));
      }
      __syncwarp(gmask);
    }
  }
}

__global__ void __launch_bounds__(256) k_lfm_norm(float *__restrict__ out, const LfmTablesDev t, const LfmParams prm) {
  __shared__ double red[2][8][32];
  const int c = blockIdx.x, bg = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = bg * 32 + lane;
  const bool live = b < prm.n_mels;
  const int nf = t.frame_off[c + 1] - t.frame_off[c], eff = t.eff[c];
  float *base = out + (int64_t)t.frame_off[c] * prm.n_mels + b;
  // one pass for the first two moments, in float64. Only the first moment is
  // exact for a band whose values are all equal; s2 / n - mean^2 can round to
  // a tiny value of either sign, which the clamp at zero and var_eps (> 0,
  // checked on the host) absorb
  double s1 = 0.0, s2 = 0.0;
  if (live) {
#pragma unroll 8
    for (int f = warp; f < eff; f += 8) {
      const double v = (double)base[(int64_t)f * prm.n_mels];
      s1 += v;
      s2 = fma(v, v, s2);
    }
  }
  red[0][warp][lane] = s1;
  red[1][warp][lane] = s2;
  __syncthreads();
  s1 = 0.0;
  s2 = 0.0;
  for (int w = 0; w < 8; ++w) {  // fixed order: deterministic
    s1 += red[0][w][lane];
    s2 += red[1][w][lane];
  }
  const double n = eff > 0 ? (double)eff : 1.0;
  const double mean = s1 / n;
  const double var = fmax(0.0, s2 / n - mean * mean);
  const double inv = 1.0 / sqrt(var + (double)prm.var_eps);
  if (live) {
#pragma unroll 8
    for (int f = warp; f < nf; f += 8) {
      float *p = base + (int64_t)f * prm.n_mels;
      *p = f < eff ? (float)(((double)*p - mean) * inv) : 0.f;
    }
  }
}

cudaError_t launch_lfm(const float *wave, float *out, const LfmTablesDev &t, const LfmParams &prm, cudaStream_t s) {
  if (t.n_tiles <= 0) return cudaSuccess;
  const size_t smem = lfm_smem_bytes(prm.hop);
  cudaError_t e = cudaFuncSetAttribute(k_lfm_spec, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int grid = t.n_tiles < 2 * sms ? t.n_tiles : 2 * sms;
  if ((e = launch_k(k_lfm_spec, dim3((unsigned)grid), dim3(kLfmThreads), smem, s, wave, out, t, prm)) != cudaSuccess)
    return e;
  return launch_k(k_lfm_norm, dim3((unsigned)t.n_clips, (unsigned)((prm.n_mels + 31) / 32)), dim3(256), 0, s, out, t,
                  prm);
}

}  // namespace ae
