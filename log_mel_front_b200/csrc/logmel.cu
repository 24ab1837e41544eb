// Log-mel front-end (egemma2_audio.rs, MelFrontend::log_mel), fused in one
// kernel: framing with the 160-sample semicausal pad, periodic Hann window,
// 512-point real FFT, magnitude, sparse 128-band HTK mel projection and
// ln(mel + 0.001).
//
// Work item: 64 consecutive frames of one clip. The CTA stages the
// contiguous waveform span those frames cover (64*160 + 160 samples) in
// shared memory with coalesced loads; 16 groups of 16 threads then take one
// frame each. Per frame the 320 windowed samples are packed as 160 complex
// values z[n] = x[2n] + i x[2n+1] (the other 96 are zero) and transformed
// by a 256-point complex FFT in the four-step form 16 x 16: each thread does
// a 16-point DFT in registers, multiplies by the W256 twiddles, the group
// transposes through padded shared memory, and each thread does the second
// 16-point DFT. The real spectrum follows from the usual split
// X[k] = E[k] - i W512^k O[k] with E, O from Z[k] and conj(Z[256-k]). The
// mel projection walks only each band's nonzero bins (at most 11, 506 in
// all) instead of the dense 257 x 128 product.
//
// Tables (twiddles, window, mel bank) are built per CTA in float64 from
// their definitions; CTAs are persistent, so this costs once per CTA.
#include "ae_internal.h"
#include "common.cuh"
#include "fft16.cuh"

namespace ae {

namespace {
constexpr int kGroups = 16;                        // frames in flight per CTA
constexpr int kThreads = kGroups * 16;             // 256
constexpr int kWaveSpan = kMelTile * kHop + kHop;  // samples staged per work item
constexpr int kMaxBins = 12;                       // bins per band (11 suffice), zero-padded
constexpr int kPitch = 17;                         // padded row of the 16 x 16 transpose

struct LogmelSmem {
  float2 tw[kFft];                         // W512^m = (cos, -sin)(2 pi m / 512)
  float win[kFrame];                       // Hann / 2 (the split's 1/2 folded in)
  float wts[kMels][kMaxBins + 1];          // sparse mel bank, zero-padded (row pitch 13 against bank conflicts)
  int band_lo[kMels];
  float wave[kWaveSpan];
  float2 xs[kGroups][kPitch * 16];         // per-group transpose / spectrum exchange
  float mag[kGroups][kFft / 2 + 16];       // per-group magnitudes (zero tail for the padded mel loop)
  int tile_clip, tile_f0, tile_nf;
};
}  // namespace

__global__ void __launch_bounds__(kThreads, 2)
    k_logmel(const float *__restrict__ wave, float *__restrict__ mel, const ClipTablesDev t, int n_tiles) {
  extern __shared__ uint8_t smem_raw[];
  LogmelSmem &S = *reinterpret_cast<LogmelSmem *>(smem_raw);
  const int tid = threadIdx.x;

  // ---- tables, float64 from their definitions
  for (int m = tid; m < kFft; m += kThreads) {
    double s, c;
    sincospi((double)m / 256.0, &s, &c);  // angle 2 pi m / 512
    S.tw[m] = make_float2((float)c, (float)-s);
  }
  for (int j = tid; j < kFrame; j += kThreads) S.win[j] = (float)(0.25 - 0.25 * cospi((double)j / 160.0));
  if (tid < kMels) {
    // HTK: 130 mel points over [mel(0), mel(8000)] (last point exact), bins at k * 31.25 Hz;
    // band b is the triangle over [f_b, f_b+2]; only the bins inside it are visited
    const double mel_hi = 2595.0 * log10(1.0 + 8000.0 / 700.0);
    const double step = mel_hi / 129.0;
    double f[3];
    for (int i = 0; i < 3; ++i) {
      const int p = tid + i;
      const double mm = (p == 129) ? mel_hi : p * step;
      f[i] = 700.0 * (pow(10.0, mm / 2595.0) - 1.0);
    }
    for (int q = 0; q < kMaxBins; ++q) S.wts[tid][q] = 0.f;
    int lo = -1, n = 0;
    const int k0 = max(0, (int)floor(f[0] / 31.25)), k1 = min(kFft / 2, (int)ceil(f[2] / 31.25));
    for (int k = k0; k <= k1; ++k) {
      const double fk = k * 31.25;
      const double down = (fk - f[0]) / (f[1] - f[0]);
      const double up = (f[2] - fk) / (f[2] - f[1]);
      const double w = fmax(0.0, fmin(down, up));
      if (w > 0.0 && n < kMaxBins) {
        if (lo < 0) lo = k;
        S.wts[tid][n++] = (float)w;
      }
    }
    S.band_lo[tid] = lo < 0 ? 0 : lo;
  }
  for (int x = tid; x < kGroups * 16; x += kThreads) S.mag[x / 16][kFft / 2 + x % 16] = 0.f;

  __syncthreads();
  const int g = tid >> 4, j = tid & 15;
  const unsigned gmask = 0xFFFFu << (16 * (g & 1));
  float2 tw1[16];  // W256^(j k1): depends only on the thread
#pragma unroll
  for (int k1 = 0; k1 < 16; ++k1) tw1[k1] = S.tw[(2 * j * k1) & (kFft - 1)];
  float2 *xs = S.xs[g];
  float *mag = S.mag[g];

  for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    __syncthreads();  // previous work item done with the staged wave
    if (tid == 0) {
      int lo = 0, hi = t.n_clips;  // last clip c with mel_tile_off[c] <= tile
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (t.mel_tile_off[mid] <= tile) lo = mid; else hi = mid;
      }
      const int nfr = t.frame_off[lo + 1] - t.frame_off[lo];
      S.tile_clip = lo;
      S.tile_f0 = (tile - t.mel_tile_off[lo]) * kMelTile;
      S.tile_nf = min(kMelTile, nfr - S.tile_f0);
    }
    __syncthreads();
    const int c = S.tile_clip, f0 = S.tile_f0, nf = S.tile_nf;
    const int64_t s_begin = t.sample_off[c];
    const int64_t n_samp = min(t.sample_off[c + 1] - s_begin, (int64_t)kMaxSamples);
    // local sample i is clip sample (f0 - 1) * 160 + i
    const int64_t first = (int64_t)(f0 - 1) * kHop;
    const int span = nf * kHop + kHop;
    for (int i = tid; i < span; i += kThreads) {
      const int64_t sidx = first + i;
      S.wave[i] = (sidx >= 0 && sidx < n_samp) ? __ldg(wave + s_begin + sidx) : 0.0f;
    }
    __syncthreads();

    for (int fi = g; fi < nf; fi += kGroups) {
      const float *wv = S.wave + fi * kHop;
      // ---- stage 1: z[16 n1 + j], n1 < 10 nonzero; DFT over n1
      float2 x[16];
#pragma unroll
      for (int n1 = 0; n1 < 16; ++n1) {
        if (n1 < 10) {
          const int m = 32 * n1 + 2 * j;
          const float2 a = *reinterpret_cast<const float2 *>(wv + m);
          const float2 w = *reinterpret_cast<const float2 *>(S.win + m);
          x[n1] = make_float2(a.x * w.x, a.y * w.y);
        } else {
          x[n1] = make_float2(0.f, 0.f);
        }
      }
      dft16(x);
#pragma unroll
      for (int k1 = 1; k1 < 16; ++k1) x[k1] = cmul(x[k1], tw1[k1]);  // W256^(j k1)
#pragma unroll
      for (int k1 = 0; k1 < 16; ++k1) xs[k1 * kPitch + j] = x[k1];
      __syncwarp(gmask);
      // ---- stage 2: thread j = k1 gathers over n2 and finishes
#pragma unroll
      for (int n2 = 0; n2 < 16; ++n2) x[n2] = xs[j * kPitch + n2];
      dft16(x);  // x[k2] = Z[j + 16 k2]
      __syncwarp(gmask);
#pragma unroll
      for (int k2 = 0; k2 < 16; ++k2) xs[k2 * kPitch + j] = x[k2];
      __syncwarp(gmask);
      // ---- real split and magnitude: X[k] = (Z_k + conj Z_k') - i W512^k (Z_k - conj Z_k'), k' = 256 - k
#pragma unroll
      for (int k2 = 0; k2 < 16; ++k2) {
        const int k = j + 16 * k2;
        float2 b;
        if (j == 0) {
          const int kk = (16 - k2) & 15;  // k' = 16 (16 - k2) mod 256
          b = xs[kk * kPitch];
        } else {
          b = xs[(15 - k2) * kPitch + (16 - j)];
        }
        const float2 a = x[k2];
        const float2 A = make_float2(a.x + b.x, a.y - b.y);
        const float2 B = make_float2(a.x - b.x, a.y + b.y);
        const float2 w = S.tw[k];  // (cos, -sin)
        // -i (w B) = (Im(wB), -Re(wB))
        const float wbr = fmaf(w.x, B.x, -w.y * B.y);
        const float wbi = fmaf(w.x, B.y, w.y * B.x);
        const float re = A.x + wbi, im = A.y - wbr;
        const float m2 = fmaf(re, re, im * im);
        mag[k] = m2 * rsqrtf(fmaxf(m2, 1e-37f));  // |X| (2 ulp), 0 for 0
        if (k == 0) mag[kFft / 2] = fabsf(2.0f * (a.x - a.y));  // Nyquist: Re Z0 - Im Z0 (Z halved)
      }
      __syncwarp(gmask);
      // ---- mel bands j, j+16, ...: sparse dot, log, store
      float *orow = mel + ((int64_t)t.frame_off[c] + f0 + fi) * kMels;
#pragma unroll
      for (int i = 0; i < kMels / 16; ++i) {
        const int b = j + 16 * i;
        const float *mg = mag + S.band_lo[b];
        float acc = 0.f;
#pragma unroll
        for (int q = 0; q < kMaxBins; ++q) acc = fmaf(S.wts[b][q], mg[q], acc);
        orow[b] = logf(acc + 1e-3f);
      }
      __syncwarp(gmask);
    }
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
