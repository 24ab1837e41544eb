// Host-side builder of the second log-mel front-end's Slaney filterbank, as
// the sparse table its kernel reads. Plain C++ (no CUDA), so that it can be
// tested on its own.
#pragma once

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <vector>

#include "../../include/ae.h"

namespace ae {

// Slaney mel scale: 3 f / 200 below 1 kHz, 15 + 27 ln(f / 1000) / ln 6.4 above.
inline double slaney_mel(double f) { return f < 1000.0 ? 3.0 * f / 200.0 : 15.0 + 27.0 * std::log(f / 1000.0) / std::log(6.4); }
inline double slaney_hz(double m) { return m < 15.0 ? 200.0 * m / 3.0 : 1000.0 * std::exp((m - 15.0) * std::log(6.4) / 27.0); }

// The bank as (first nonzero bin, max_bins weights from there) per band,
// float64 from the definition; false if a band has more nonzero bins.
inline bool lfm_bank(const ae_lfm_config &c, std::vector<int32_t> &lo, std::vector<float> &w, int *widest,
                     int max_bins) {
  const int nb = c.n_fft / 2 + 1;
  lo.assign(c.n_mels, 0);
  w.assign((size_t)c.n_mels * max_bins, 0.f);
  *widest = 0;
  const double m_hi = slaney_mel(c.sample_rate / 2.0);
  std::vector<double> pts(c.n_mels + 2);
  for (int i = 0; i < c.n_mels + 2; ++i) pts[i] = slaney_hz(m_hi * i / (c.n_mels + 1));
  for (int b = 0; b < c.n_mels; ++b) {
    const double enorm = 2.0 / (pts[b + 2] - pts[b]);
    int first = -1, last = -1;
    std::vector<double> v(nb, 0.0);
    for (int k = 0; k < nb; ++k) {
      const double fk = (double)k * c.sample_rate / c.n_fft;
      const double down = (fk - pts[b]) / (pts[b + 1] - pts[b]);
      const double up = (pts[b + 2] - fk) / (pts[b + 2] - pts[b + 1]);
      v[k] = std::max(0.0, std::min(down, up)) * enorm;
      if (v[k] > 0.0) {
        if (first < 0) first = k;
        last = k;
      }
    }
    if (first < 0) continue;  // an empty band (narrower than a bin): all zero weights
    if (last - first + 1 > max_bins) return false;
    *widest = std::max(*widest, last - first + 1);
    lo[b] = first;
    for (int q = 0; first + q <= last; ++q) w[(size_t)b * max_bins + q] = (float)v[first + q];
  }
  return true;
}

// The bank as the spectrum kernel reads it: per band its first bin, its number
// of bins up to the last nonzero weight and the offset of those weights in one
// packed array; and the bands of each of the `warps` warps of the band phase,
// contiguous and balanced by work (one multiply-add per weight and
// kLfmBandCost more per band: the log, the floor and the store).
constexpr int kLfmBandCost = 8;
struct LfmPackedBank {
  std::vector<int32_t> lo, cnt, off;
  std::vector<float> w;
  std::vector<int32_t> wband;  // warps + 1 boundaries, 0 .. n_mels
};

inline LfmPackedBank lfm_bank_pack(const std::vector<int32_t> &lo, const std::vector<float> &w, int n_mels,
                                   int max_bins, int warps) {
  LfmPackedBank P;
  P.lo.assign(lo.begin(), lo.begin() + n_mels);
  P.cnt.assign(n_mels, 0);
  P.off.assign(n_mels, 0);
  int64_t total = 0;
  for (int b = 0; b < n_mels; ++b) {
    int n = 0;
    for (int q = 0; q < max_bins; ++q)
      if (w[(size_t)b * max_bins + q] != 0.f) n = q + 1;
    P.cnt[b] = n;
    P.off[b] = (int32_t)P.w.size();
    for (int q = 0; q < n; ++q) P.w.push_back(w[(size_t)b * max_bins + q]);
    total += n + kLfmBandCost;
  }
  P.wband.assign(1, 0);
  int64_t acc = 0;
  for (int b = 0; b < n_mels; ++b) {
    acc += P.cnt[b] + kLfmBandCost;
    if ((int)P.wband.size() < warps && acc * warps >= total * (int64_t)P.wband.size()) P.wband.push_back(b + 1);
  }
  while ((int)P.wband.size() <= warps) P.wband.push_back(n_mels);
  P.wband[warps] = n_mels;
  return P;
}

}  // namespace ae
