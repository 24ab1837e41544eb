// Host-side encoder of OCP e4m3 codes, used at model creation to quantise
// the e4m3 projections' weight rows. Plain C++ (no CUDA), so that it can be
// tested on its own.
#pragma once

#include <cmath>
#include <cstddef>
#include <cstdint>

namespace ae {

// OCP e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; largest
// finite 448, subnormals k 2^-9) code of t, rounded to nearest even, with
// magnitudes beyond 448 saturated to 448.
inline uint8_t e4m3_code(double t) {
  const uint8_t sign = std::signbit(t) ? 0x80 : 0x00;
  const double a = std::fabs(t);
  if (!(a < 448.0)) return sign | 0x7E;  // also NaN: never produced from finite weights
  if (a < 0.015625) {                    // below 2^-6: subnormal grid of 2^-9 (k = 8 is the smallest normal)
    return sign | (uint8_t)std::nearbyint(std::ldexp(a, 9));
  }
  int ex;
  std::frexp(a, &ex);  // a = f 2^ex, f in [0.5, 1)
  const int e = ex - 1;  // a in [2^e, 2^(e+1))
  int k = (int)std::nearbyint(std::ldexp(a, 3 - e));  // 8 .. 16 steps of 2^(e-3)
  int be = e + 7;
  if (k == 16) {
    k = 8;
    ++be;
  }
  if (be > 15 || (be == 15 && k > 14)) return sign | 0x7E;
  return sign | (uint8_t)((be << 3) | (k - 8));
}

// One weight row of an e4m3 projection: *scale = max_k |w[k]| / 448 (1 for an
// all-zero row) and codes[k] = e4m3_code(w[k] / *scale), in float64.
inline void e4m3_quantise_row(const float *w, size_t cols, uint8_t *codes, double *scale) {
  double amax = 0.0;
  for (size_t k = 0; k < cols; ++k) amax = std::fmax(amax, std::fabs((double)w[k]));
  const double sn = amax > 0.0 ? amax / 448.0 : 1.0;
  for (size_t k = 0; k < cols; ++k) codes[k] = e4m3_code((double)w[k] / sn);
  *scale = sn;
}

}  // namespace ae
