// Complex helpers and the in-register 16-point DFT of the log-mel front-ends
// (a 256-point complex FFT is done in the four-step form 16 x 16 on top).
#pragma once

#include <cuda_runtime.h>

namespace ae {

// complex add and subtract on the packed two-lane float32 pipe (one
// instruction each; the subtraction as a fused multiply-add by -1, exact)
__device__ __forceinline__ float2 cadd(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 csub(float2 a, float2 b) { return __ffma2_rn(b, make_float2(-1.f, -1.f), a); }
__device__ __forceinline__ float2 cmul(float2 a, float2 w) {
  return make_float2(fmaf(a.x, w.x, -a.y * w.y), fmaf(a.x, w.y, a.y * w.x));
}

// In-place 4-point DFT: y_k = sum_n a_n (-i)^(n k).
__device__ __forceinline__ void dft4(float2 &a0, float2 &a1, float2 &a2, float2 &a3) {
  const float2 s02 = cadd(a0, a2), d02 = csub(a0, a2), s13 = cadd(a1, a3), d13 = csub(a1, a3);
  a0 = cadd(s02, s13);
  a2 = csub(s02, s13);
  const float2 q = make_float2(d13.y, -d13.x);    // -i d13
  a1 = cadd(d02, q);                               // d02 - i d13
  a3 = csub(d02, q);                               // d02 + i d13
}

// 16-point DFT in registers, natural order in and out: x[k] <- sum_n x[n] W16^(n k).
// Four-step 4 x 4: n = 4 n1 + n2, k = k1 + 4 k2.
__device__ __forceinline__ void dft16(float2 (&x)[16]) {
  constexpr float C1 = 0.92387953251128674f, S1 = 0.38268343236508977f, R = 0.70710678118654752f;
#pragma unroll
  for (int n2 = 0; n2 < 4; ++n2) dft4(x[n2], x[4 + n2], x[8 + n2], x[12 + n2]);
  // x[4 k1 + n2] *= W16^(n2 k1)
  x[5] = cmul(x[5], make_float2(C1, -S1));    // W^1
  x[6] = cmul(x[6], make_float2(R, -R));      // W^2
  x[7] = cmul(x[7], make_float2(S1, -C1));    // W^3
  x[9] = cmul(x[9], make_float2(R, -R));      // W^2
  x[10] = make_float2(x[10].y, -x[10].x);     // W^4 = -i
  x[11] = cmul(x[11], make_float2(-R, -R));   // W^6
  x[13] = cmul(x[13], make_float2(S1, -C1));  // W^3
  x[14] = cmul(x[14], make_float2(-R, -R));   // W^6
  x[15] = cmul(x[15], make_float2(-C1, S1));  // W^9
#pragma unroll
  for (int k1 = 0; k1 < 4; ++k1) dft4(x[4 * k1], x[4 * k1 + 1], x[4 * k1 + 2], x[4 * k1 + 3]);
  // X[k1 + 4 k2] sits at x[4 k1 + k2]: transpose the 4 x 4
  float2 t[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) t[k] = x[4 * (k & 3) + (k >> 2)];
#pragma unroll
  for (int k = 0; k < 16; ++k) x[k] = t[k];
}

}  // namespace ae
