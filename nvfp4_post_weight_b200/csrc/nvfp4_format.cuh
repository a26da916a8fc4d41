// NVFP4 number formats on the device: E2M1 element codes and E4M3 block scales.
//
// "Replay the Curvature" (arXiv 2609.36654v1), Abstract: every 16 E2M1 weights
// share one E4M3 block scale.  Rounding is round-to-nearest with ties to the
// even code and saturation (E2M1 at 6, E4M3 at 448); a zero magnitude is
// stored as +0.
//
// All rounding here is written out with IEEE additions (the "add and subtract
// 1.5 * 2^p" method: adding a constant whose unit in the last place is the
// target spacing h makes the hardware's round-to-nearest-even do the rounding
// to a multiple of h), so the same decision is taken in fp32 or fp64 without
// any conversion routine.
#pragma once

#include <stdint.h>

namespace nvfp4 {

// Value of a positive E4M3 (fn) code 0..126: subnormal m * 2^-9 for e == 0,
// else (1 + m/8) * 2^(e-7).  Exact in fp32 and fp64.
__device__ __forceinline__ double e4m3_value(int code) {
  const int e = code >> 3, m = code & 7;
  // 2^(e-7) * (8 + m) / 8 for normals; m * 2^-9 for subnormals
  return e == 0 ? (double)m * 0x1p-9
                : __longlong_as_double((long long)(e + 1016) << 52) * (double)(8 + m) * 0.125;
}

// E4M3 code of non-negative t (fp64): round to nearest, ties to even,
// saturating at 448 (code 126); 0 for t <= 0 or NaN.
__device__ __forceinline__ int e4m3_code_rn(double t) {
  if (!(t > 0.0)) return 0;
  if (t >= 448.0) return 126;
  const long long bits = __double_as_longlong(t);
  int e = (int)((bits >> 52) & 0x7ff) - 1023;          // t >= 2^-1074 is normal here
  // spacing of E4M3 values around t: 2^(e-3) for normals, 2^-9 below 2^-6
  const int ulp_e = e < -6 ? -9 : e - 3;
  const double M = __longlong_as_double((long long)(ulp_e + 52 + 1023) << 52) * 1.5;
  const double r = __dsub_rn(__dadd_rn(t, M), M);     // nearest multiple of 2^ulp_e
  if (r == 0.0) return 0;
  const long long rb = __double_as_longlong(r);
  const int re = (int)((rb >> 52) & 0x7ff) - 1023;
  if (re < -6) return (int)(r * 512.0);                // subnormal: m * 2^-9
  return ((re + 7) << 3) | (int)((rb >> 49) & 7);
}

// Round |x| to the E2M1 magnitude grid {0, 0.5, 1, 1.5, 2, 3, 4, 6} (fp64),
// ties to the even code, saturating at 6.  The spacing h is 0.5 below 2, 1 in
// [2, 4) and 2 from 4 up; an even multiple of h is exactly a code whose
// mantissa bit is clear, so IEEE ties-to-even gives the even code.
__device__ __forceinline__ double e2m1_round_mag(double ax) {
  const double M = ax < 2.0 ? 0x1.8p51 : (ax < 4.0 ? 0x1.8p52 : 0x1.8p53);
  const double r = __dsub_rn(__dadd_rn(ax, M), M);
  return fmin(r, 6.0);
}

// 3-bit magnitude index of a grid magnitude r (0..7).
__device__ __forceinline__ uint32_t e2m1_index(double r) {
  // r < 2: 2r;  r in {2, 3}: r + 2;  r in {4, 6}: r / 2 + 4
  return (uint32_t)(r < 2.0 ? 2.0 * r : (r < 4.0 ? r + 2.0 : 0.5 * r + 4.0));
}

// Magnitude (E2M1 value) of a code nibble, signed.
__device__ __forceinline__ float e2m1_value(uint32_t nib) {
  const uint32_t m = nib & 7;
  const float mag = (m < 4) ? 0.5f * (float)m : (m < 6 ? (float)(m - 2) : (float)(2 * m - 8));
  return (nib & 8) ? -mag : mag;
}

}  // namespace nvfp4
