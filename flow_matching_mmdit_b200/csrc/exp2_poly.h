// 2^x on the FMA pipe, for the share of the softmax exponentials that the attention
// kernel takes off the exponential unit (16 results per clock per SM on B200, against
// 128 fp32 FMAs).  Usable from host code too, so the CPU tests check the very
// constants and steps the kernel uses.
//
// Method (Cody-Waite style range reduction, then a polynomial):
//   2^x = 2^j * 2^f,  j = round-to-nearest(x),  f = x - j in [-1/2, 1/2].
//   * j: adding 1.5 * 2^23 rounds x to an integer and leaves j in the low mantissa
//     bits of the sum t, so neither a conversion nor a rounding instruction is needed
//     (on B200 those issue on the exponential unit as well); t - 1.5 * 2^23 is j as a
//     float, exactly.
//   * 2^f: the cubic p(f) = c0 + c1 f + c2 f^2 + c3 f^3 whose coefficients minimise the
//     largest relative error |p(f) / 2^f - 1| over [-1/2, 1/2] (computed by a Remez
//     exchange for this file and rounded to fp32): at most 7.5e-5 once evaluated in
//     fp32 by Horner's rule with fused multiply-adds.
//   * 2^j: j << 23 added to p's bits moves p's exponent by j; (bits(t) << 23) is that
//     integer already, since the constant's own bits shift out past bit 31.
//   x is clamped to >= -125 first, which keeps the result a normal float (2^-125
//   stands in for 0, e.g. for masked scores of -inf).  Valid for x <= 127.
#pragma once
#include <math.h>
#include <stdint.h>
#include <string.h>

#if defined(__CUDACC__)
#define LENS_HD __host__ __device__ __forceinline__
#else
#define LENS_HD inline
#endif

namespace lens {

constexpr float kExp2Round = 12582912.0f;     // 1.5 * 2^23
constexpr float kExp2Floor = -125.0f;
constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716685295105f;

LENS_HD uint32_t exp2_poly_bits(float v) {
  uint32_t u;
  memcpy(&u, &v, 4);
  return u;
}
LENS_HD float exp2_poly_float(uint32_t u) {
  float v;
  memcpy(&v, &u, 4);
  return v;
}

// Scalar form (the kernel runs the same steps on fp32 pairs).
LENS_HD float exp2_poly(float x) {
  x = x > kExp2Floor ? x : kExp2Floor;
  const float t = x + kExp2Round;
  const float j = t - kExp2Round;
  const float f = x - j;
  float p = fmaf(f, kExp2C3, kExp2C2);
  p = fmaf(p, f, kExp2C1);
  p = fmaf(p, f, kExp2C0);
  return exp2_poly_float(exp2_poly_bits(p) + (exp2_poly_bits(t) << 23));
}

}  // namespace lens
