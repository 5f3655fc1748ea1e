// noise.cuh -- device-side counter-based Gumbel noise of the FMMS step.
//
// Philox4x32-10 follows Salmon, Moraes, Dror and Shaw, "Parallel Random
// Numbers: As Easy as 1, 2, 3" (SC'11): a 4 x 32-bit counter, a 2 x 32-bit
// key, ten rounds of two 32x32->64 multiplies with the published multipliers,
// and Weyl increments of the key between rounds.  FlashSampling draws its
// noise from Philox keyed on a master seed and coordinates (readus.org page,
// "seed management"); here the coordinates are (token >> 2, row, step, tag)
// and the key is the 64-bit seed, so the noise does not depend on the launch
// grid.
//
// The Gumbel transform maps a word r to g = -log(-log u) with
// u = (r + 1) / (2^32 + 1) (readus.org page, "floating point precision").
// In fp32, (float)(r + 1) / (2^32 + 1) rounds to 1.0 for the top 256 words,
// which would make g infinite; so the transform works from
//   a = q 2^-32,  q = r + 1 (r < 2^31, then a = u) or 2^32 - r (then a = 1 - u),
// a value in (0, 1/2] that fp32 holds to 2^-24 relative (the neglected factor
// 2^32 / (2^32 + 1) is 1 - 2.3e-10).  The inner value t = -ln u is then
//   lower half:  t = -ln a,       with |ln a| >= ln 2, so the hardware log2
//                                 (__log2f, at most 2 ulp off away from 1)
//                                 keeps t to about 2^-22 relative;
//   upper half:  t = -ln(1 - a) = 2 atanh(w) = 2 (w + w^3/3 + w^5/5 + ...),
//                w = a / (2 - a) in (0, 1/3]: seven terms leave a relative
//                remainder below (1/9)^7 / 15 < 2e-8, with no cancellation
//                however small a is;
// and g = -ln t through __log2f again.  Both halves are evaluated and one is
// selected, so lanes never diverge.  The error of g against the exact value
// stays within 2 ulp(g) plus about 2^-21 absolute (the GPU test checks it
// against the fp64 oracle over both 2^20-word tails and a stratified sample).
#pragma once

#include <stdint.h>

namespace fmms {

struct Philox4 {
  uint32_t w0, w1, w2, w3;
};

__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2,
                                                 uint32_t c3, uint32_t k0, uint32_t k1) {
  const uint32_t kMulA = 0xD2511F53u, kMulB = 0xCD9E8D57u;
  const uint32_t kWeylA = 0x9E3779B9u, kWeylB = 0xBB67AE85u;
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    const uint32_t hiA = __umulhi(kMulA, c0), loA = kMulA * c0;
    const uint32_t hiB = __umulhi(kMulB, c2), loB = kMulB * c2;
    const uint32_t n0 = hiB ^ c1 ^ k0;
    const uint32_t n2 = hiA ^ c3 ^ k1;
    c0 = n0;
    c1 = loB;
    c2 = n2;
    c3 = loA;
    k0 += kWeylA;
    k1 += kWeylB;
  }
  return Philox4{c0, c1, c2, c3};
}

__device__ __forceinline__ float gumbel_from_u32(uint32_t r) {
  const float kTwoPowM32 = 2.3283064365386963e-10f;  // 2^-32
  const float kMinusLn2 = -0.69314718055994531f;
  const bool upper = r >= 0x80000000u;
  const uint32_t q = upper ? (0u - r) : (r + 1u);     // in [1, 2^31]
  const float a = __uint2float_rn(q) * kTwoPowM32;    // in (0, 1/2]
  const float t_lower = __log2f(a) * kMinusLn2;       // -ln a
  const float w = __fdividef(a, 2.0f - a);            // atanh argument, (0, 1/3]
  const float w2 = w * w;
  float p = 2.0f / 13.0f;
  p = fmaf(p, w2, 2.0f / 11.0f);
  p = fmaf(p, w2, 2.0f / 9.0f);
  p = fmaf(p, w2, 2.0f / 7.0f);
  p = fmaf(p, w2, 2.0f / 5.0f);
  p = fmaf(p, w2, 2.0f / 3.0f);
  p = fmaf(p, w2, 2.0f);
  const float t_upper = w * p;                        // -ln(1 - a)
  const float t = upper ? t_upper : t_lower;
  return __log2f(t) * kMinusLn2;
}

// A cheap upper bound of gumbel_from_u32(r), with no logarithm, for the
// epilogue's filter.  Lower half (u < 1/2): t = -ln u > ln 2, so
// g < -ln(ln 2) = 0.36651.  Upper half: with z = 1 - u = q / (2^32 + 1),
// q = 2^32 - r, t = -ln(1 - z) >= z gives g <= -ln z <= 32 ln 2 - ln q, and
// log2 q >= e + m for q = 2^e (1 + m) (log2(1 + m) >= m on [0, 1]); the
// float bits of q hold e + m as bits / 2^23 - 127, so
//   g <= ln 2 * (159 - bits(float(q)) / 2^23).
// The constant 1e-4 covers the fp32 rounding of this expression (< 2e-5) and
// the error of gumbel_from_u32 itself (< 3 ulp + 1e-6), so the bound holds
// for the computed value, not only the exact one.
__device__ __forceinline__ float gumbel_upper_bound(uint32_t r) {
  const float kSlope = -0.69314718055994531f * 1.1920928955078125e-07f;  // -ln2 / 2^23
  const float kOffset = 0.69314718055994531f * 159.0f + 1e-4f;
  const float fq = __uint2float_rn(0u - r);
  const float upper = fmaf(__uint2float_rn(__float_as_uint(fq)), kSlope, kOffset);
  return r >= 0x80000000u ? upper : 0.36661f;
}

}  // namespace fmms
