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
// which would make g infinite; so the inner log is taken on whichever of u
// and 1 - u is below one half, both of which are exact-enough fp32 values:
//   r <  2^31:  t = -log(u),        u     = (r + 1) 2^-32 (1 - 2^-32 ...)
//   r >= 2^31:  t = -log1p(-z),     z = 1 - u = (2^32 - r) 2^-32 (...)
// then g = -log(t).  Dropping the factor 2^32 / (2^32 + 1) changes u by a
// relative 2.3e-10, far below fp32 rounding.  logf and log1pf are CUDA's
// accurate library functions (this file must not be built with fast-math).
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
  float t;
  if (r >= 0x80000000u) {
    const float z = __uint2float_rn(0u - r) * kTwoPowM32;  // 1 - u, in (0, 1/2]
    t = -log1pf(-z);
  } else {
    const float u = __uint2float_rn(r + 1u) * kTwoPowM32;  // u, in (0, 1/2]
    t = -logf(u);
  }
  return -logf(t);
}

}  // namespace fmms
