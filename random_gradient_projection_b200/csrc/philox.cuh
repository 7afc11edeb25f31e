// Philox4x32-10 and Box-Muller on the device.
//
// Philox4x32-10: Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy
// as 1, 2, 3" (SC'11), section 3.2 and table 2.  Four 32-bit counter words,
// two 32-bit key words, ten rounds; a round multiplies counter words 0 and 2
// by the two round multipliers, and the key is bumped by the two Weyl
// constants between rounds.
//
// Stream layout of the method's randomness (this library's reading of
// Metodologia design choice 1 of the DP-GRAPE technical summary, which has P
// rebuilt from a seed instead of stored): key = (seed lo, seed hi), counter =
// (q, layer, step, stream), stream 0 = projection matrix, 1 = noise.  Element
// e of a stream uses block q = e / 4: words (x0, x1) give elements 4q, 4q+1
// (cosine, sine) and words (x2, x3) give 4q+2, 4q+3.
#pragma once
#include <cstdint>

namespace grape {

constexpr uint32_t kPhiloxM0 = 0xD2511F53u;
constexpr uint32_t kPhiloxM1 = 0xCD9E8D57u;
constexpr uint32_t kPhiloxW0 = 0x9E3779B9u;
constexpr uint32_t kPhiloxW1 = 0xBB67AE85u;

constexpr uint32_t kStreamProjection = 0;
constexpr uint32_t kStreamNoise = 1;

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    if (round > 0) {
      k0 += kPhiloxW0;
      k1 += kPhiloxW1;
    }
    const uint32_t lo0 = kPhiloxM0 * c.x;
    const uint32_t hi0 = __umulhi(kPhiloxM0, c.x);
    const uint32_t lo1 = kPhiloxM1 * c.z;
    const uint32_t hi1 = __umulhi(kPhiloxM1, c.z);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

// The four words of block q of (seed, layer, step, stream).
__device__ __forceinline__ uint4 philox_block(uint64_t seed, uint32_t layer, uint32_t step,
                                              uint32_t stream, uint32_t q) {
  return philox4x32_10(make_uint4(q, layer, step, stream), static_cast<uint32_t>(seed),
                       static_cast<uint32_t>(seed >> 32));
}

// Box-Muller (1958) in fp32: u1 = (xa + 1) 2^-32 in (0, 1], u2 = xb 2^-32 in [0, 1);
// returns (rho cos 2 pi u2, rho sin 2 pi u2), rho = sqrt(-2 ln u1).
__device__ __forceinline__ float2 box_muller(uint32_t xa, uint32_t xb) {
  const float u1 = fmaf(static_cast<float>(xa), 0x1p-32f, 0x1p-32f);
  const float two_u2 = static_cast<float>(xb) * 0x1p-31f;
  const float rho = sqrtf(-2.0f * logf(u1));
  float s, c;
  sincospif(two_u2, &s, &c);
  return make_float2(rho * c, rho * s);
}

// Box-Muller with the special-function unit's log and sine/cosine (__logf,
// __sincosf), for normals that are rounded to bf16 at once.  The angle is moved into
// [-pi, pi), where __sincosf is most accurate: theta = 2 pi u2 - pi, and
// (cos 2 pi u2, sin 2 pi u2) = -(cos theta, sin theta).  Against the exact transform
// of the same words the error is at most about 1e-3 absolute, reached only where
// rho is that small (the log's absolute error, about 4e-7 near u1 = 1, under the
// square root), and a few 1e-6 elsewhere: below bf16's half ulp, 2^-9 of |z|, for
// all but such tiny values.  That absolute error can make the log of a u1 just below
// 1 positive, so -2 ln u1 is clamped at 0 before the square root.
__device__ __forceinline__ float2 box_muller_fast(uint32_t xa, uint32_t xb) {
  const float u1 = fmaf(static_cast<float>(xa), 0x1p-32f, 0x1p-32f);
  const float theta = fmaf(static_cast<float>(xb), 0x1.921fb6p-30f, -0x1.921fb6p+1f);
  const float rho = sqrtf(fmaxf(-2.0f * __logf(u1), 0.0f));
  float s, c;
  __sincosf(theta, &s, &c);
  return make_float2(-rho * c, -rho * s);
}

// The four normals of block q: elements 4q .. 4q+3.
__device__ __forceinline__ float4 gaussian4(uint64_t seed, uint32_t layer, uint32_t step,
                                            uint32_t stream, uint32_t q) {
  const uint4 w = philox_block(seed, layer, step, stream, q);
  const float2 a = box_muller(w.x, w.y);
  const float2 b = box_muller(w.z, w.w);
  return make_float4(a.x, a.y, b.x, b.y);
}

// gaussian4 through box_muller_fast.
__device__ __forceinline__ float4 gaussian4_fast(uint64_t seed, uint32_t layer, uint32_t step,
                                                 uint32_t stream, uint32_t q) {
  const uint4 w = philox_block(seed, layer, step, stream, q);
  const float2 a = box_muller_fast(w.x, w.y);
  const float2 b = box_muller_fast(w.z, w.w);
  return make_float4(a.x, a.y, b.x, b.y);
}

}  // namespace grape
