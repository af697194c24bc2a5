// counter_rng.cuh -- in-kernel Gaussian gradient streams for the simulated
// workers, so that their gradients cost no HBM bytes.
//
// Generator: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random
// Numbers: As Easy as 1, 2, 3", SC 2011). Ten rounds over a 128-bit counter;
// a round takes the 64-bit products of counter words 0 and 2 with two odd
// multipliers and forms the new counter from the high halves xor-ed with the
// other two words and the key, and the low halves; the key advances by two
// Weyl increments between rounds.
//
// Stream: entry i (row-major) of worker k's gradient of matrix j at step t is
// Gaussian number i % 4 of Philox(counter = (i/4 low, i/4 high, t, 0),
// key = (seed_base + k, matrix_base + j)), times sigma. Each counter's four
// words give two Box-Muller pairs. The transform runs in float32 with
// explicitly rounded operations (no contraction into fused multiply-adds), so
// its bits are reproducible by any IEEE float32 evaluation of the same steps:
//   u1 = ((x0 >> 8) + 1) * 2^-24 in (0, 1],   radius = sqrt(-2 ln u1)
//   quadrant q = x1 >> 30, position r = ((x1 >> 8) & 0x3fffff) * 2^-22
//   angle (q + r) * pi/2; cos and sin from Taylor polynomials of r * pi/2
//   ln u = e ln2 + 2 atanh((f - 1)/(f + 1)) with u = 2^e f, f in [sqrt(1/2), sqrt(2))
#pragma once

#include <stdint.h>

namespace smuon {
namespace crng {

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

// float32 constants: the float nearest to each real number (via its double)
constexpr float kLn2 = (float)0.69314718055994530942;
constexpr float kHalfPi = (float)(3.14159265358979323846 / 2.0);

// ln(u), u in (0, 1]
__device__ __forceinline__ float ln_unit(float u) {
  const uint32_t b = __float_as_uint(u);
  int e = (int)(b >> 23) - 127;
  uint32_t fb = (b & 0x7FFFFFu) | 0x3F800000u;
  if (fb > 0x3FB504F3u) {  // f above sqrt(2): halve it (exact), one more in the exponent
    fb -= 0x00800000u;
    e += 1;
  }
  const float f = __uint_as_float(fb);
  const float t = __fdiv_rn(__fsub_rn(f, 1.f), __fadd_rn(f, 1.f));
  const float s = __fmul_rn(t, t);
  // atanh(t)/t = 1 + s/3 + s^2/5 + ... + s^6/13
  float p = (float)(1.0 / 13.0);
  p = __fadd_rn(__fmul_rn(p, s), (float)(1.0 / 11.0));
  p = __fadd_rn(__fmul_rn(p, s), (float)(1.0 / 9.0));
  p = __fadd_rn(__fmul_rn(p, s), (float)(1.0 / 7.0));
  p = __fadd_rn(__fmul_rn(p, s), (float)(1.0 / 5.0));
  p = __fadd_rn(__fmul_rn(p, s), (float)(1.0 / 3.0));
  p = __fadd_rn(__fmul_rn(p, s), 1.f);
  const float lnf = __fmul_rn(__fmul_rn(2.f, t), p);
  return __fadd_rn(__fmul_rn((float)e, kLn2), lnf);
}

// cos and sin of (q + r) * pi/2, r in [0, 1)
__device__ __forceinline__ void sincos_quadrant(uint32_t q, float r, float* cs, float* sn) {
  const float x = __fmul_rn(r, kHalfPi);
  const float s = __fmul_rn(x, x);
  // sin(x)/x = sum_i (-1)^i s^i / (2i+1)!,  i = 0..6
  float ps = (float)(1.0 / 6227020800.0);
  ps = __fadd_rn(__fmul_rn(ps, s), (float)(-1.0 / 39916800.0));
  ps = __fadd_rn(__fmul_rn(ps, s), (float)(1.0 / 362880.0));
  ps = __fadd_rn(__fmul_rn(ps, s), (float)(-1.0 / 5040.0));
  ps = __fadd_rn(__fmul_rn(ps, s), (float)(1.0 / 120.0));
  ps = __fadd_rn(__fmul_rn(ps, s), (float)(-1.0 / 6.0));
  ps = __fadd_rn(__fmul_rn(ps, s), 1.f);
  const float sx = __fmul_rn(x, ps);
  // cos(x) = sum_i (-1)^i s^i / (2i)!,  i = 0..7
  float pc = (float)(-1.0 / 87178291200.0);
  pc = __fadd_rn(__fmul_rn(pc, s), (float)(1.0 / 479001600.0));
  pc = __fadd_rn(__fmul_rn(pc, s), (float)(-1.0 / 3628800.0));
  pc = __fadd_rn(__fmul_rn(pc, s), (float)(1.0 / 40320.0));
  pc = __fadd_rn(__fmul_rn(pc, s), (float)(-1.0 / 720.0));
  pc = __fadd_rn(__fmul_rn(pc, s), (float)(1.0 / 24.0));
  pc = __fadd_rn(__fmul_rn(pc, s), -0.5f);
  pc = __fadd_rn(__fmul_rn(pc, s), 1.f);
  const float cx = pc;
  switch (q) {
    case 0: *cs = cx; *sn = sx; break;
    case 1: *cs = -sx; *sn = cx; break;
    case 2: *cs = -cx; *sn = -sx; break;
    default: *cs = sx; *sn = -cx; break;
  }
}

__device__ __forceinline__ void box_muller(uint32_t x0, uint32_t x1, float* z0, float* z1) {
  const float u1 = __fmul_rn(__uint2float_rn((x0 >> 8) + 1u), 5.9604644775390625e-8f);  // 2^-24
  const float r = __fmul_rn(__uint2float_rn((x1 >> 8) & 0x3FFFFFu), 2.384185791015625e-7f);  // 2^-22
  const float rad = __fsqrt_rn(__fmul_rn(-2.f, ln_unit(u1)));
  float c, s;
  sincos_quadrant(x1 >> 30, r, &c, &s);
  *z0 = __fmul_rn(rad, c);
  *z1 = __fmul_rn(rad, s);
}

// sigma * the 8 Gaussians of entries e0 .. e0 + 7 (e0 a multiple of 4) of one stream
__device__ __forceinline__ void gaussian8(uint32_t key0, uint32_t key1, uint32_t step, int64_t e0, float sigma,
                                          float* out) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint64_t g = (uint64_t)(e0 >> 2) + h;
    const uint4 x = philox4x32_10(make_uint4((uint32_t)g, (uint32_t)(g >> 32), step, 0u), key0, key1);
    float z[4];
    box_muller(x.x, x.y, &z[0], &z[1]);
    box_muller(x.z, x.w, &z[2], &z[3]);
#pragma unroll
    for (int j = 0; j < 4; ++j) out[4 * h + j] = __fmul_rn(z[j], sigma);
  }
}

}  // namespace crng
}  // namespace smuon
