// mxfp4.cuh -- MXFP4 (E2M1 codes, UE8M0 scale per 32 elements) encoding on the device.
//
// Rule (the lightning indexer runs in FP4 -- dev.to "How DeepSeek-V4 Achieves
// Million-Token Contexts ...", section "Two Compression Strategies: CSA and HCA"):
//   E    = smallest integer with amax <= 6 * 2^E, clamped to [-127, 127]; amax == 0 -> -127
//   code = round-half-even of x / 2^E onto {0, .5, 1, 1.5, 2, 3, 4, 6}; bit 3 = sign of x
//   scale byte = E + 127; element 2i in the low nibble of byte i.
// Every step is exact (power-of-two scaling, comparisons or the hardware E2M1 rounding
// of an exactly scaled value), so the bytes are a pure function of the input bits.
#pragma once
#include <cstdint>

namespace csa {

// smallest E with amax <= 6 * 2^E: write amax = f * 2^k, f in [1,2); 6 * 2^E = 1.5 * 2^(E+2),
// so E = k - 2 when f <= 1.5 and k - 1 otherwise.
__device__ __forceinline__ int mx_block_exponent(float amax) {
  if (!(amax > 0.f)) return -127;
  const uint32_t bits = __float_as_uint(amax);
  const int ef = static_cast<int>((bits >> 23) & 0xFFu);
  if (ef == 0) return -127;  // subnormal amax < 2^-126 <= 6 * 2^-127
  int E = ef - 129 + ((bits & 0x7FFFFFu) > 0x400000u ? 1 : 0);
  return E < -127 ? -127 : (E > 127 ? 127 : E);
}

// 2^E as a float, E in [-127, 127] (2^-127 is the subnormal 0x00400000)
__device__ __forceinline__ float mx_pow2(int E) {
  return E >= -126 ? __uint_as_float(static_cast<uint32_t>(E + 127) << 23) : __uint_as_float(0x00400000u);
}

// E2M1 code of x / 2^E, taken as comparisons of |x| against the rounding boundaries
// scaled by T = 2^E (products by powers of two, all representable): the same decision
// as rounding |x| / 2^E half-to-even onto {0, .5, 1, 1.5, 2, 3, 4, 6}, without forming
// the quotient.  Bit 3 is the sign of x.
__device__ __forceinline__ uint32_t e2m1_code(float x, float T) {
  const float a = fabsf(x);
  uint32_t c = (a > 0.25f * T ? 1u : 0u) + (a >= 0.75f * T ? 1u : 0u) + (a > 1.25f * T ? 1u : 0u) +
               (a >= 1.75f * T ? 1u : 0u) + (a > 2.5f * T ? 1u : 0u) + (a >= 3.5f * T ? 1u : 0u) +
               (a > 5.0f * T ? 1u : 0u);
  if (a == INFINITY) c = 7u;  // the scaled boundaries overflow only when T = 2^127
  return c | (signbit(x) ? 8u : 0u);
}

// 2^-E as a float, E in [-127, 127] (2^-127 is the subnormal 0x00400000)
__device__ __forceinline__ float mx_pow2_neg(int E) { return mx_pow2(-E); }

// The same codes through the hardware conversion: with y = x * 2^-E (exact: a power-of-two
// scaling whose result is normal whenever it can round to a nonzero code, and a
// subnormal y rounds to a signed zero either way), cvt.rn.satfinite.e2m1x2 rounds y to
// the nearest E2M1 value, ties to the even code, which is the rule above; |y| <= 6 by the
// choice of E, so saturation never acts.  Returns the byte (lo in bits 0-3, hi in 4-7).
__device__ __forceinline__ uint32_t e2m1x2_rn(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 q;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q, %2, %1;\n\t"
      "cvt.u32.u8 %0, q;\n\t}\n"
      : "=r"(r)
      : "f"(lo), "f"(hi));
  return r;
}

// Eight values scaled by inv_T = 2^-E into four packed bytes (element 2i in the low nibble
// of byte i).
__device__ __forceinline__ uint32_t e2m1x8_rn(const float (&v)[8], float inv_T) {
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) w |= e2m1x2_rn(v[2 * i] * inv_T, v[2 * i + 1] * inv_T) << (8 * i);
  return w;
}

// Encode the pair (x0, x1) held by this thread, where 16 consecutive lanes (aligned
// to 16) hold one 32-element block.  All 32 lanes of the warp must call it.
__device__ __forceinline__ void mxfp4_encode_pair(float x0, float x1, uint8_t& byte, uint8_t& scale_byte) {
  float am = fmaxf(fabsf(x0), fabsf(x1));
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  const int E = mx_block_exponent(am);
  const float inv_T = mx_pow2_neg(E);
  byte = static_cast<uint8_t>(e2m1x2_rn(x0 * inv_T, x1 * inv_T));
  scale_byte = static_cast<uint8_t>(E + 127);
}

}  // namespace csa
