// FP4 (E2M1) main-KV and E4M3 scale codecs on the device.
//
// Rounding is decided by exact fp32 comparisons against midpoints, never by a
// division: every E4M3 value has at most 4 significant bits and every E2M1
// midpoint at most 3, so the products compared below are exact in fp32.
#pragma once

#include "common.cuh"

namespace csa2 {

// Value of a non-negative E4M3 code c in [0, 126] (bias 7, subnormal below
// exponent field 1: m * 2^-9).
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t E = c >> 3, M = c & 7u;
  return E ? __uint_as_float(((E + 120u) << 23) | (M << 20)) : static_cast<float>(M) * 0.001953125f;
}

// E4M3 code nearest to amax / 6 (ties to the even code, saturating at 448).
// Found as the largest code c with 6 * value(c) <= amax, then moved up when
// amax lies above the midpoint 3 * (value(c) + value(c + 1)) (or on it with
// c odd).
__device__ __forceinline__ uint32_t e4m3_code_of_sixth(float amax) {
  int lo = 0, hi = 126;
#pragma unroll
  for (int it = 0; it < 7; ++it) {
    const int mid = (lo + hi + 1) >> 1;
    if (lo < hi) {
      if (6.0f * e4m3_value(static_cast<uint32_t>(mid)) <= amax) lo = mid;
      else hi = mid - 1;
    }
  }
  uint32_t c = static_cast<uint32_t>(lo);
  if (c < 126u) {
    const float mid6 = 3.0f * (e4m3_value(c) + e4m3_value(c + 1u));
    if (amax > mid6 || (amax == mid6 && (c & 1u))) c += 1u;
  }
  return c;
}

// E2M1 code (0..15) of x under scale s > 0: nearest grid value of |x| / s,
// ties to the even code, saturating at 6, sign bit 8, -0 stored as +0.  The
// thresholds are the midpoints g between consecutive grid values times s.
__device__ __forceinline__ uint32_t e2m1_code(float x, float s) {
  const float a = fabsf(x);
  uint32_t c = 0;
  c += (a > 0.25f * s);
  c += (a > 0.75f * s) || (a == 0.75f * s);   // midpoint between codes 1 and 2: tie -> 2
  c += (a > 1.25f * s);
  c += (a > 1.75f * s) || (a == 1.75f * s);   // codes 3 / 4: tie -> 4
  c += (a > 2.5f * s);
  c += (a > 3.5f * s) || (a == 3.5f * s);     // codes 5 / 6: tie -> 6
  c += (a > 5.0f * s);
  if (x < 0.0f && c != 0u) c |= 8u;
  return c;
}

// E2M1 magnitude (codes 0..7) as fp16 bit patterns: 0, 0.5, 1, 1.5, 2, 3, 4, 6.
__device__ __forceinline__ uint16_t e2m1_half_bits(uint32_t c) {
  // fp16: sign(1) exp(5, bias 15) mant(10)
  constexpr uint16_t lut[8] = {0x0000, 0x3800, 0x3C00, 0x3E00, 0x4000, 0x4200, 0x4400, 0x4600};
  return lut[c & 7u] | static_cast<uint16_t>((c & 8u) << 12);
}

// E4M3 scale code as an fp16 bit pattern (exact: E4M3 range is inside fp16's).
__device__ __forceinline__ uint16_t e4m3_half_bits(uint32_t c) {
  const uint32_t E = (c >> 3) & 0xFu, M = c & 7u;
  if (E) return static_cast<uint16_t>(((E + 8u) << 10) | (M << 7));
  // subnormal E4M3: M * 2^-9 = fp16 normal (M in 1..7)
  if (M == 0) return 0;
  const uint32_t lz = __clz(M) - 29;           // 0 for M >= 4, 1 for 2..3, 2 for 1
  const uint32_t mm = (M << lz) & 3u;          // remaining fraction bits after the leading 1
  const uint32_t e = 15u - 9u + 2u - lz;       // exponent of M * 2^-9 with M = 1.mm * 2^(2-lz)
  return static_cast<uint16_t>((e << 10) | (mm << 8));
}

}  // namespace csa2
