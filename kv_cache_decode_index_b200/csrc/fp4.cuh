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

// E4M3 code nearest to amax / 6 (ties to the even code, saturating at 448),
// from the correctly rounded fp32 quotient and the hardware conversion (round
// to nearest even, saturating).  The rounded quotient lies on the same side
// of every E4M3 midpoint as the exact one: a midpoint m has at most 5
// significant bits, so 6m is an fp32 value; amax either equals 6m (and the
// quotient is m exactly) or differs from it by at least one ulp of 6m's
// binade, which is more than 6 times the quotient's rounding error (half an
// ulp of m's binade, a quarter to an eighth of 6m's).  NaN gives code 0.
__device__ __forceinline__ uint32_t e4m3_code_of_sixth(float amax) {
  if (!(amax >= 0.0f)) return 0u;
  const float x = amax / 6.0f;
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));   // low byte: x
  return r & 0xFFu;
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

// FP4 indexer row (128 elements: E2M1 codes with one E4M3 scale per 16,
// s = E4M3(amax / 6); the main-KV format on the indexer's row) held by a warp,
// lane l owning elements 4l .. 4l+3 of group l / 4.  Returns the lane's two
// code bytes (element 4l in the low nibble of the low byte) and the group's
// scale code in *scale.
__device__ __forceinline__ uint32_t fp4_row_lane(float4 v, uint32_t* scale) {
  float m = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
  const uint32_t sc = e4m3_code_of_sixth(m);
  const float s = e4m3_value(sc);
  *scale = sc;
  if (!(s > 0.0f)) return 0u;
  return e2m1_code(v.x, s) | (e2m1_code(v.y, s) << 4) | (e2m1_code(v.z, s) << 8) | (e2m1_code(v.w, s) << 12);
}

// FP4 codes and block scales of query heads 8*ew .. 8*ew+7 of q [32][128]
// (one warp) as rows row0 + h of a tensor-core B operand: the codes into the
// 64-byte-swizzled tile `qtile`, the scales into `qscale` in the tensor-core
// order (row0 + 32 <= 128).
__device__ __forceinline__ void prepare_query_fp4(const float* __restrict__ q, uint8_t* qtile, uint8_t* qscale,
                                                  int row0, int ew, int lane) {
  float4 v[8];
#pragma unroll
  for (int hh = 0; hh < 8; ++hh) v[hh] = reinterpret_cast<const float4*>(q + (ew * 8 + hh) * kIndexDim)[lane];
#pragma unroll
  for (int hh = 0; hh < 8; ++hh) {
    const uint32_t r = static_cast<uint32_t>(row0 + ew * 8 + hh);
    uint32_t sc;
    const uint32_t codes = fp4_row_lane(v[hh], &sc);
    *reinterpret_cast<uint16_t*>(qtile + sw64_offset(r, 2u * lane)) = static_cast<uint16_t>(codes);
    if ((lane & 3) == 0) qscale[block_scale_offset(r, lane >> 2)] = static_cast<uint8_t>(sc);
  }
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
