// Pieces shared by the Full scan (csa2_index_full) and the pool re-score
// (csa2_reindex), so that both produce bit-identical fp32 scores:
//   * quantisation of one request's indexer query into the swizzled B-operand
//     tile (32 heads x 128 FP8 codes) plus w_h * sigma^q_h per head;
//   * the score epilogue  s_t = sigma_t * sum_h (w_h sigma^q_h) * ReLU(acc_h)
//     with a fixed summation order h = 0..31 (fp32 FMA).
// Score reading (the pages give none): s_t = sigma_t * sum_h w_h *
// ReLU(sigma^q_h <q^_h, k^_t>) [4sapi blog, section 四: 32 heads x 128].
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kTileBytes = kTile * kIndexDim;          // 16 KB: 128 rows x 128 B
constexpr int kQBytes = kIndexHeads * kIndexDim;       // 4 KB: 32 rows x 128 B
constexpr int kAccCols = 32;                           // fp32 columns per accumulator (N = 32 heads)
constexpr uint32_t kIdesc = idesc_e4m3_f32(kTile, kIndexHeads);

// Byte offset of (row, byte c) in a 128-byte-swizzled tile of 128-byte rows.
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t c) {
  return row * 128u + ((((c >> 4) ^ row) & 7u) << 4) + (c & 15u);
}

// Quantise heads 8*ew .. 8*ew+7 of query q[32][128] (fp32, row-major) into
// `qtile` (swizzled FP8 codes) and store ws[h] = w[h] * sigma^q_h for those
// heads into ws_sh.  One warp per call (four warps cover a query); the eight
// heads' loads are issued together.
__device__ __forceinline__ void prepare_query_part(const float* __restrict__ q, const float* __restrict__ w,
                                                   uint8_t* qtile, float* ws_sh, int ew, int lane) {
  float4 v[8];
#pragma unroll
  for (int hh = 0; hh < 8; ++hh) v[hh] = reinterpret_cast<const float4*>(q + (ew * 8 + hh) * kIndexDim)[lane];
  const float wl = lane < 8 ? w[ew * 8 + lane] : 0.0f;
#pragma unroll
  for (int hh = 0; hh < 8; ++hh) {
    const int h = ew * 8 + hh;
    float m = fmaxf(fmaxf(fabsf(v[hh].x), fabsf(v[hh].y)), fmaxf(fabsf(v[hh].z), fabsf(v[hh].w)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const int e = indexer_exponent(m);
    const float inv = exp2i(-e);
    const uint32_t codes = e4m3x2(v[hh].x * inv, v[hh].y * inv) | (e4m3x2(v[hh].z * inv, v[hh].w * inv) << 16);
    *reinterpret_cast<uint32_t*>(qtile + sw128_offset(h, 4u * lane)) = codes;
    if (lane == hh) ws_sh[h] = wl * exp2i(e);
  }
}

// Quantise heads 8*ew .. 8*ew+7 of query q[32][128] into `qtile` (swizzled
// FP8 codes) only.  One warp per call; the eight heads' loads are issued
// together.
__device__ __forceinline__ void prepare_query_codes(const float* __restrict__ q, uint8_t* qtile, int ew, int lane) {
  float4 v[8];
#pragma unroll
  for (int hh = 0; hh < 8; ++hh) v[hh] = reinterpret_cast<const float4*>(q + (ew * 8 + hh) * kIndexDim)[lane];
#pragma unroll
  for (int hh = 0; hh < 8; ++hh) {
    float m = fmaxf(fmaxf(fabsf(v[hh].x), fabsf(v[hh].y)), fmaxf(fabsf(v[hh].z), fabsf(v[hh].w)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float inv = exp2i(-indexer_exponent(m));
    const uint32_t codes = e4m3x2(v[hh].x * inv, v[hh].y * inv) | (e4m3x2(v[hh].z * inv, v[hh].w * inv) << 16);
    *reinterpret_cast<uint32_t*>(qtile + sw128_offset(ew * 8 + hh, 4u * lane)) = codes;
  }
}

// ws[h] = w[h] * sigma^q_h for all 32 heads, in every lane of the calling
// warp; eight heads' loads are in flight at a time.
__device__ __forceinline__ void load_head_weights(const float* __restrict__ q, const float* __restrict__ w,
                                                  float (&ws)[32], int lane) {
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    float4 v[8];
#pragma unroll
    for (int hh = 0; hh < 8; ++hh) v[hh] = reinterpret_cast<const float4*>(q + (g * 8 + hh) * kIndexDim)[lane];
    const float wl = lane < 8 ? w[g * 8 + lane] : 0.0f;
#pragma unroll
    for (int hh = 0; hh < 8; ++hh) {
      float m = fmaxf(fmaxf(fabsf(v[hh].x), fabsf(v[hh].y)), fmaxf(fabsf(v[hh].z), fabsf(v[hh].w)));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      ws[g * 8 + hh] = __shfl_sync(0xffffffffu, wl, hh) * exp2i(indexer_exponent(m));
    }
  }
}

// Score of one position from its 32 fp32 head dot products.
__device__ __forceinline__ float score_from_acc(const uint32_t (&acc)[32], const float (&ws)[32], uint32_t e_byte) {
  float s = 0.0f;
#pragma unroll
  for (int h = 0; h < 32; ++h) s = fmaf(ws[h], fmaxf(__uint_as_float(acc[h]), 0.0f), s);
  return s * exp2i(static_cast<int>(e_byte) - 127);
}

}  // namespace csa2
