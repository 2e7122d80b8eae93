// Quantise-on-append (and the sequence compressor in front of it): one warp
// per new row.
//
// Main KV (512 fp32) -> 256 bytes of E2M1 pairs + 32 E4M3 scales; lane g owns
// channel group g (16 channels): s = E4M3(amax / 6), codes = E2M1(x / s)
// [FP4 main-KV format: 4sapi "DeepSeek V4.1 Flash CED/CSA2" blog, section 五;
// animattoys article, section 把精度降到4比特].
// Indexer K (128 fp32) -> 128 E4M3 bytes + one exponent byte, sigma = 2^e with
// e the smallest integer such that 448 * 2^e >= amax (reading: the pages give
// no indexer dtype).
#include "fp4.cuh"
#include "launch.h"

namespace csa2 {

namespace {

// Cache row of position t of request b, or -1 (error recorded) when the
// request, the position or its page is out of range.
__device__ __forceinline__ long long row_of(const csa2_cache& cache, int b, int t, int lane) {
  const long long capacity = static_cast<long long>(cache.max_pages_per_req) * cache.page_size;
  if (b < 0 || b >= cache.batch || t < 0 || t >= capacity) {
    if (lane == 0) report_error(cache.err_word, CSA2_ERR_DEVICE_BOUNDS, kKAppend, b, t);
    return -1;
  }
  const int page = cache.page_table[static_cast<long long>(b) * cache.max_pages_per_req + t / cache.page_size];
  if (page < 0 || page >= cache.num_pages) {
    if (lane == 0) report_error(cache.err_word, CSA2_ERR_DEVICE_BOUNDS, kKAppend, b, t);
    return -1;
  }
  return static_cast<long long>(page) * cache.page_size + t % cache.page_size;
}

// Quantise one row held by a warp and store it: x = main-KV channels
// 16*lane .. 16*lane+15, k = indexer-K elements 4*lane .. 4*lane+3.
__device__ __forceinline__ void quantize_store(const csa2_cache& cache, long long row, const float (&x)[16], float4 k,
                                               int lane) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
  const uint32_t sc = e4m3_code_of_sixth(amax);
  const float s = e4m3_value(sc);
  uint32_t lo = 0, hi = 0;
  if (s > 0.0f) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t byte = e2m1_code(x[2 * i], s) | (e2m1_code(x[2 * i + 1], s) << 4);
      if (i < 4) lo |= byte << (8 * i);
      else hi |= byte << (8 * (i - 4));
    }
  }
  reinterpret_cast<uint2*>(cache.kv_codes + row * kKvCodeBytes)[lane] = make_uint2(lo, hi);
  cache.kv_scales[row * kKvScaleBytes + lane] = static_cast<uint8_t>(sc);

  float km = fmaxf(fmaxf(fabsf(k.x), fabsf(k.y)), fmaxf(fabsf(k.z), fabsf(k.w)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) km = fmaxf(km, __shfl_xor_sync(0xffffffffu, km, o));
  const int e = indexer_exponent(km);
  const float inv = exp2i(-e);
  const uint32_t codes = e4m3x2(k.x * inv, k.y * inv) | (e4m3x2(k.z * inv, k.w * inv) << 16);
  reinterpret_cast<uint32_t*>(cache.ik_codes + row * kIndexDim)[lane] = codes;
  if (lane == 0) cache.ik_exp[row] = static_cast<uint8_t>(e + 127);
}

__global__ void __launch_bounds__(256) append_kernel(csa2_cache cache, int n_rows, const float* __restrict__ kv_new,
                                                     const float* __restrict__ ik_new,
                                                     const int32_t* __restrict__ req,
                                                     const int32_t* __restrict__ pos) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n_rows) return;
  const long long row = row_of(cache, req ? req[warp] : warp, pos[warp], lane);
  if (row < 0) return;
  const float4* src = reinterpret_cast<const float4*>(kv_new + static_cast<long long>(warp) * kKvDim) + lane * 4;
  float x[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 v = src[i];
    x[4 * i] = v.x; x[4 * i + 1] = v.y; x[4 * i + 2] = v.z; x[4 * i + 3] = v.w;
  }
  const float4 k = reinterpret_cast<const float4*>(ik_new + static_cast<long long>(warp) * kIndexDim)[lane];
  quantize_store(cache, row, x, k, lane);
}

// Sequence compressor + quantise-on-append: entry i is the mean of token rows
// m*i .. m*i + m - 1 (summed in fp64 in token order, scaled by 1/m, m a power
// of two, rounded once to fp32), then stored like an appended row
// [4sapi blog, section 三: encoder groups compress the sequence with m = 2].
__global__ void __launch_bounds__(256) compress_append_kernel(csa2_cache cache, int n_entries, int m,
                                                              const float* __restrict__ kv_tok,
                                                              const float* __restrict__ ik_tok,
                                                              const int32_t* __restrict__ req,
                                                              const int32_t* __restrict__ pos) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n_entries) return;
  const long long row = row_of(cache, req ? req[warp] : 0, pos[warp], lane);
  if (row < 0) return;
  double xs[16], ks[4];
#pragma unroll
  for (int i = 0; i < 16; ++i) xs[i] = 0.0;
#pragma unroll
  for (int i = 0; i < 4; ++i) ks[i] = 0.0;
  const long long t0 = static_cast<long long>(warp) * m;
  for (int j = 0; j < m; ++j) {
    const float4* src = reinterpret_cast<const float4*>(kv_tok + (t0 + j) * kKvDim) + lane * 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = src[i];
      xs[4 * i] += v.x; xs[4 * i + 1] += v.y; xs[4 * i + 2] += v.z; xs[4 * i + 3] += v.w;
    }
    const float4 k = reinterpret_cast<const float4*>(ik_tok + (t0 + j) * kIndexDim)[lane];
    ks[0] += k.x; ks[1] += k.y; ks[2] += k.z; ks[3] += k.w;
  }
  const double inv_m = 1.0 / m;   // exact: m is a power of two
  float x[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) x[i] = __double2float_rn(xs[i] * inv_m);
  const float4 k = make_float4(__double2float_rn(ks[0] * inv_m), __double2float_rn(ks[1] * inv_m),
                               __double2float_rn(ks[2] * inv_m), __double2float_rn(ks[3] * inv_m));
  quantize_store(cache, row, x, k, lane);
}

// Sliding-window (SWA) KV append: one warp per row; the 512-d row is stored
// in FP8 E4M3 with one power-of-two scale, by the indexer's per-row rule, in
// ring slot pos % window of its request [4sapi blog, section 五: the local
// SWA KV stays in FP8].
__global__ void __launch_bounds__(256) swa_append_kernel(csa2_cache cache, int window, uint8_t* __restrict__ codes,
                                                         uint8_t* __restrict__ exps, int n_rows,
                                                         const float* __restrict__ x, const int32_t* __restrict__ req,
                                                         const int32_t* __restrict__ pos) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n_rows) return;
  const int b = req ? req[warp] : warp;
  const int t = pos[warp];
  if (b < 0 || b >= cache.batch || t < 0) {
    if (lane == 0) report_error(cache.err_word, CSA2_ERR_DEVICE_BOUNDS, kKAppend, b, t);
    return;
  }
  const float4* src = reinterpret_cast<const float4*>(x + static_cast<long long>(warp) * kKvDim) + lane * 4;
  float v[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 f = src[i];
    v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
  }
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const int e = indexer_exponent(m);
  const float inv = exp2i(-e);
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    w[i] = e4m3x2(v[4 * i] * inv, v[4 * i + 1] * inv) | (e4m3x2(v[4 * i + 2] * inv, v[4 * i + 3] * inv) << 16);
  const long long slot = static_cast<long long>(b) * window + t % window;
  reinterpret_cast<uint4*>(codes + slot * kKvDim)[lane] = make_uint4(w[0], w[1], w[2], w[3]);
  if (lane == 0) exps[slot] = static_cast<uint8_t>(e + 127);
}

}  // namespace

cudaError_t launch_swa_append(const csa2_cache& cache, int window, uint8_t* swa_codes, uint8_t* swa_exp, int n_rows,
                              const float* x, const int32_t* req, const int32_t* pos, cudaStream_t stream) {
  const int threads = 256;
  const long long blocks = (static_cast<long long>(n_rows) * 32 + threads - 1) / threads;
  swa_append_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(cache, window, swa_codes, swa_exp, n_rows,
                                                                          x, req, pos);
  return cudaGetLastError();
}

cudaError_t launch_compress_append(const csa2_cache& cache, int n_entries, int m, const float* kv_tok,
                                   const float* ik_tok, const int32_t* req, const int32_t* pos, cudaStream_t stream) {
  const int threads = 256;
  const long long blocks = (static_cast<long long>(n_entries) * 32 + threads - 1) / threads;
  compress_append_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(cache, n_entries, m, kv_tok, ik_tok,
                                                                               req, pos);
  return cudaGetLastError();
}

cudaError_t launch_append(const csa2_cache& cache, int n_rows, const float* kv_new, const float* ik_new,
                          const int32_t* req, const int32_t* pos, cudaStream_t stream) {
  const int threads = 256;
  const long long blocks = (static_cast<long long>(n_rows) * 32 + threads - 1) / threads;
  append_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(cache, n_rows, kv_new, ik_new, req, pos);
  return cudaGetLastError();
}

}  // namespace csa2
