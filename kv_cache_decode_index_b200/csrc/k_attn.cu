// Sparse MQA attention over the gathered Top-k rows of the FP4 main KV
// (K = V = the dequantised 512-d row) [readance summary, section 4.2; 4sapi
// blog, section 二: every layer attends over its Top-K, Reuse layers with
// their own query; FP4 rows: 4sapi blog, section 五].
//
// One CTA per (query, tile of 16 heads); it walks the query's k rows in
// chunks of 64:
//   * the rows' cache addresses are resolved once (Top-k entry -> page);
//   * the raw FP4 rows (256 code bytes + 32 scale bytes) of the next chunk are
//     staged with cp.async while the current chunk is processed;
//   * dequantisation: E2M1 code x E4M3 scale has <= 5 significant bits and lies
//     in [2^-10, 2688], so the fp16 row is exact; codes become fp16 through a
//     byte-permute table lookup;
//   * the query is moved to fp16 with a power-of-two scale per head (bf16 ->
//     fp16 keeps every significant bit in the normal range);
//   * S = Q K^T (each warp 8 keys) and O = P V (each warp 64 output dims) on
//     mma.sync m16n8k16, fp16 in, fp32 accumulate; online softmax in fp32 in the
//     exp2 domain, P rounded to fp16.
// No cross-CTA reduction, no scratch memory.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fp4.cuh"
#include "launch.h"

namespace csa2 {

namespace {

constexpr int kAThreads = 256;
constexpr int kChunk = 64;                   // rows per chunk
constexpr int kHT = 16;                      // heads per CTA
constexpr int kRowBytes = kKvDim * 2;        // fp16 row: 1024 B
constexpr int kRawRow = kKvCodeBytes + kKvScaleBytes;   // 288 B
constexpr int kSStride = kChunk + 4;         // fp32 row stride of S
constexpr float kLog2e = 1.4426950408889634f;

struct AttnLayout {
  static constexpr uint32_t q_off = 0;                                  // fp16 [16][512], swizzled
  static constexpr uint32_t kv_off = q_off + kHT * kRowBytes;           // fp16 [64][512], swizzled
  static constexpr uint32_t raw_off = kv_off + kChunk * kRowBytes;      // u8 [2][64][288]
  static constexpr uint32_t s_off = raw_off + 2 * kChunk * kRawRow;     // fp32 [16][68]
  static constexpr uint32_t p_off = s_off + kHT * kSStride * 4;         // fp16 [16][64], swizzled (128 B rows)
  static constexpr uint32_t st_off = p_off + kHT * kChunk * 2;          // fp32 qscale[16], m[16], l[16], corr[16]
  static constexpr uint32_t rows_off = st_off + 4 * kHT * 4;            // int32 [k] cache row of each entry
  __host__ __device__ static uint32_t total(int k) { return rows_off + 4u * static_cast<uint32_t>(k); }
};

__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t chunk) {   // 16-byte chunk of a 1 KB row
  return row * kRowBytes + ((chunk ^ (row & 7u)) << 4);
}
__device__ __forceinline__ uint32_t swz_p(uint32_t row, uint32_t chunk) {  // 16-byte chunk of a 128 B row
  return row * (kChunk * 2) + ((chunk ^ (row & 7u)) << 4);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// Four E2M1 codes (two bytes, low nibble first) -> four fp16 values times the
// fp16 scale s2 (two half2 words).  The magnitude bits index a byte table of
// the fp16 high bytes of 0, 0.5, 1, 1.5, 2, 3, 4, 6; the sign bit of each code
// becomes bit 15 of its fp16.
__device__ __forceinline__ uint2 e2m1x4_to_half2(uint32_t two_bytes, __half2 s2) {
  // the permute selects byte n by the low 3 bits of nibble n: code n's magnitude
  const uint32_t hib = __byte_perm(0x3E3C3800u, 0x46444240u, two_bytes);            // table[code & 7] per byte
  // code n spread to byte n, so that its sign bit (bit 3) moves to bit 7 of byte n
  const uint32_t spread = (two_bytes & 0xFu) | ((two_bytes & 0xF0u) << 4) | ((two_bytes & 0xF00u) << 8) |
                          ((two_bytes & 0xF000u) << 12);
  const uint32_t sgn = (spread << 4) & 0x80808080u;
  const uint32_t h = hib | sgn;
  uint32_t w0 = __byte_perm(h, 0u, 0x1404u);   // [0, h0, 0, h1]: fp16 of codes 0, 1
  uint32_t w1 = __byte_perm(h, 0u, 0x3424u);   // fp16 of codes 2, 3
  __half2 v0 = __hmul2(*reinterpret_cast<__half2*>(&w0), s2);
  __half2 v1 = __hmul2(*reinterpret_cast<__half2*>(&w1), s2);
  return make_uint2(*reinterpret_cast<uint32_t*>(&v0), *reinterpret_cast<uint32_t*>(&v1));
}

__global__ void __launch_bounds__(kAThreads, 1)
    sparse_attn_kernel(const csa2_cache cache, const int32_t* __restrict__ q_req, const int32_t* __restrict__ topk,
                       int K, int H, const __nv_bfloat16* __restrict__ qg, float softmax_scale,
                       __nv_bfloat16* __restrict__ out) {
  using L = AttnLayout;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  float* s_sh = reinterpret_cast<float*>(smem + L::s_off);
  float* qscale = reinterpret_cast<float*>(smem + L::st_off);
  float* m_sh = qscale + kHT;
  float* l_sh = m_sh + kHT;
  float* corr_sh = l_sh + kHT;
  int* rows = reinterpret_cast<int*>(smem + L::rows_off);

  const int tiles_per_q = H / kHT;
  const int qi = blockIdx.x / tiles_per_q, ht = blockIdx.x % tiles_per_q;
  const int b = q_req != nullptr ? q_req[qi] : qi;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long capacity = static_cast<long long>(cache.max_pages_per_req) * cache.page_size;
  int n = (b >= 0 && b < cache.batch) ? cache.ctx_len[b] : 0;
  n = n < 0 ? 0 : (n > capacity ? static_cast<int>(capacity) : n);
  const int32_t* idx = topk + static_cast<long long>(qi) * K;

  // ---- cache row of every Top-k entry (-1: skipped) ----
  for (int base = 0; base < K; base += kAThreads * 4) {
    int t[4], pg[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = base + u * kAThreads + tid;
      t[u] = i < K ? idx[i] : -1;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      pg[u] = (t[u] >= 0 && t[u] < n)
                  ? cache.page_table[static_cast<long long>(b) * cache.max_pages_per_req + t[u] / cache.page_size]
                  : -1;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = base + u * kAThreads + tid;
      if (i >= K) continue;
      int row = -1;
      if (t[u] >= 0 && t[u] < n) {
        if (pg[u] >= 0 && pg[u] < cache.num_pages) row = pg[u] * cache.page_size + t[u] % cache.page_size;
        else if (ht == 0) report_error(cache.err_word, CSA2_ERR_DEVICE_BOUNDS, kKAttn, b, t[u]);
      } else if (t[u] != -1 && ht == 0) {
        report_error(cache.err_word, CSA2_ERR_DEVICE_BOUNDS, kKAttn, b, t[u]);
      }
      rows[i] = row;
    }
  }

  // ---- query heads [16 ht, 16 ht + 16) -> fp16 with a power-of-two scale per head ----
  {
    uint4 raw[2][2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int h = ht * kHT + warp * 2 + hh;
      const uint4* src = reinterpret_cast<const uint4*>(qg + (static_cast<long long>(qi) * H + h) * kKvDim) + lane * 2;
      raw[hh][0] = src[0];
      raw[hh][1] = src[1];
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int hl = warp * 2 + hh;   // head inside the tile
      const uint4 v0 = raw[hh][0], v1 = raw[hh][1];
      const uint32_t wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      float f[16];
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        f[2 * i] = __uint_as_float(wv[i] << 16);
        f[2 * i + 1] = __uint_as_float(wv[i] & 0xFFFF0000u);
        amax = fmaxf(amax, fmaxf(fabsf(f[2 * i]), fabsf(f[2 * i + 1])));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      int E = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF) - 127;   // amax in [2^E, 2^(E+1))
      if (amax == 0.0f) E = 14;
      E = max(E, -100);
      const float up = exp2i(14 - E), down = exp2i(E - 14);
      uint32_t hv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) hv[i] = pack_half2(f[2 * i] * up, f[2 * i + 1] * up);
      *reinterpret_cast<uint4*>(smem + L::q_off + swz(hl, 2 * lane)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
      *reinterpret_cast<uint4*>(smem + L::q_off + swz(hl, 2 * lane + 1)) = make_uint4(hv[4], hv[5], hv[6], hv[7]);
      if (lane == 0) {
        qscale[hl] = softmax_scale * down * kLog2e;
        m_sh[hl] = -INFINITY;
        l_sh[hl] = 0.0f;
      }
    }
  }
  __syncthreads();   // rows[] ready

  // ---- staging of a chunk's raw rows: 64 rows x 18 pieces of 16 bytes ----
  const int nchunks = (K + kChunk - 1) / kChunk;
  auto stage = [&](int c) {
    const uint32_t dst0 = sbase + L::raw_off + (c & 1) * kChunk * kRawRow;
    for (int p = tid; p < kChunk * (kRawRow / 16); p += kAThreads) {
      const int r = p / (kRawRow / 16), u = p % (kRawRow / 16);
      const int key = c * kChunk + r;
      const int row = key < K ? rows[key] : -1;
      if (row < 0) continue;
      const uint8_t* src =
          u < kKvCodeBytes / 16
              ? cache.kv_codes + static_cast<long long>(row) * kKvCodeBytes + u * 16
              : cache.kv_scales + static_cast<long long>(row) * kKvScaleBytes + (u - kKvCodeBytes / 16) * 16;
      cp_async16(dst0 + r * kRawRow + u * 16, src);
    }
    cp_async_commit();
  };
  stage(0);

  float o_acc[8][4];   // O[16 heads x 64 dims of this warp]
#pragma unroll
  for (int i = 0; i < 8; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.0f;
  const int r0 = lane >> 2;

  for (int c = 0; c < nchunks; ++c) {
    if (c + 1 < nchunks) stage(c + 1);
    else cp_async_commit();   // keep the group count uniform
    cp_async_wait_1();        // chunk c has landed (this thread's copies)
    __syncthreads();          // ... and everyone's

    // ---- dequantise chunk c: thread = (row, quarter of 128 channels) ----
    {
      const int row = tid >> 2, part = tid & 3;
      const uint8_t* raw = smem + L::raw_off + (c & 1) * kChunk * kRawRow + row * kRawRow;
      const int key = c * kChunk + row;
      const bool valid = key < K && rows[key] >= 0;
      const uint4* cw = reinterpret_cast<const uint4*>(raw + part * 64);
      const uint2 sc = *reinterpret_cast<const uint2*>(raw + kKvCodeBytes + part * 8);
#pragma unroll
      for (int j = 0; j < 4; ++j) {   // 16 code bytes = 32 channels = 2 scale groups
        const uint4 v = valid ? cw[j] : make_uint4(0, 0, 0, 0);
        const uint32_t sbytes = j < 2 ? (sc.x >> (16 * j)) : (sc.y >> (16 * (j - 2)));
        const uint16_t s0b = valid ? e4m3_half_bits(sbytes & 0xFFu) : 0;
        const uint16_t s1b = valid ? e4m3_half_bits((sbytes >> 8) & 0xFFu) : 0;
        const __half2 s0 = __halves2half2(__ushort_as_half(s0b), __ushort_as_half(s0b));
        const __half2 s1 = __halves2half2(__ushort_as_half(s1b), __ushort_as_half(s1b));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t hv[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {   // 4 code bytes = 8 channels per word
          const uint2 lo = e2m1x4_to_half2(w[q] & 0xFFFFu, q < 2 ? s0 : s1);
          const uint2 hi = e2m1x4_to_half2(w[q] >> 16, q < 2 ? s0 : s1);
          hv[4 * q] = lo.x;
          hv[4 * q + 1] = lo.y;
          hv[4 * q + 2] = hi.x;
          hv[4 * q + 3] = hi.y;
        }
        const int chunk0 = part * 16 + j * 4;   // 8 fp16 per 16-byte chunk
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4*>(smem + L::kv_off + swz(row, chunk0 + q)) =
              make_uint4(hv[4 * q], hv[4 * q + 1], hv[4 * q + 2], hv[4 * q + 3]);
      }
    }
    __syncthreads();

    // ---- S = Q K^T: warp w scores keys [8w, 8w + 8) over all 512 dims ----
    {
      float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
      for (int ks = 0; ks < kKvDim / 16; ++ks) {
        uint32_t a0, a1, a2, a3, b0, b1;
        ldsm_x4(sbase + L::q_off + swz(lane & 15, 2 * ks + (lane >> 4)), a0, a1, a2, a3);
        ldsm_x2(sbase + L::kv_off + swz(warp * 8 + (lane & 7), 2 * ks + ((lane >> 3) & 1)), b0, b1);
        mma_f16(s, a0, a1, a2, a3, b0, b1);
      }
      const int col = warp * 8 + 2 * (lane & 3);
      const int k0 = c * kChunk + col;
      const bool v0 = k0 < K && rows[k0] >= 0, v1 = k0 + 1 < K && rows[k0 + 1] >= 0;
      const float sc0 = qscale[r0], sc1 = qscale[r0 + 8];
      s_sh[r0 * kSStride + col] = v0 ? s[0] * sc0 : -INFINITY;
      s_sh[r0 * kSStride + col + 1] = v1 ? s[1] * sc0 : -INFINITY;
      s_sh[(r0 + 8) * kSStride + col] = v0 ? s[2] * sc1 : -INFINITY;
      s_sh[(r0 + 8) * kSStride + col + 1] = v1 ? s[3] * sc1 : -INFINITY;
    }
    __syncthreads();

    // ---- online softmax: warp w owns heads 2w, 2w+1 ----
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int h = warp * 2 + hh;
      const float x0 = s_sh[h * kSStride + lane], x1 = s_sh[h * kSStride + lane + 32];
      float mx = fmaxf(x0, x1);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_old = m_sh[h];
      const float m_new = fmaxf(m_old, mx);
      const float ref = m_new == -INFINITY ? 0.0f : m_new;
      const float p0 = exp2f(x0 - ref), p1 = exp2f(x1 - ref);
      float sum = p0 + p1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      // P[h][lane] and P[h][lane + 32] as fp16: 128-byte rows, swizzled 16-byte chunks
      *reinterpret_cast<__half*>(smem + L::p_off + swz_p(h, lane >> 3) + (lane & 7) * 2) = __float2half_rn(p0);
      *reinterpret_cast<__half*>(smem + L::p_off + swz_p(h, (lane + 32) >> 3) + (lane & 7) * 2) = __float2half_rn(p1);
      __syncwarp();
      if (lane == 0) {
        const float cr = exp2f(m_old - ref);   // 0 when m_old = -inf
        corr_sh[h] = cr;
        l_sh[h] = l_sh[h] * cr + sum;
        m_sh[h] = m_new;
      }
    }
    __syncthreads();

    // ---- O = O * corr + P V: warp w owns output dims [64w, 64w + 64) ----
    {
      const float c0 = corr_sh[r0], c1 = corr_sh[r0 + 8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        o_acc[i][0] *= c0;
        o_acc[i][1] *= c0;
        o_acc[i][2] *= c1;
        o_acc[i][3] *= c1;
      }
#pragma unroll
      for (int kk = 0; kk < kChunk / 16; ++kk) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(sbase + L::p_off + swz_p(lane & 15, 2 * kk + (lane >> 4)), a0, a1, a2, a3);
#pragma unroll
        for (int np = 0; np < 4; ++np) {   // pairs of 8-dim tiles
          const int mi = lane >> 3;
          const int dchunk = warp * 8 + np * 2 + (mi >> 1);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(sbase + L::kv_off + swz(kk * 16 + (mi & 1) * 8 + (lane & 7), dchunk), b0, b1, b2, b3);
          mma_f16(o_acc[2 * np], a0, a1, a2, a3, b0, b1);
          mma_f16(o_acc[2 * np + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
    __syncthreads();   // kv, S and P are rewritten by the next chunk
  }

  // ---- normalise and write bf16 ----
  const float l0 = l_sh[r0], l1 = l_sh[r0 + 8];
  const float i0 = l0 > 0.0f ? 1.0f / l0 : 0.0f, i1 = l1 > 0.0f ? 1.0f / l1 : 0.0f;
  const long long head0 = static_cast<long long>(qi) * H + ht * kHT;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int col = warp * 64 + i * 8 + 2 * (lane & 3);
    const __nv_bfloat162 v0 = __floats2bfloat162_rn(o_acc[i][0] * i0, o_acc[i][1] * i0);
    const __nv_bfloat162 v1 = __floats2bfloat162_rn(o_acc[i][2] * i1, o_acc[i][3] * i1);
    *reinterpret_cast<__nv_bfloat162*>(out + (head0 + r0) * kKvDim + col) = v0;
    *reinterpret_cast<__nv_bfloat162*>(out + (head0 + r0 + 8) * kKvDim + col) = v1;
  }
}

}  // namespace

cudaError_t launch_sparse_attn(const csa2_cache& cache, int n_queries, const int32_t* q_req, const int32_t* topk,
                               int k, const uint16_t* q, int H, float scale, uint16_t* out, cudaStream_t stream) {
  static bool done = false;
  constexpr int kMaxK = 4096;
  if (!done) {
    const cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(AttnLayout::total(kMaxK)));
    if (e != cudaSuccess) return e;
    done = true;
  }
  sparse_attn_kernel<<<n_queries * (H / kHT), kAThreads, AttnLayout::total(k), stream>>>(
      cache, q_req, topk, k, H, reinterpret_cast<const __nv_bfloat16*>(q), scale,
      reinterpret_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

}  // namespace csa2
