// Sparse MQA attention over the gathered Top-k rows of the FP4 main KV
// (K = V = the dequantised 512-d row) [readance summary, section 4.2; 4sapi
// blog, section 二: every layer attends over its Top-K, Reuse layers with
// their own query; FP4 rows: 4sapi blog, section 五].
//
// One thread-block cluster of CL CTAs (key splits) per (layer, query): 4 for
// up to 6 queries (a decode group's six layers of them fill one wave of the
// GPU's SMs), 2 for up to 12, else 1 (16 heads: always 4).  CTA r takes
// entries [r*kc, (r+1)*kc) (kc = ceil(k/CL)) in chunks of 64 rows:
//   * prologue: the query's bf16 rows are loaded and converted before the
//     wait on the preceding launch, then the CTA turns its Top-k entries into
//     cache rows (page table) once, into shared memory;
//   * the packed rows (256 code bytes + 32 scale bytes each) are copied into
//     a staging buffer by cp.async one chunk ahead of their use and
//     dequantised shared -> shared with the E2M1 -> f16x2 conversion: E2M1
//     code x E4M3 scale has <= 5 significant bits and lies in [2^-10, 2688],
//     so the fp16 row is exact;
//   * the query is moved to fp16 with a power-of-two scale per head (bf16 ->
//     fp16 keeps every significant bit in the normal range);
//   * S = Q K^T on mma.sync m16n8k16 (fp16 in, fp32 accumulate) with the
//     chunk's keys split over the warps, an online softmax in fp32 (exp2
//     domain) whose row maxima and sums are combined through shared memory,
//     P rounded to fp16 in shared memory, O += P V with each warp on 64 of
//     the 512 output dims of every head;
// then CTA r merges the CL partial (O, max, sum) sets for output dims
// [512r/CL, 512(r+1)/CL) and writes those dims of every head.  The partials
// reach it through a caller workspace in global memory (L2) when one is
// given, else by stores into its shared memory from the other CTAs
// (distributed shared memory), between cluster barriers.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>

#include "fp4.cuh"
#include "launch.h"

namespace csa2 {

namespace {

namespace cg = cooperative_groups;

constexpr int kAThreads = 256;
constexpr int kAWarps = kAThreads / 32;
constexpr int kAMaxCluster = 4;             // CTAs (key splits) per query, at most
constexpr int kChunk = 64;                   // keys per chunk
constexpr int kRowBytes = kKvDim * 2;        // fp16 row: 1024 B
constexpr int kPRowBytes = kChunk * 2;       // fp16 row of P: 128 B
constexpr int kPVDims = kKvDim / kAWarps;    // output dims per warp in P V: 64
constexpr int kCodeGran = kKvCodeBytes / 16;                    // 16-byte granules of a packed row's codes
constexpr int kRowGran = (kKvCodeBytes + kKvScaleBytes) / 16;   // ... of codes + scales
constexpr float kLog2e = 1.4426950408889634f;

// CL: CTAs (key splits) per query.
template <int H, int CL>
struct AttnLayout {
  static constexpr int kODims = kKvDim / CL;   // output dims owned by one CTA of the cluster
  // Top-k entries one CTA resolves: k <= 4096 and a window <= 4096 give at
  // most ceil((4096 + 4096) / CL) entries per CTA.
  static constexpr int kMaxTop = (4096 + CSA2_SWA_MAX_WINDOW + CL - 1) / CL;
  static constexpr int HT = H / 16;            // head tiles of 16 query rows
  static constexpr int KG = kAWarps / HT;      // key groups in S
  static constexpr int KW = kChunk / KG;       // keys per warp in S
  static constexpr int NT = KW / 8;            // 8-key tiles per warp in S
  static constexpr uint32_t q_off = 0;                                     // fp16 [H][512]
  static constexpr uint32_t kv_off = q_off + H * kRowBytes;                // fp16 [64][512]
  static constexpr uint32_t raw_off = kv_off + kChunk * kRowBytes;         // u8 [64][256] codes
  static constexpr uint32_t raw_scale_off = raw_off + kChunk * kKvCodeBytes;   // u8 [64][32] scales
  static constexpr uint32_t p_off = raw_scale_off + kChunk * kKvScaleBytes;    // fp16 [H][64]
  static constexpr uint32_t red_off = p_off + H * kPRowBytes;              // fp32 [2][KG][H]: row max, row sum
  static constexpr uint32_t qscale_off = red_off + 2 * KG * H * 4;
  static constexpr uint32_t kvalid_off = qscale_off + H * 4;               // int [64]
  static constexpr uint32_t srow_off = kvalid_off + kChunk * 4;            // int32 [kMaxTop] cache rows
  static constexpr uint32_t ml_off = srow_off + kMaxTop * 4;               // fp32 [CL][2][H]: m, l
  static constexpr uint32_t fac_off = ml_off + CL * 2 * H * 4;             // fp32 [CL][H]
  static constexpr uint32_t total = fac_off + CL * H * 4;
  // received partial O: [CL source ranks][H][kODims dims] fp32, over the Q + KV region
  static_assert(CL * H * kODims * 4 <= raw_off, "received partials must fit in the Q + KV region");
  static_assert(KW % 8 == 0 && (NT == 1 || NT % 2 == 0), "whole 8-key tiles per warp");
};

// Column (float index) of dim c of head h in a swizzled [H][dims] fp32
// slice: the 16-byte granule index is XORed with h % 8.
__device__ __forceinline__ int attn_swz(int h, int c) { return (((c >> 2) ^ (h & 7)) << 2) | (c & 3); }

__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t chunk) {   // 16-byte chunk of a 1 KB row
  return row * kRowBytes + ((chunk ^ (row & 7u)) << 4);
}
__device__ __forceinline__ uint32_t pswz(uint32_t row, uint32_t chunk) {  // 16-byte chunk of a 128 B row of P
  return row * kPRowBytes + ((chunk ^ (row & 7u)) << 4);
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

// cp.async (LSU path, no tensor map): 16 bytes global -> shared, completion
// tracked per thread by commit groups.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Two E2M1 codes (low nibble = even channel) -> f16x2, low half = even channel.
__device__ __forceinline__ uint32_t e2m1x2_half2(uint32_t byte) {
  const __half2_raw r = __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>(byte & 0xFFu), __NV_E2M1);
  return static_cast<uint32_t>(r.x) | (static_cast<uint32_t>(r.y) << 16);
}

// Dequantise 16 code bytes (32 channels, 2 scale groups) into 4 fp16 chunks.
__device__ __forceinline__ void dequant16(uint4 codes, uint32_t s01, uint4 (&out)[4]) {
  const uint32_t sc0 = e4m3_half_bits(s01 & 0xFFu), sc1 = e4m3_half_bits((s01 >> 8) & 0xFFu);
  const __half2 s0 = __halves2half2(__ushort_as_half(sc0), __ushort_as_half(sc0));
  const __half2 s1 = __halves2half2(__ushort_as_half(sc1), __ushort_as_half(sc1));
  const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
  uint32_t h[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t pair = e2m1x2_half2(w[i >> 2] >> (8 * (i & 3)));
    __half2 v = *reinterpret_cast<const __half2*>(&pair);
    v = __hmul2(v, i < 8 ? s0 : s1);   // exact: <= 5 significant bits, inside fp16's normal range
    h[i] = *reinterpret_cast<const uint32_t*>(&v);
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) out[c] = make_uint4(h[4 * c], h[4 * c + 1], h[4 * c + 2], h[4 * c + 3]);
}

// Top-k, query and output of each layer of one launch (layers may share a
// Top-k: a Full or Reindex layer and the Reuse layers that take its indices).
struct AttnLayers {
  const int32_t* topk[CSA2_ATTN_MAX_LAYERS];
  const __nv_bfloat16* q[CSA2_ATTN_MAX_LAYERS];
  __nv_bfloat16* out[CSA2_ATTN_MAX_LAYERS];
};

// The local sliding window (SWA) merged into the attention: FP8 E4M3 rows
// with one power-of-two scale each, a ring of `window` slots per request
// (token t in slot t % window); codes == nullptr: no window.
struct SwaArgs {
  const uint8_t* codes;      // [batch][window][512]
  const uint8_t* exp;        // [batch][window]
  const int32_t* q_pos;      // [n_queries] token position of each query
  int window;
};

template <int H, int CL>
__global__ void __launch_bounds__(kAThreads, H == 16 ? 2 : 1)
    sparse_attn_kernel(const csa2_cache cache, int n_queries, const int32_t* __restrict__ q_req,
                       int K, const __grid_constant__ AttnLayers io, float softmax_scale,
                       const SwaArgs swa, float* __restrict__ xchg) {
  using L = AttnLayout<H, CL>;
  constexpr int kODims = L::kODims;
  constexpr int kMaxTop = L::kMaxTop;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  float* red_max = reinterpret_cast<float*>(smem + L::red_off);   // [KG][H]
  float* red_sum = red_max + L::KG * H;                            // [KG][H]
  float* qscale = reinterpret_cast<float*>(smem + L::qscale_off);
  int* kvalid = reinterpret_cast<int*>(smem + L::kvalid_off);
  int32_t* srow = reinterpret_cast<int32_t*>(smem + L::srow_off);
  float* ml_sh = reinterpret_cast<float*>(smem + L::ml_off);
  float* fac = reinterpret_cast<float*>(smem + L::fac_off);

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int layer = static_cast<int>(blockIdx.x / CL) / n_queries;
  const int qi = static_cast<int>(blockIdx.x / CL) % n_queries;
  const __nv_bfloat16* __restrict__ qg = io.q[layer];
  __nv_bfloat16* __restrict__ out = io.out[layer];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ht = warp % L::HT, kg = warp / L::HT;

  // ---- query rows, loaded and converted before the wait on the preceding
  // launch (which does not write them) ----
  constexpr int kHpw = H / kAWarps;   // heads per warp
  uint4 raw[kHpw][2];
#pragma unroll
  for (int hh = 0; hh < kHpw; ++hh) {
    const uint4* src =
        reinterpret_cast<const uint4*>(qg + (static_cast<long long>(qi) * H + warp * kHpw + hh) * kKvDim) + lane * 2;
    raw[hh][0] = src[0];
    raw[hh][1] = src[1];
  }

  // ---- query -> fp16 with a power-of-two scale per head ----
#pragma unroll
  for (int hh = 0; hh < kHpw; ++hh) {
    const int h = warp * kHpw + hh;
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
    // lane holds dims [16*lane, 16*lane+16): chunks 2*lane, 2*lane+1
    *reinterpret_cast<uint4*>(smem + swz(h, 2 * lane)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
    *reinterpret_cast<uint4*>(smem + swz(h, 2 * lane + 1)) = make_uint4(hv[4], hv[5], hv[6], hv[7]);
    if (lane == 0) qscale[h] = softmax_scale * down * kLog2e;
  }

  pdl_wait();                 // everything the preceding launch wrote (the Top-k) is visible
  pdl_launch_dependents();
  const int b = q_req != nullptr ? q_req[qi] : qi;
  const long long capacity = static_cast<long long>(cache.max_pages_per_req) * cache.page_size;
  const bool b_ok = b >= 0 && b < cache.batch;
  if (!b_ok && rank == 0 && tid == 0) report_error(cache.err_word, CSA2_ERR_DEVICE_BOUNDS, kKAttn, b, -1);
  const int n_raw = b_ok ? checked_ctx_len(cache, b, capacity, kKAttn, rank == 0 && tid == 0) : -1;
  const int n = max(0, n_raw);   // n_raw < 0: no entry of this query is used (or checked)
  const int32_t* idx = io.topk[layer] + static_cast<long long>(qi) * K;

  // ---- this CTA's entries: the Top-k entries, then the window's tokens ----
  const int n_win = swa.codes != nullptr ? swa.window : 0;
  const int p_tok = n_win > 0 ? swa.q_pos[qi] : 0;
  const int K_all = K + n_win;
  const int kc = (K_all + CL - 1) / CL;
  const int key_begin = min(rank * kc, K_all), key_end = min(key_begin + kc, K_all);
  const int n_top = n_raw < 0 ? 0 : min(max(0, min(key_end, K) - key_begin), kMaxTop);
  for (int i = tid; i < n_top; i += kAThreads) {
    const int t = idx[key_begin + i];
    int r = -1;
    if (t >= 0 && t < n) {
      const int page = cache.page_table[static_cast<long long>(b) * cache.max_pages_per_req + t / cache.page_size];
      if (page >= 0 && page < cache.num_pages) r = page * cache.page_size + t % cache.page_size;
      else report_error(cache.err_word, CSA2_ERR_DEVICE_BOUNDS, kKAttn, b, t);
    } else if (t >= n || t < -1) {
      report_error(cache.err_word, CSA2_ERR_DEVICE_BOUNDS, kKAttn, b, t);
    }
    srow[i] = r;
  }
  __syncthreads();

  // cp.async of the packed rows of the chunk starting at entry c into the
  // staging buffer (code granules XOR-swizzled by row % 8)
  auto issue_chunk = [&](int c) {
    const int nk = min(kChunk, key_end - c);
    for (int g = tid; g < nk * kRowGran; g += kAThreads) {
      const int row = g / kRowGran, part = g - row * kRowGran;
      const int i = c + row - key_begin;
      if (c + row >= K || i >= n_top) continue;
      const int r = srow[i];
      if (r < 0) continue;
      if (part < kCodeGran)
        cp_async16(sbase + L::raw_off + row * kKvCodeBytes + ((part ^ (row & 7)) << 4),
                   cache.kv_codes + static_cast<long long>(r) * kKvCodeBytes + part * 16);
      else
        cp_async16(sbase + L::raw_scale_off + row * kKvScaleBytes + (part - kCodeGran) * 16,
                   cache.kv_scales + static_cast<long long>(r) * kKvScaleBytes + (part - kCodeGran) * 16);
    }
    cp_async_commit();
  };
  if (key_begin < key_end) issue_chunk(key_begin);

  // P V: warp w owns output dims [64w, 64w + 64) of every head; the running
  // max / sum of rows t*16 + r0 and t*16 + r0 + 8 of every head tile t are
  // kept in every warp (identical values)
  float o_acc[L::HT][kPVDims / 8][4];
#pragma unroll
  for (int t = 0; t < L::HT; ++t)
#pragma unroll
    for (int i = 0; i < kPVDims / 8; ++i) o_acc[t][i][0] = o_acc[t][i][1] = o_acc[t][i][2] = o_acc[t][i][3] = 0.0f;
  float m_run[L::HT][2], l_run[L::HT][2];
#pragma unroll
  for (int t = 0; t < L::HT; ++t) m_run[t][0] = m_run[t][1] = -INFINITY, l_run[t][0] = l_run[t][1] = 0.0f;
  const int r0 = lane >> 2;   // fragment row (and row + 8)
  const int h0 = ht * 16 + r0, h1 = h0 + 8;   // rows of this warp's S tile

  for (int c0 = key_begin; c0 < key_end; c0 += kChunk) {
    const int nk = min(kChunk, key_end - c0);
    cp_async_wait_all();
    __syncthreads();   // staged rows visible; the previous chunk's S and P V are done
    {
      // dequantise: thread (row, part) writes channels [128*part, 128*part + 128) of the row
      const int row = tid & (kChunk - 1), part = tid / kChunk;
      const int e = c0 + row;
      if (row < nk && e >= K) {
        // window entry j: token p - window + 1 + j (none before token 0)
        const int tw = p_tok - n_win + 1 + (e - K);
        const bool ok = tw >= 0 && n_raw >= 0;
        if (part == 0) kvalid[row] = ok;
        if (ok) {
          const long long slot = static_cast<long long>(b) * n_win + tw % n_win;
          const uint4* cp = reinterpret_cast<const uint4*>(swa.codes + slot * kKvDim) + part * 8;
          const float sigma = exp2i(static_cast<int>(swa.exp[slot]) - 127);
          uint4 cv[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) cv[j] = cp[j];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            // 16 E4M3 codes -> 16 fp16 values (exact while sigma keeps them in fp16's range)
            const uint32_t w4[4] = {cv[j].x, cv[j].y, cv[j].z, cv[j].w};
            uint32_t hv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const uint32_t two = (w4[i >> 1] >> (16 * (i & 1))) & 0xFFFFu;
              const uint32_t c_lo = two & 0xFFu, c_hi = two >> 8;
              const float v_lo = (c_lo & 0x80u ? -1.0f : 1.0f) * e4m3_value(c_lo & 0x7Fu) * sigma;
              const float v_hi = (c_hi & 0x80u ? -1.0f : 1.0f) * e4m3_value(c_hi & 0x7Fu) * sigma;
              hv[i] = pack_half2(v_lo, v_hi);
            }
            const int chunk0 = part * 16 + j * 2;
            *reinterpret_cast<uint4*>(smem + L::kv_off + swz(row, chunk0)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
            *reinterpret_cast<uint4*>(smem + L::kv_off + swz(row, chunk0 + 1)) = make_uint4(hv[4], hv[5], hv[6], hv[7]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c)
            *reinterpret_cast<uint4*>(smem + L::kv_off + swz(row, part * 16 + c)) = make_uint4(0, 0, 0, 0);
        }
      } else {
        const int i = e - key_begin;
        const bool ok = row < nk && i < n_top && srow[i] >= 0;
        if (part == 0) kvalid[row] = ok;
        if (ok) {
          const uint8_t* rc = smem + L::raw_off + row * kKvCodeBytes;
          const uint2 sp = *reinterpret_cast<const uint2*>(smem + L::raw_scale_off + row * kKvScaleBytes + part * 8);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 cv = *reinterpret_cast<const uint4*>(rc + (((4 * part + j) ^ (row & 7)) << 4));
            uint4 hv[4];
            dequant16(cv, j < 2 ? (sp.x >> (16 * j)) : (sp.y >> (16 * (j - 2))), hv);
            const int chunk0 = part * 16 + j * 4;   // 8 fp16 per chunk
#pragma unroll
            for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(smem + L::kv_off + swz(row, chunk0 + c)) = hv[c];
          }
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c)
            *reinterpret_cast<uint4*>(smem + L::kv_off + swz(row, part * 16 + c)) = make_uint4(0, 0, 0, 0);
        }
      }
    }
    __syncthreads();   // the chunk's fp16 rows are visible; the staging buffer is free
    if (c0 + kChunk < key_end) issue_chunk(c0 + kChunk);

    // ---- S = Q K^T: this warp's 16 heads x KW keys over all 512 dims ----
    float s[L::NT][4];
#pragma unroll
    for (int j = 0; j < L::NT; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.0f;
    const int key0 = kg * L::KW;
#pragma unroll 4
    for (int ks = 0; ks < kKvDim / 16; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(sbase + L::q_off + swz(ht * 16 + (lane & 15), ks * 2 + (lane >> 4)), a0, a1, a2, a3);
      if constexpr (L::NT == 1) {
        uint32_t b0, b1;
        ldsm_x2(sbase + L::kv_off + swz(key0 + (lane & 7), ks * 2 + ((lane >> 3) & 1)), b0, b1);
        mma_f16(s[0], a0, a1, a2, a3, b0, b1);
      } else {
#pragma unroll
        for (int np = 0; np < L::NT / 2; ++np) {   // pairs of 8-key tiles
          const int mi = lane >> 3;
          uint32_t b0, b1, b2, b3;
          ldsm_x4(sbase + L::kv_off + swz(key0 + np * 16 + (mi >> 1) * 8 + (lane & 7), ks * 2 + (mi & 1)), b0, b1,
                  b2, b3);
          mma_f16(s[2 * np], a0, a1, a2, a3, b0, b1);
          mma_f16(s[2 * np + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }

    // ---- online softmax (log2 domain), maxima and sums combined over the key groups ----
    const float sc0 = qscale[h0], sc1 = qscale[h1];
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int j = 0; j < L::NT; ++j) {
      const int col = key0 + j * 8 + 2 * (lane & 3);
      const bool v0 = col < nk && kvalid[col], v1 = col + 1 < nk && kvalid[col + 1];
      s[j][0] = v0 ? s[j][0] * sc0 : -INFINITY;
      s[j][1] = v1 ? s[j][1] * sc0 : -INFINITY;
      s[j][2] = v0 ? s[j][2] * sc1 : -INFINITY;
      s[j][3] = v1 ? s[j][3] * sc1 : -INFINITY;
      mx0 = fmaxf(mx0, fmaxf(s[j][0], s[j][1]));
      mx1 = fmaxf(mx1, fmaxf(s[j][2], s[j][3]));
    }
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    if ((lane & 3) == 0) {
      red_max[kg * H + h0] = mx0;
      red_max[kg * H + h1] = mx1;
    }
    __syncthreads();   // every key group's row maxima
    // this warp's S rows: the new running max (the same value every warp
    // derives for those rows below) and P
    float mn0 = m_run[0][0], mn1 = m_run[0][1];
#pragma unroll
    for (int t = 1; t < L::HT; ++t)   // select head tile ht without indexing registers by a variable
      if (t == ht) mn0 = m_run[t][0], mn1 = m_run[t][1];
#pragma unroll
    for (int g = 0; g < L::KG; ++g) {
      mn0 = fmaxf(mn0, red_max[g * H + h0]);
      mn1 = fmaxf(mn1, red_max[g * H + h1]);
    }
    const float ref0 = mn0 == -INFINITY ? 0.0f : mn0, ref1 = mn1 == -INFINITY ? 0.0f : mn1;
    float sum0 = 0.0f, sum1 = 0.0f;
#pragma unroll
    for (int j = 0; j < L::NT; ++j) {
      const float p0 = exp2f(s[j][0] - ref0), p1 = exp2f(s[j][1] - ref0);
      const float p2 = exp2f(s[j][2] - ref1), p3 = exp2f(s[j][3] - ref1);
      sum0 += p0 + p1;
      sum1 += p2 + p3;
      const int col = key0 + j * 8 + 2 * (lane & 3);
      const uint32_t within = (col & 7) * 2;
      *reinterpret_cast<uint32_t*>(smem + L::p_off + pswz(h0, col >> 3) + within) = pack_half2(p0, p1);
      *reinterpret_cast<uint32_t*>(smem + L::p_off + pswz(h1, col >> 3) + within) = pack_half2(p2, p3);
    }
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
      sum0 += __shfl_xor_sync(0xffffffffu, sum0, o);
      sum1 += __shfl_xor_sync(0xffffffffu, sum1, o);
    }
    if ((lane & 3) == 0) {
      red_sum[kg * H + h0] = sum0;
      red_sum[kg * H + h1] = sum1;
    }
    __syncthreads();   // P and every key group's row sums
    // every head tile's rows: running max, sum and the rescaling of O
#pragma unroll
    for (int t = 0; t < L::HT; ++t) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int row = t * 16 + r0 + 8 * hf;
        float mn = m_run[t][hf], tot = 0.0f;
#pragma unroll
        for (int g = 0; g < L::KG; ++g) {
          mn = fmaxf(mn, red_max[g * H + row]);
          tot += red_sum[g * H + row];
        }
        const float ref = mn == -INFINITY ? 0.0f : mn;
        const float corr = exp2f(m_run[t][hf] - ref);
        l_run[t][hf] = l_run[t][hf] * corr + tot;
        m_run[t][hf] = mn;
#pragma unroll
        for (int i = 0; i < kPVDims / 8; ++i) {
          o_acc[t][i][2 * hf] *= corr;
          o_acc[t][i][2 * hf + 1] *= corr;
        }
      }
    }

    // ---- O += P V: every head x this warp's 64 dims over the chunk's 64 keys ----
#pragma unroll
    for (int kk = 0; kk < kChunk / 16; ++kk) {
      uint32_t a[L::HT][4];
#pragma unroll
      for (int t = 0; t < L::HT; ++t)
        ldsm_x4(sbase + L::p_off + pswz(t * 16 + (lane & 15), kk * 2 + (lane >> 4)), a[t][0], a[t][1], a[t][2],
                a[t][3]);
#pragma unroll
      for (int np = 0; np < kPVDims / 16; ++np) {
        const int mi = lane >> 3;
        const int dchunk = (warp * kPVDims) / 8 + np * 2 + (mi >> 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sbase + L::kv_off + swz(kk * 16 + (mi & 1) * 8 + (lane & 7), dchunk), b0, b1, b2, b3);
#pragma unroll
        for (int t = 0; t < L::HT; ++t) {
          mma_f16(o_acc[t][2 * np], a[t][0], a[t][1], a[t][2], a[t][3], b0, b1);
          mma_f16(o_acc[t][2 * np + 1], a[t][0], a[t][1], a[t][2], a[t][3], b2, b3);
        }
      }
    }
  }

  // ---- partial O slices, maxima and sums to their owners ----
  // Output dims [kODims*r, kODims*(r+1)) belong to CTA r.  With a workspace
  // (xchg) every CTA writes its partial O as [owner][H][kODims] fp32 plus its
  // (m, l) into its own region of global memory (L2) and the owner reads the
  // four slices back after one cluster barrier; without one, the slices go
  // straight into the owner's shared memory (distributed shared memory,
  // recv[src][h][kODims] with 16-byte granules XOR-swizzled by the head, and
  // ml_sh[src]) between two cluster barriers.  Every CTA of the cluster
  // passes the same barriers.
  constexpr long long kRegion = static_cast<long long>(H) * kKvDim + 2 * H;   // floats per CTA in xchg
  float* recv = reinterpret_cast<float*>(smem);
  const float* src_slice[CL];      // where the owner reads source r's slice of its dims
  const float* src_ml[CL];         // ... and source r's (m[H], l[H])
  int slice_swz;                          // 1: swizzled shared-memory slices
  const int owner = (warp * kPVDims) / kODims, cd0 = (warp * kPVDims) % kODims;   // this warp's dims
  if (xchg != nullptr) {
    float* mine = xchg + static_cast<long long>(blockIdx.x) * kRegion;
    float* dst = mine + owner * H * kODims;
#pragma unroll
    for (int t = 0; t < L::HT; ++t)
#pragma unroll
      for (int i = 0; i < kPVDims / 8; ++i) {
        const int cd = cd0 + i * 8 + 2 * (lane & 3), row = t * 16 + r0;
        *reinterpret_cast<float2*>(dst + row * kODims + cd) = make_float2(o_acc[t][i][0], o_acc[t][i][1]);
        *reinterpret_cast<float2*>(dst + (row + 8) * kODims + cd) = make_float2(o_acc[t][i][2], o_acc[t][i][3]);
      }
    if (warp == 0 && (lane & 3) == 0) {
#pragma unroll
      for (int t = 0; t < L::HT; ++t)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          mine[H * kKvDim + t * 16 + r0 + 8 * hf] = m_run[t][hf];
          mine[H * kKvDim + H + t * 16 + r0 + 8 * hf] = l_run[t][hf];
        }
    }
    cluster.sync();   // every CTA's partials are in the workspace (cluster-scope release / acquire)
    const float* first = xchg + static_cast<long long>(blockIdx.x - rank) * kRegion;
#pragma unroll
    for (int r = 0; r < CL; ++r) {
      src_slice[r] = first + r * kRegion + rank * H * kODims;
      src_ml[r] = first + r * kRegion + H * kKvDim;
    }
    slice_swz = 0;
  } else {
    cluster.sync();   // every CTA is done reading its Q / KV region, which receives the partials
    float* dst = cluster.map_shared_rank(recv, owner) + rank * H * kODims;
#pragma unroll
    for (int t = 0; t < L::HT; ++t)
#pragma unroll
      for (int i = 0; i < kPVDims / 8; ++i) {
        const int cd = cd0 + i * 8 + 2 * (lane & 3), row = t * 16 + r0;
        *reinterpret_cast<float2*>(dst + row * kODims + attn_swz(row, cd)) =
            make_float2(o_acc[t][i][0], o_acc[t][i][1]);
        *reinterpret_cast<float2*>(dst + (row + 8) * kODims + attn_swz(row + 8, cd)) =
            make_float2(o_acc[t][i][2], o_acc[t][i][3]);
      }
    if (warp == 0 && (lane & 3) == 0) {
#pragma unroll
      for (int o = 0; o < CL; ++o) {
        float* ml = cluster.map_shared_rank(ml_sh, o) + rank * 2 * H;
#pragma unroll
        for (int t = 0; t < L::HT; ++t)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            ml[t * 16 + r0 + 8 * hf] = m_run[t][hf];
            ml[H + t * 16 + r0 + 8 * hf] = l_run[t][hf];
          }
      }
    }
    cluster.sync();   // every partial has landed; no CTA touches another's memory after this
#pragma unroll
    for (int r = 0; r < CL; ++r) {
      src_slice[r] = recv + r * H * kODims;
      src_ml[r] = ml_sh + r * 2 * H;
    }
    slice_swz = 1;
  }

  // merge factors per (source rank, head): exp2(m_r - M) / L
  for (int h = tid; h < H; h += kAThreads) {
    float mr[CL], lr[CL];
    float M = -INFINITY;
#pragma unroll
    for (int r = 0; r < CL; ++r) {
      mr[r] = src_ml[r][h];
      lr[r] = src_ml[r][H + h];
      M = fmaxf(M, mr[r]);
    }
    float Lsum = 0.0f;
#pragma unroll
    for (int r = 0; r < CL; ++r) {
      mr[r] = (M == -INFINITY || mr[r] == -INFINITY) ? 0.0f : exp2f(mr[r] - M);
      Lsum += lr[r] * mr[r];
    }
    const float inv = Lsum > 0.0f ? 1.0f / Lsum : 0.0f;
#pragma unroll
    for (int r = 0; r < CL; ++r) fac[r * H + h] = mr[r] * inv;
  }
  __syncthreads();
  // this CTA writes dims [kODims*rank, kODims*(rank+1)) of every head, 4 dims
  // per item; every item's partial slices are loaded before any is used
  constexpr int kItems = H * (kODims / 4) / kAThreads;
  static_assert(H * (kODims / 4) % kAThreads == 0, "whole items per thread");
  float4 part[kItems][CL];
#pragma unroll
  for (int it = 0; it < kItems; ++it) {
    const int item = it * kAThreads + tid;
    const int h = item / (kODims / 4), d4 = (item % (kODims / 4)) * 4;
    const int c = slice_swz ? attn_swz(h, d4) : d4;
#pragma unroll
    for (int r = 0; r < CL; ++r) part[it][r] = *reinterpret_cast<const float4*>(src_slice[r] + h * kODims + c);
  }
#pragma unroll
  for (int it = 0; it < kItems; ++it) {
    const int item = it * kAThreads + tid;
    const int h = item / (kODims / 4), d4 = (item % (kODims / 4)) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < CL; ++r) {
      const float4 v = part[it][r];
      const float f = fac[r * H + h];
      acc.x += v.x * f; acc.y += v.y * f; acc.z += v.z * f; acc.w += v.w * f;
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&lo);
    pk.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(out + (static_cast<long long>(qi) * H + h) * kKvDim + rank * kODims + d4) = pk;
  }
}

template <int H, int CL>
cudaError_t launch_hc(const csa2_cache& cache, int n_layers, int n_queries, const int32_t* q_req, int k,
                      const AttnLayers& io, float scale, const SwaArgs& swa, float* xchg, cudaStream_t stream) {
  static ContextMemo attrs;
  const size_t smem = AttnLayout<H, CL>::total;
  const cudaError_t e = attrs.once([&] {
    return cudaFuncSetAttribute(sparse_attn_kernel<H, CL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(smem));
  });
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_layers * n_queries * CL);
  cfg.blockDim = dim3(kAThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // the kernel calls pdl_wait() before reading the Top-k
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, sparse_attn_kernel<H, CL>, cache, n_queries, q_req, k, io, scale, swa, xchg);
}

// Key splits per query, from the number of queries alone (so that one query's
// result does not depend on how many layers a launch covers): 4 while a
// decode group's six layers of all queries fit one wave of the GPU's SMs at
// 4 CTAs per query, then 2, then 1 (more queries fill the GPU by themselves,
// and one CTA per query merges no partial outputs).  16 heads keep 4: their
// CTAs fit two per SM, which the larger entry table of fewer splits would
// prevent.
int key_splits(int n_queries, int H) {
  if (H == 16) return 4;
  return n_queries <= 6 ? 4 : (n_queries <= 12 ? 2 : 1);
}

template <int H>
cudaError_t launch_h(const csa2_cache& cache, int n_layers, int n_queries, const int32_t* q_req, int k,
                     const AttnLayers& io, float scale, const SwaArgs& swa, float* xchg, cudaStream_t stream) {
  if constexpr (H == 16) {
    return launch_hc<H, 4>(cache, n_layers, n_queries, q_req, k, io, scale, swa, xchg, stream);
  } else {
    switch (key_splits(n_queries, H)) {
      case 4: return launch_hc<H, 4>(cache, n_layers, n_queries, q_req, k, io, scale, swa, xchg, stream);
      case 2: return launch_hc<H, 2>(cache, n_layers, n_queries, q_req, k, io, scale, swa, xchg, stream);
      default: return launch_hc<H, 1>(cache, n_layers, n_queries, q_req, k, io, scale, swa, xchg, stream);
    }
  }
}

}  // namespace

size_t attn_workspace_bytes(long long n_layers, long long n_queries, int H) {
  return static_cast<size_t>(n_layers * n_queries * kAMaxCluster) * (static_cast<size_t>(H) * kKvDim + 2 * H) * 4;
}

cudaError_t launch_sparse_attn(const csa2_cache& cache, int n_layers, int n_queries, const int32_t* q_req,
                               const int32_t* const* topk, int k, const uint16_t* const* q, int H, float scale,
                               uint16_t* const* out, cudaStream_t stream, const uint8_t* swa_codes,
                               const uint8_t* swa_exp, const int32_t* q_pos, int window, void* xchg) {
  AttnLayers io = {};
  for (int l = 0; l < n_layers; ++l) {
    io.topk[l] = topk[l];
    io.q[l] = reinterpret_cast<const __nv_bfloat16*>(q[l]);
    io.out[l] = reinterpret_cast<__nv_bfloat16*>(out[l]);
  }
  const SwaArgs swa = {swa_codes, swa_exp, q_pos, window};
  float* xf = static_cast<float*>(xchg);
  switch (H) {
    case 16: return launch_h<16>(cache, n_layers, n_queries, q_req, k, io, scale, swa, xf, stream);
    case 32: return launch_h<32>(cache, n_layers, n_queries, q_req, k, io, scale, swa, xf, stream);
    case 64: return launch_h<64>(cache, n_layers, n_queries, q_req, k, io, scale, swa, xf, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace csa2
