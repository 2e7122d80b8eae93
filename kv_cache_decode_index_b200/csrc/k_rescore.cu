// Top-k of every Full and Reindex layer of a layer group over the pool, in two
// launches for all layers together [4sapi blog, section 四: Reindex layers
// re-score only the pool's 2048 x 8 candidates with their own indexer query;
// readance summary, section 4.2: layer modes; alphalab analysis, section 2].
//
// pool_score_kernel: every SM gathers pool blocks (1 KB TMA boxes of 8
// indexer-K rows) ONCE and scores them for all L layers in one tcgen05 MMA
// (M = 128 positions, N = 32 heads x L layers, K = 128, FP8), with the
// epilogue of the Full scan per layer (bit-identical scores for the Full
// layer).  Each layer's order keys go to a workspace, and each valid key adds
// one count to a 4096-bin histogram of its leading 12 bits per (request,
// layer).
//
// layer_select_kernel: one CTA of 1024 threads per (request, layer) holds the
// request's pool keys of that layer in registers, reads (and zeroes) its
// histogram to find the threshold's leading 12 bits at once, finishes the
// exact Top-k with 10-bit radix passes over the few keys in that bin, and
// writes the positions ascending (ties to the lower position, -1 padding).
#include "block_topk.cuh"
#include "fp4.cuh"
#include "index_common.cuh"
#include "launch.h"

namespace csa2 {

namespace {

constexpr int kSThreads = 192;   // warp 0: TMA producer, warp 1: MMA, warps 2..5: epilogue
constexpr int kSStages = 4;
constexpr int kSMaxTiles = 8;    // tiles (16 pool blocks each) per CTA
constexpr int kSBlocksPerTile = kTile / kBlock;   // 16
constexpr uint32_t kSTmemCols = 256;
constexpr int kSMaxAcc = 4;
constexpr int kRsHistBins = CSA2_RESCORE_HIST_BINS;   // 4096: leading 12 key bits
constexpr int kRsHistBits = 12;

struct ScoreLayers {
  const float* q[CSA2_MAX_SCORE_LAYERS];
  const float* w[CSA2_MAX_SCORE_LAYERS];
};
struct TopkLayers {
  int32_t* topk[CSA2_MAX_SCORE_LAYERS];
};

constexpr int kMaxFp4ScoreLayers = 4;
constexpr int kMaxPoolSlots = 4096;     // pool blocks (the host accepts up to 4096)   // N = 32 x layers <= 128: one block of query scales

// Shared memory of the scoring kernel for the FP8 indexer (kFp4 = false: 128
// code bytes and an exponent byte per row) or the FP4 one (64 code bytes and
// the block scales of each row, gathered into the tensor-core order per tile).
template <bool kFp4>
struct __align__(1024) ScoreSmemT {
  static constexpr int kRowBytes = kFp4 ? CSA2_IK4_CODE_BYTES : kIndexDim;
  static constexpr int kLayers = kFp4 ? kMaxFp4ScoreLayers : CSA2_MAX_SCORE_LAYERS;
  uint8_t tiles[kSStages][kTile * kRowBytes];
  uint8_t qtile[kLayers][kIndexHeads * kRowBytes];          // layer l: B-operand rows 32l .. 32l+31
  uint8_t qscale[kFp4 ? 1024 : 16];                         // FP4: the query heads' block scales
  uint8_t tscale[kFp4 ? kSMaxTiles : 1][kFp4 ? 1024 : 16];  // FP4: each tile's block scales
  float ws[kLayers][kIndexHeads];                           // w_h (FP4) or w_h * sigma^q_h (FP8) per layer
  int blk_row[kSMaxTiles * kSBlocksPerTile];
  int blk_id[kSMaxTiles * kSBlocksPerTile];
  uint64_t full[kSStages];
  uint64_t empty[kSStages];
  uint64_t acc_full[kSMaxAcc];
  uint64_t acc_empty[kSMaxAcc];
  uint64_t q_full;
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort_flag;
};

// keys: uint32 [batch][L][P * 8]; hist: uint32 [batch][L][4096].  ik4_scales:
// the FP4 keys' block scales (kFp4 only); blk_map: 8-row boxes of the index
// codes (FP8: 128-byte rows, 128-byte swizzle; FP4: 64-byte rows, 64-byte
// swizzle).
template <bool kFp4>
__global__ void __launch_bounds__(kSThreads, 2)
    pool_score_kernel(const csa2_cache cache, const uint8_t* __restrict__ ik4_scales, const int32_t* __restrict__ pool,
                      int P, int L, int tiles_per_cta, const __grid_constant__ ScoreLayers io,
                      uint32_t* __restrict__ keys, uint32_t* __restrict__ hist,
                      const __grid_constant__ CUtensorMap blk_map, uint64_t wait_ns) {
  using Smem = ScoreSmemT<kFp4>;
  constexpr int kBlkBytes = kBlock * Smem::kRowBytes;
  constexpr int kTileB = kTile * Smem::kRowBytes;
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tiles_per_req = (P + kSBlocksPerTile - 1) / kSBlocksPerTile;
  const int ctas_per_req = (tiles_per_req + tiles_per_cta - 1) / tiles_per_cta;
  const int b = blockIdx.x / ctas_per_req, c = blockIdx.x % ctas_per_req;
  const long long capacity = static_cast<long long>(cache.max_pages_per_req) * cache.page_size;
  const int slot0 = c * tiles_per_cta * kSBlocksPerTile;                 // first pool slot of this CTA
  const int nblk = max(0, min(tiles_per_cta * kSBlocksPerTile, P - slot0));   // pool slots of this CTA
  const int n_tiles = (nblk + kSBlocksPerTile - 1) / kSBlocksPerTile;
  const int ncols = kIndexHeads * L;                                     // accumulator columns per tile
  // accumulators start at multiples of the next power of two >= ncols; with
  // FP4, each accumulator also has 8 columns of its tile's block scales and the
  // query scales take 8 more
  // (in the columns an accumulator slot leaves unused when there are 16 of
  // them: 3 layers, N = 96 in 128-column slots, keep two slots)
  const int acc_stride = ncols <= 32 ? 32 : (ncols <= 64 ? 64 : (ncols <= 128 ? 128 : 256));
  const bool sf_inside = kFp4 && acc_stride - ncols >= 16;
  const int n_acc = !kFp4 || sf_inside ? min(kSMaxAcc, static_cast<int>(kSTmemCols) / acc_stride)
                                       : max(1, min(kSMaxAcc, static_cast<int>(kSTmemCols - 8) / (acc_stride + 8)));
  // FP4: tile scales of accumulator a at sfa_col + sfa_step * a, query scales at sfb_col
  const uint32_t sfa_col = static_cast<uint32_t>(sf_inside ? ncols : n_acc * acc_stride);
  const uint32_t sfa_step = static_cast<uint32_t>(sf_inside ? acc_stride : 8);
  const uint32_t sfb_col = sf_inside ? static_cast<uint32_t>(ncols + 8) : sfa_col + 8u * n_acc;
  const long long key_stride = static_cast<long long>(P) * kBlock;

  // ---- independent of the preceding launch (it selects the pool): the
  // barriers, tensor memory and the layers' queries, overlapping its tail ----
  if (tid == 0) {
    for (int s = 0; s < kSStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    for (int a = 0; a < kSMaxAcc; ++a) {
      mbar_init(&S.acc_full[a], 1);
      mbar_init(&S.acc_empty[a], 4);
    }
    mbar_init(&S.q_full, 4);
    mbar_init(&S.drain, 1);
    S.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, kSTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) tma_prefetch_map(&blk_map);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  if (warp >= 2) {   // the epilogue warps: every layer's query codes and head weights
    const int ew = warp - 2;
    for (int l = 0; l < L; ++l) {
      const float* ql = io.q[l] + static_cast<long long>(b) * kIndexHeads * kIndexDim;
      const float* wl = io.w[l] + static_cast<long long>(b) * kIndexHeads;
      if constexpr (kFp4) {
        prepare_query_fp4(ql, S.qtile[0], S.qscale, kIndexHeads * l, ew, lane);
        if (lane < 8) S.ws[l][ew * 8 + lane] = wl[ew * 8 + lane];
      } else {
        prepare_query_part(ql, wl, S.qtile[l], S.ws[l], ew, lane);
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.q_full);
  }

  pdl_wait();                 // the pool of the preceding launch is complete
  pdl_launch_dependents();
  const int n_raw = checked_ctx_len(cache, b, capacity, kKReindex, c == 0 && tid == 0);
  if (n_raw < 0) {            // corrupt length: every key of this CTA's slots is "no candidate"
    for (int l = 0; l < L; ++l)
      for (int i = tid; i < nblk * kBlock; i += kSThreads)
        keys[(static_cast<long long>(b) * L + l) * key_stride + slot0 * kBlock + i] = 0u;
  }
  const int n = max(n_raw, 0);
  const int n_work = n_raw < 0 ? 0 : n_tiles;   // tiles this CTA scores

  // ---- this CTA's pool blocks: block id -> page -> row (the exponent bytes
  // are read by the epilogue while the codes are gathered) ----
  for (int i = tid; i < (n_raw < 0 ? 0 : nblk); i += kSThreads) {
    const int j = pool[static_cast<long long>(b) * P + slot0 + i];
    int row = -1;
    if (j >= 0 && static_cast<long long>(j) * kBlock < n) {
      const int t = j * kBlock;
      const int page = cache.page_table[static_cast<long long>(b) * cache.max_pages_per_req + t / cache.page_size];
      if (page >= 0 && page < cache.num_pages) {
        row = page * cache.page_size + t % cache.page_size;
      } else {
        report_error(cache.err_word, CSA2_ERR_DEVICE_BOUNDS, kKReindex, b, t);
      }
    } else if (j >= 0 || j < -1) {
      report_error(cache.err_word, CSA2_ERR_DEVICE_BOUNDS, kKReindex, b, j);
    }
    S.blk_row[i] = row;
    S.blk_id[i] = row >= 0 ? j : -1;
  }
  if constexpr (kFp4) {
    // block scales of the CTA's blocks, moved into each tile's tensor-core
    // order: tile row m = 8 * (block % 16) + r takes the scales of the
    // block's row r (4 bytes per half of the row's 8 scales)
    __syncthreads();
    // all of a thread's loads are issued before any is used
    constexpr int kWords = (kSMaxTiles * kSBlocksPerTile * kBlock * 2 + kSThreads - 1) / kSThreads;
    const int n_words = n_work * kSBlocksPerTile * kBlock * 2;   // none after a corrupt length
    uint32_t v[kWords];
#pragma unroll
    for (int u = 0; u < kWords; ++u) {
      const int x = tid + u * kSThreads;
      const int kh = x & 1, r = (x >> 1) & 7, i = x >> 4;
      const int row = (x < n_words && i < nblk) ? S.blk_row[i] : -1;
      v[u] = row >= 0 ? *reinterpret_cast<const uint32_t*>(ik4_scales + static_cast<long long>(row / kTile) * 1024 +
                                                           block_scale_offset(row % kTile + r, 4 * kh))
                      : 0u;
    }
#pragma unroll
    for (int u = 0; u < kWords; ++u) {
      const int x = tid + u * kSThreads;
      if (x >= n_words) continue;
      const int kh = x & 1, r = (x >> 1) & 7, i = x >> 4;
      const int t = i / kSBlocksPerTile, m = kBlock * (i % kSBlocksPerTile) + r;
      *reinterpret_cast<uint32_t*>(S.tscale[t] + block_scale_offset(m, 4 * kh)) = v[u];
    }
    fence_proxy_async_smem();
  }
  __syncthreads();   // the blocks' rows and ids; every layer's head weights

  if (n_work > 0) {
    if (warp == 0) {
      // ---- producer: lane l < 16 gathers block l of each tile ----
      const uint64_t policy = l2_policy_evict_normal();
      int issued = 0;
      for (int t = 0; t < n_tiles; ++t) {
        const int s = t % kSStages;
        const uint32_t ph = (t / kSStages) & 1;
        if (!mbar_wait_warp(&S.empty[s], ph ^ 1, wait_ns) || warp_flag(&S.abort_flag)) {
          if (lane == 0) {
            report_error(cache.err_word, CSA2_ERR_TIMEOUT, kKReindex, b, t);
            S.abort_flag = 1;
          }
          break;
        }
        const int e = t * kSBlocksPerTile + lane;
        const int row = (lane < kSBlocksPerTile && e < nblk) ? S.blk_row[e] : -1;
        const uint32_t bytes = __popc(__ballot_sync(0xffffffffu, row >= 0)) * kBlkBytes;
        if (lane == 0) mbar_arrive_expect_tx(&S.full[s], bytes);   // before any of the tile's copies
        __syncwarp();
        if (row >= 0) tma_load_2d(S.tiles[s] + lane * kBlkBytes, &blk_map, &S.full[s], 0, row, policy);
        ++issued;
      }
      if (lane == 0)
        for (int i = issued > kSStages ? issued - kSStages : 0; i < issued; ++i)
          (void)mbar_wait(&S.full[i % kSStages], (i / kSStages) & 1, kWaitLimitNs / 2);
    } else if (warp == 1) {
      if (lane == 0) {   // ---- MMA issuer: one N = 32L MMA chain per tile ----
        const uint32_t idesc = kFp4 ? idesc_mxf4nvf4(kTile, ncols) : idesc_e4m3_f32(kTile, ncols);
        const uint64_t bdesc = kFp4 ? sw64_kmajor_desc(smem_u32(S.qtile[0])) : sw128_kmajor_desc(smem_u32(S.qtile[0]));
        bool ok = mbar_wait(&S.q_full, 0, wait_ns);
        if constexpr (kFp4) {
          if (ok) {
            tc_fence_after();
            for (int kh = 0; kh < 2; ++kh) tmem_cp_scales(tmem + sfb_col + 4 * kh, smem_u32(S.qscale + 512 * kh));
          }
        }
        for (int t = 0; ok && t < n_tiles; ++t) {
          const int s = t % kSStages;
          const uint32_t ph = (t / kSStages) & 1;
          const int a = t % n_acc;
          const uint32_t aph = (t / n_acc) & 1;
          if (!mbar_wait(&S.acc_empty[a], aph ^ 1, wait_ns) || !mbar_wait(&S.full[s], ph, wait_ns)) {
            ok = false;
            break;
          }
          if (S.abort_flag) break;
          tc_fence_after();
          if constexpr (kFp4) {
            const uint32_t sfa = tmem + sfa_col + sfa_step * a;
            for (int kh = 0; kh < 2; ++kh) tmem_cp_scales(sfa + 4 * kh, smem_u32(S.tscale[t] + 512 * kh));
            const uint64_t adesc = sw64_kmajor_desc(smem_u32(S.tiles[s]));
#pragma unroll
            for (int kh = 0; kh < 2; ++kh)
              umma_mxf4nvf4(tmem + a * acc_stride, adesc + 2 * kh, bdesc + 2 * kh, idesc, sfa + 4 * kh,
                            tmem + sfb_col + 4 * kh, kh > 0 ? 1u : 0u);
          } else {
            const uint64_t adesc = sw128_kmajor_desc(smem_u32(S.tiles[s]));
#pragma unroll
            for (int k = 0; k < kIndexDim / 32; ++k)
              umma_f8f6f4(tmem + a * acc_stride, adesc + 2 * k, bdesc + 2 * k, idesc, k > 0 ? 1u : 0u);
          }
          umma_commit(&S.empty[s]);
          umma_commit(&S.acc_full[a]);
        }
        if (!ok) {
          report_error(cache.err_word, CSA2_ERR_TIMEOUT, kKReindex, b, -1);
          S.abort_flag = 1;
        }
        umma_commit(&S.drain);
        (void)mbar_wait(&S.drain, 0, kWaitLimitNs);
      }
    } else {
      // ---- epilogue (warps 2..5): one position per thread, every layer ----
      const int quarter = warp & 3, m = quarter * 32 + lane;
      for (int t = 0; t < n_tiles; ++t) {
        const int a = t % n_acc;
        const uint32_t aph = (t / n_acc) & 1;
        const int e = t * kSBlocksPerTile + m / kBlock;
        const int o = m % kBlock;
        const bool in_range = e < nblk;
        const bool valid = in_range && S.blk_row[e] >= 0 && S.blk_id[e] * kBlock + o < n;
        // issued before the wait for the accumulator: its latency overlaps the gather and the MMA
        const uint32_t e_byte = (!kFp4 && valid) ? static_cast<uint32_t>(cache.ik_exp[S.blk_row[e] + o]) : 127u;
        if (!mbar_wait_warp(&S.acc_full[a], aph, wait_ns)) {
          if (lane == 0) {
            report_error(cache.err_word, CSA2_ERR_TIMEOUT, kKReindex, b, t);
            S.abort_flag = 1;
          }
          break;
        }
        tc_fence_after();
        for (int l = 0; l < L; ++l) {
          uint32_t acc[32];
          tmem_ld_32x32b_x32(tmem + a * acc_stride + l * kIndexHeads + (static_cast<uint32_t>(quarter * 32) << 16), acc);
          tmem_ld_wait();
          float ws[32];
#pragma unroll
          for (int h = 0; h < 32; ++h) ws[h] = S.ws[l][h];
          float sc;
          if constexpr (kFp4) {
            sc = 0.0f;
#pragma unroll
            for (int h = 0; h < 32; ++h) sc = fmaf(ws[h], fmaxf(__uint_as_float(acc[h]), 0.0f), sc);
          } else {
            sc = score_from_acc(acc, ws, e_byte);
          }
          const uint32_t key = valid ? order_key(sc) : 0u;
          const long long bl = static_cast<long long>(b) * L + l;
          if (in_range) keys[bl * key_stride + static_cast<long long>(slot0 + e) * kBlock + o] = key;
          // one count per distinct bin of the warp's keys: the keys crowd into few bins
          const uint32_t vm = __ballot_sync(0xffffffffu, valid);
          if (valid) {
            const uint32_t bin = key >> (32 - kRsHistBits);
            const uint32_t peers = __match_any_sync(vm, bin);
            if ((peers & ((1u << lane) - 1u)) == 0u) atomicAdd(&hist[bl * kRsHistBins + bin], __popc(peers));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.acc_empty[a]);
        if (warp_flag(&S.abort_flag)) break;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kSTmemCols);
  }
}

// One CTA per (request, layer): exact Top-k of the layer's pool keys.
template <int ITEMS>
__global__ void __launch_bounds__(kBlockSelectThreads, 1)
    layer_select_kernel(const int32_t* __restrict__ pool, int P, int L, int K, const uint32_t* __restrict__ keys,
                        uint32_t* __restrict__ hist, const __grid_constant__ TopkLayers out) {
  __shared__ BlockSelectSmem S;
  __shared__ int32_t pool_ids[kMaxPoolSlots];
  const int tid = threadIdx.x;
  const int b = blockIdx.x / L, l = blockIdx.x % L;
  const long long bl = static_cast<long long>(b) * L + l;
  const int n_keys = P * kBlock;
  // The request's pool (block ids of the key groups), used by the emits
  // after the select's barriers.  The scoring launch lets this one start only
  // after its own wait for the pool's launch to complete, so the pool is read
  // before this launch's wait.
  for (int i = tid; i < P; i += kBlockSelectThreads) pool_ids[i] = pool[static_cast<long long>(b) * P + i];
  pdl_wait();                 // the keys and histograms of the scoring launch are complete
  pdl_launch_dependents();
  // keys [tid*ITEMS, (tid+1)*ITEMS) in registers (groups of 4: n_keys is a multiple of 8)
  uint32_t k[ITEMS];
  const uint32_t* src = keys + bl * n_keys;
#pragma unroll
  for (int i = 0; i < ITEMS; i += 4) {
    const int idx = tid * ITEMS + i;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (idx < n_keys) v = *reinterpret_cast<const uint4*>(src + idx);
    k[i] = v.x;
    k[i + 1] = v.y;
    k[i + 2] = v.z;
    k[i + 3] = v.w;
  }
  // this thread's 4 histogram bins, highest first (thread order = descending
  // bins), read and zeroed for the next call
  uint32_t* hb = hist + bl * kRsHistBins + 4 * (kBlockSelectThreads - 1 - tid);
  const uint4 hv = *reinterpret_cast<const uint4*>(hb);
  *reinterpret_cast<uint4*>(hb) = make_uint4(0u, 0u, 0u, 0u);
  const uint32_t c[4] = {hv.w, hv.z, hv.y, hv.x};
  int valid = 0;
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) valid += k[i] != 0u ? 1 : 0;
  const bool ok = hist_head_start<kBlockSelectThreads, 4, true>(c, 4 * (kBlockSelectThreads - 1 - tid) + 3,
                                                                kRsHistBits, valid, K, S.warp_tmp, &S.start);
  int32_t* dst = out.topk[l] + static_cast<long long>(b) * K;
  block_topk<ITEMS>(
      k, K, S, [&](int i, int r) { dst[r] = pool_ids[i / kBlock] * kBlock + (i % kBlock); },
      [&](int r) { dst[r] = -1; }, ok ? &S.start : nullptr);
}

}  // namespace

size_t rescore_workspace_bytes(long long batch, int n_layers, int pool_blocks) {
  if (batch <= 0 || n_layers <= 0 || pool_blocks <= 0) return 0;
  return static_cast<size_t>(batch) * n_layers *
         (static_cast<size_t>(pool_blocks) * kBlock + kRsHistBins) * sizeof(uint32_t);
}

cudaError_t launch_rescore_layers(const csa2_cache& cache, const uint8_t* ik4_scales, int n_layers,
                                  const int32_t* pool, int pool_blocks, const float* const* q, const float* const* w,
                                  int k, int32_t* const* topk, void* workspace, const CUtensorMap& blk_map,
                                  int num_sms, uint64_t wait_ns, cudaStream_t stream) {
  const bool fp4 = ik4_scales != nullptr;
  static ContextMemo attrs8, attrs4;
  const size_t smem = (fp4 ? sizeof(ScoreSmemT<true>) : sizeof(ScoreSmemT<false>)) + 1024;
  cudaError_t e = fp4 ? attrs4.once([&] {
    return cudaFuncSetAttribute(pool_score_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(smem));
  })
                      : attrs8.once([&] {
                          return cudaFuncSetAttribute(pool_score_kernel<false>,
                                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                      static_cast<int>(smem));
                        });
  if (e != cudaSuccess) return e;
  ScoreLayers io = {};
  TopkLayers out = {};
  for (int l = 0; l < n_layers; ++l) {
    io.q[l] = q[l];
    io.w[l] = w[l];
    out.topk[l] = topk[l];
  }
  uint32_t* keys = static_cast<uint32_t*>(workspace);
  uint32_t* hist = keys + static_cast<size_t>(cache.batch) * n_layers * pool_blocks * kBlock;
  // tiles per CTA: enough CTAs for two per SM, at most kSMaxTiles tiles each
  const int tiles_per_req = (pool_blocks + kSBlocksPerTile - 1) / kSBlocksPerTile;
  const long long total_tiles = static_cast<long long>(cache.batch) * tiles_per_req;
  int tpc = static_cast<int>((total_tiles + 2LL * num_sms - 1) / (2LL * num_sms));
  tpc = max(1, min(kSMaxTiles, tpc));
  const int ctas_per_req = (tiles_per_req + tpc - 1) / tpc;

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.stream = stream;
  cfg.gridDim = dim3(cache.batch * ctas_per_req);
  cfg.blockDim = dim3(kSThreads);
  cfg.dynamicSmemBytes = smem;
  if (fp4)
    e = cudaLaunchKernelEx(&cfg, pool_score_kernel<true>, cache, ik4_scales, pool, pool_blocks, n_layers, tpc, io, keys,
                           hist, blk_map, wait_ns);
  else
    e = cudaLaunchKernelEx(&cfg, pool_score_kernel<false>, cache, ik4_scales, pool, pool_blocks, n_layers, tpc, io,
                           keys, hist, blk_map, wait_ns);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3(cache.batch * n_layers);
  cfg.blockDim = dim3(kBlockSelectThreads);
  cfg.dynamicSmemBytes = 0;
  if (pool_blocks * kBlock <= kBlockSelectThreads * 16)
    return cudaLaunchKernelEx(&cfg, layer_select_kernel<16>, pool, pool_blocks, n_layers, k,
                              static_cast<const uint32_t*>(keys), hist, out);
  return cudaLaunchKernelEx(&cfg, layer_select_kernel<32>, pool, pool_blocks, n_layers, k,
                            static_cast<const uint32_t*>(keys), hist, out);
}

}  // namespace csa2
