// Selection kernels of the Hierarchical Sparse Indexer:
//   * pool_select: the pool_blocks blocks with the largest block max, one
//     cluster per request [4sapi blog, section 四; animattoys article, section
//     層與層之間拼車: 2048 blocks x 8 positions];
//   * reindex: Top-k of one layer among the candidates (the pool's positions,
//     or every visible position without a pool).  Reindex re-scores them with
//     the layer's own query on tcgen05 (same tile shape and epilogue as the
//     Full scan, so identical fp32 scores); Full either reads its stored scores
//     or recomputes them the same way [readance summary, section 4.2: modes];
//   * copy_topk: Reuse mode, the previous layer's indices.
// Ties go to the lower block id / position; outputs are ascending, -1 padded.
#include "block_topk.cuh"
#include "cluster_topk.cuh"
#include "index_common.cuh"
#include "launch.h"

namespace csa2 {

namespace {

// ------------------------------------------------------------------ pool ----
constexpr int kPoolThreads = 512;
constexpr int kPoolKeysPerCta = 16384;

struct PoolSmem {
  uint32_t keys[kPoolKeysPerCta];
  SelectSmem sel;
  SelectStart start;
};

// With `hist` (the scan's per-request histogram of the leading 11 bits of the
// block-max order keys), every CTA of the cluster reads it, finds the bin that
// holds the pool's threshold and starts the radix select below those 11 bits;
// the CTAs then zero their slices of it for the next scan.  A histogram that
// does not hold exactly one count per block is ignored (select from scratch).
__global__ void __launch_bounds__(kPoolThreads, 1)
    pool_select_kernel(const csa2_cache cache, const float* __restrict__ blockmax, uint32_t* __restrict__ hist, int P,
                       int32_t* __restrict__ pool) {
  extern __shared__ uint8_t smem_raw[];
  PoolSmem& S = *reinterpret_cast<PoolSmem*>(smem_raw);
  pdl_wait();                 // the block maxima of the scan are complete
  pdl_launch_dependents();
  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int b = blockIdx.x / C;
  const long long capacity = static_cast<long long>(cache.max_pages_per_req) * cache.page_size;
  const long long stride = capacity / kBlock;
  const int n = max(0, checked_ctx_len(cache, b, capacity, kKPoolSelect, rank == 0 && threadIdx.x == 0));
  const int nblk = (n + kBlock - 1) / kBlock;
  const int per = (nblk + C - 1) / C;
  const int j0 = min(rank * per, nblk);
  const int nloc = min(per, nblk - j0);
  const float* src = blockmax + b * stride + j0;
  for (int base = 0; base < nloc; base += kPoolThreads * 8) {   // 8 independent loads per thread in flight
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * kPoolThreads + threadIdx.x;
      v[u] = i < nloc ? src[i] : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * kPoolThreads + threadIdx.x;
      if (i < nloc) S.keys[i] = order_key(v[u]);
    }
  }
  const SelectStart* start = nullptr;
  if (hist != nullptr) {
    // this thread's 4 bins, highest first: thread order is descending bin order
    constexpr int kNB = kPoolHistBins / kPoolThreads;   // 4
    const int base = kNB * (kPoolThreads - 1 - static_cast<int>(threadIdx.x));
    const uint4* hb = reinterpret_cast<const uint4*>(hist + static_cast<long long>(b) * kPoolHistBins + base);
    uint32_t c[kNB];
#pragma unroll
    for (int i = 0; i < kNB / 4; ++i) {
      const uint4 v = hb[i];
      c[kNB - 1 - 4 * i] = v.x;
      c[kNB - 2 - 4 * i] = v.y;
      c[kNB - 3 - 4 * i] = v.z;
      c[kNB - 4 - 4 * i] = v.w;
    }
    if (hist_head_start<kPoolThreads, kNB>(c, base + kNB - 1, kPoolHistBits, nblk, P, S.sel.warp_tmp, &S.start))
      start = &S.start;
  }
  __syncthreads();   // the keys (and a head start) are in shared memory
  int32_t* out = pool + static_cast<long long>(b) * P;
  cluster_topk<kPoolThreads>(
      S.keys, nloc, P, S.sel, [&](int i, int r) { out[r] = j0 + i; }, [&](int r) { out[r] = -1; }, start);
  if (hist != nullptr) {   // every CTA has read the histogram before the select's last cluster barrier
    const int per = kPoolHistBins / C;
    uint4* hz = reinterpret_cast<uint4*>(hist + static_cast<long long>(b) * kPoolHistBins + rank * per);
    for (int i = threadIdx.x; i < per / 4; i += kPoolThreads) hz[i] = make_uint4(0u, 0u, 0u, 0u);
  }
}

// --------------------------------------------------------------- reindex ----
constexpr int kRThreads = 320;          // producer, MMA, two epilogue warpgroups
constexpr int kRStages = 4;
constexpr int kRAcc = 4;
constexpr int kBlkBytes = kBlock * kIndexDim;       // 1 KB: one block of 8 indexer-K rows
constexpr int kBlocksPerTile = kTile / kBlock;      // 16
constexpr uint32_t kRTmemCols = kRAcc * kAccCols;
constexpr int kMaxReindexBlocks = 1024;   // candidate blocks per CTA (8 CTAs: 65,536 positions without a pool)

struct ReindexBarriers {
  uint64_t full[kRStages];
  uint64_t empty[kRStages];
  uint64_t acc_full[kRAcc];
  uint64_t acc_empty[kRAcc];
  uint64_t q_full;
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort_flag;
};

// Dynamic shared memory: [tiles][q tile][barriers][select][keys][blk_exp][blk_row][blk_id]
struct ReindexLayout {
  uint32_t tiles, qtile, bars, sel, keys, blk_exp, blk_row, blk_id, total;
  __host__ __device__ static ReindexLayout make(int max_blocks) {
    ReindexLayout L;
    L.tiles = 0;
    L.qtile = kRStages * kTileBytes;
    L.bars = L.qtile + kQBytes;
    L.sel = (L.bars + sizeof(ReindexBarriers) + 15) & ~15u;
    L.keys = (L.sel + sizeof(SelectSmem) + 15) & ~15u;
    L.blk_exp = L.keys + max_blocks * kBlock * 4;
    L.blk_row = L.blk_exp + max_blocks * 8;
    L.blk_id = L.blk_row + max_blocks * 4;
    L.total = L.blk_id + max_blocks * 4;
    return L;
  }
};

__global__ void __launch_bounds__(kRThreads, 2)
    reindex_kernel(const csa2_cache cache, const int32_t* __restrict__ pool, int P, const float* __restrict__ q,
                   const float* __restrict__ w, const float* __restrict__ full_scores, int K,
                   int32_t* __restrict__ topk, const __grid_constant__ CUtensorMap blk_map, int max_blocks,
                   uint64_t wait_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const ReindexLayout L = ReindexLayout::make(max_blocks);
  uint8_t* tiles = base + L.tiles;
  uint8_t* qtile = base + L.qtile;
  ReindexBarriers& R = *reinterpret_cast<ReindexBarriers*>(base + L.bars);
  SelectSmem& sel = *reinterpret_cast<SelectSmem*>(base + L.sel);
  uint32_t* keys = reinterpret_cast<uint32_t*>(base + L.keys);
  uint64_t* blk_exp = reinterpret_cast<uint64_t*>(base + L.blk_exp);   // 8 exponent bytes per block
  int* blk_row = reinterpret_cast<int*>(base + L.blk_row);
  int* blk_id = reinterpret_cast<int*>(base + L.blk_id);

  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int b = blockIdx.x / C;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long capacity = static_cast<long long>(cache.max_pages_per_req) * cache.page_size;
  pdl_wait();                 // the pool (or the stored scores) of the preceding launch are complete
  pdl_launch_dependents();
  const int n_raw = checked_ctx_len(cache, b, capacity, kKReindex, rank == 0 && tid == 0);
  const int n = max(0, n_raw);

  // ---- this CTA's candidate blocks ----
  int e0, nloc;
  if (pool != nullptr) {
    const int per = (P + C - 1) / C;
    e0 = min(rank * per, P);
    nloc = min(per, P - e0);
  } else {
    const int nblk = (n + kBlock - 1) / kBlock;
    const int per = (nblk + C - 1) / C;
    e0 = min(rank * per, nblk);
    nloc = min(per, nblk - e0);
  }
  if (nloc > max_blocks) nloc = max_blocks;   // host guarantees this never clips
  if (n_raw < 0) nloc = 0;                     // corrupt length: no candidates
  // block id -> page -> exponent bytes: each level's loads are issued together
  constexpr int kU = 4;
  for (int base = 0; base < nloc; base += kRThreads * kU) {
    int j[kU], page[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = base + u * kRThreads + tid;
      j[u] = i >= nloc ? -1 : (pool != nullptr ? pool[static_cast<long long>(b) * P + e0 + i] : e0 + i);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const bool in = j[u] >= 0 && static_cast<long long>(j[u]) * kBlock < n;
      page[u] = in ? cache.page_table[static_cast<long long>(b) * cache.max_pages_per_req +
                                      j[u] * kBlock / cache.page_size]
                   : -1;
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = base + u * kRThreads + tid;
      if (i >= nloc) continue;
      int row = -1;
      if (j[u] >= 0 && static_cast<long long>(j[u]) * kBlock < n) {
        const int t = j[u] * kBlock;
        if (page[u] >= 0 && page[u] < cache.num_pages) row = page[u] * cache.page_size + t % cache.page_size;
        else report_error(cache.err_word, CSA2_ERR_DEVICE_BOUNDS, kKReindex, b, t);
      } else if (j[u] >= 0 || j[u] < -1) {
        report_error(cache.err_word, CSA2_ERR_DEVICE_BOUNDS, kKReindex, b, j[u]);
      }
      blk_row[i] = row;
      blk_id[i] = row >= 0 ? j[u] : -1;
      page[u] = row;   // reuse as the row for the exponent load below
    }
    if (full_scores == nullptr) {
      uint64_t ex[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int i = base + u * kRThreads + tid;
        ex[u] = (i < nloc && page[u] >= 0) ? *reinterpret_cast<const uint64_t*>(cache.ik_exp + page[u])
                                            : 0x7F7F7F7F7F7F7F7Full;
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int i = base + u * kRThreads + tid;
        if (i < nloc) blk_exp[i] = ex[u];
      }
    }
  }
  const int n_tiles = (nloc + kBlocksPerTile - 1) / kBlocksPerTile;
  const bool recompute = full_scores == nullptr;
  if (recompute && tid == 0) {
    for (int s = 0; s < kRStages; ++s) {
      mbar_init(&R.full[s], 1);
      mbar_init(&R.empty[s], 1);
    }
    for (int a = 0; a < kRAcc; ++a) {
      mbar_init(&R.acc_full[a], 1);
      mbar_init(&R.acc_empty[a], 4);
    }
    mbar_init(&R.q_full, 4);
    mbar_init(&R.drain, 1);
    R.abort_flag = 0;
    fence_barrier_init();
  }
  if (recompute && warp == 1) {
    tmem_alloc(&R.tmem_base, kRTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (!recompute) {
    // ---- Full mode from the stored scan scores ----
    const float* src = full_scores + b * capacity;
    for (int i = tid; i < nloc * kBlock; i += kRThreads) {
      const int e = i / kBlock;
      const int p = blk_id[e] * kBlock + (i % kBlock);
      keys[i] = (blk_id[e] >= 0 && p < n) ? order_key(src[p]) : 0u;
    }
  } else if (n_tiles > 0) {
    const uint32_t tmem = R.tmem_base;
    if (warp == 0) {
      // ---- producer: lane l < 16 gathers block l of each tile ----
      const uint64_t policy = l2_policy_evict_normal();
      int issued = 0;
      for (int t = 0; t < n_tiles; ++t) {
        const int s = t % kRStages;
        const uint32_t ph = (t / kRStages) & 1;
        if (!mbar_wait_warp(&R.empty[s], ph ^ 1, wait_ns) || warp_flag(&R.abort_flag)) {
          if (lane == 0) {
            report_error(cache.err_word, CSA2_ERR_TIMEOUT, kKReindex, b, t);
            R.abort_flag = 1;
          }
          break;
        }
        const int e = t * kBlocksPerTile + lane;
        const int row = (lane < kBlocksPerTile && e < nloc) ? blk_row[e] : -1;
        const uint32_t bytes = __popc(__ballot_sync(0xffffffffu, row >= 0)) * kBlkBytes;
        if (lane == 0) mbar_arrive_expect_tx(&R.full[s], bytes);   // before any of the tile's copies
        __syncwarp();
        if (row >= 0) tma_load_2d(tiles + s * kTileBytes + lane * kBlkBytes, &blk_map, &R.full[s], 0, row, policy);
        ++issued;
      }
      if (lane == 0)
        for (int i = issued > kRStages ? issued - kRStages : 0; i < issued; ++i)
          (void)mbar_wait(&R.full[i % kRStages], (i / kRStages) & 1, kWaitLimitNs / 2);
    } else if (warp == 1) {
      if (lane == 0) {   // ---- MMA issuer ----
        bool ok = mbar_wait(&R.q_full, 0, wait_ns);
        for (int t = 0; ok && t < n_tiles; ++t) {
          const int s = t % kRStages;
          const uint32_t ph = (t / kRStages) & 1;
          const int a = t % kRAcc;
          const uint32_t aph = (t / kRAcc) & 1;
          if (!mbar_wait(&R.acc_empty[a], aph ^ 1, wait_ns) || !mbar_wait(&R.full[s], ph, wait_ns)) {
            ok = false;
            break;
          }
          if (R.abort_flag) break;
          tc_fence_after();
          const uint64_t adesc = sw128_kmajor_desc(smem_u32(tiles + s * kTileBytes));
          const uint64_t bdesc = sw128_kmajor_desc(smem_u32(qtile));
#pragma unroll
          for (int k = 0; k < kIndexDim / 32; ++k)
            umma_f8f6f4(tmem + a * kAccCols, adesc + 2 * k, bdesc + 2 * k, kIdesc, k > 0 ? 1u : 0u);
          umma_commit(&R.empty[s]);
          umma_commit(&R.acc_full[a]);
        }
        if (!ok) {
          report_error(cache.err_word, CSA2_ERR_TIMEOUT, kKReindex, b, -1);
          R.abort_flag = 1;
        }
        umma_commit(&R.drain);
        (void)mbar_wait(&R.drain, 0, kWaitLimitNs);
      }
    } else {
      // ---- epilogue: warpgroups 2..5 and 6..9 take alternate tiles ----
      const int group = (warp - 2) >> 2, ew = (warp - 2) & 3, quarter = warp & 3, m = quarter * 32 + lane;
      const float* qb = q + static_cast<long long>(b) * kIndexHeads * kIndexDim;
      if (group == 0) {
        prepare_query_codes(qb, qtile, ew, lane);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&R.q_full);
      }
      float ws[32];
      load_head_weights(qb, w + b * kIndexHeads, ws, lane);
      for (int t = group; t < n_tiles; t += 2) {
        const int a = t % kRAcc;
        const uint32_t aph = (t / kRAcc) & 1;
        const int e = t * kBlocksPerTile + m / kBlock;
        const int o = m % kBlock;
        const int row = e < nloc ? blk_row[e] : -1;
        const bool valid = row >= 0 && blk_id[e] * kBlock + o < n;
        const uint32_t e_byte = valid ? static_cast<uint32_t>((blk_exp[e] >> (8 * o)) & 0xFFu) : 127u;
        if (!mbar_wait_warp(&R.acc_full[a], aph, wait_ns)) {
          if (lane == 0) {
            report_error(cache.err_word, CSA2_ERR_TIMEOUT, kKReindex, b, t);
            R.abort_flag = 1;
          }
          break;
        }
        tc_fence_after();
        uint32_t acc[32];
        tmem_ld_32x32b_x32(tmem + a * kAccCols + (static_cast<uint32_t>(quarter * 32) << 16), acc);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&R.acc_empty[a]);
        if (e < nloc) keys[e * kBlock + o] = valid ? order_key(score_from_acc(acc, ws, e_byte)) : 0u;
        if (warp_flag(&R.abort_flag)) break;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (recompute && warp == 1) {
    tc_fence_after();
    tmem_dealloc(R.tmem_base, kRTmemCols);
  }
  int32_t* out = topk + static_cast<long long>(b) * K;
  cluster_topk<kRThreads>(
      keys, nloc * kBlock, K, sel,
      [&](int i, int r) { out[r] = blk_id[i / kBlock] * kBlock + (i % kBlock); },
      [&](int r) { out[r] = -1; });
}

__global__ void copy_topk_kernel(const int32_t* __restrict__ src, int32_t* __restrict__ dst, long long n) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    dst[i] = src[i];
}

template <class Kernel, class... Args>
cudaError_t launch_cluster(Kernel kernel, int grid, int threads, size_t smem, int cluster, cudaStream_t stream,
                           Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // the kernels call pdl_wait()
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Attributes of a cluster kernel, set once per CUDA context.
template <class Kernel>
cudaError_t configure(Kernel kernel, size_t smem, ContextMemo& memo) {
  return memo.once([&] {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    return e;
  });
}

}  // namespace

cudaError_t launch_pool_select(const csa2_cache& cache, const float* blockmax, uint32_t* hist, int pool_blocks,
                               int32_t* pool, int cluster, cudaStream_t stream) {
  static ContextMemo done;
  const size_t smem = sizeof(PoolSmem);
  cudaError_t e = configure(pool_select_kernel, smem, done);
  if (e != cudaSuccess) return e;
  return launch_cluster(pool_select_kernel, cache.batch * cluster, kPoolThreads, smem, cluster, stream, cache,
                        blockmax, hist, pool_blocks, pool);
}

size_t reindex_smem_bytes(int max_blocks) { return ReindexLayout::make(max_blocks).total + 1024; }

cudaError_t launch_reindex(const csa2_cache& cache, const int32_t* pool, int pool_blocks, const float* q,
                           const float* w, const float* full_scores, int k, int32_t* topk,
                           const CUtensorMap& blk_map, int max_blocks, uint64_t wait_ns, cudaStream_t stream) {
  static ContextMemo done;
  // 16 CTAs per request over a pool (a few tiles each, several CTAs per SM),
  // 8 over a whole context of up to 65,536 positions
  const int cluster = pool != nullptr ? kReindexPoolCluster : 8;
  const size_t smem_max = reindex_smem_bytes(kMaxReindexBlocks);
  cudaError_t e = configure(reindex_kernel, smem_max, done);
  if (e != cudaSuccess) return e;
  return launch_cluster(reindex_kernel, cache.batch * cluster, kRThreads, reindex_smem_bytes(max_blocks), cluster,
                        stream, cache, pool, pool_blocks, q, w, full_scores, k, topk, blk_map, max_blocks, wait_ns);
}

cudaError_t launch_copy_topk(const int32_t* src, int32_t* dst, long long n, cudaStream_t stream) {
  const int threads = 256;
  const long long blocks = (n + threads - 1) / threads;
  copy_topk_kernel<<<static_cast<unsigned>(blocks < 1024 ? (blocks > 0 ? blocks : 1) : 1024), threads, 0, stream>>>(
      src, dst, n);
  return cudaGetLastError();
}

}  // namespace csa2
