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
constexpr int kPoolThreads = 1024;
constexpr int kPoolKeysPerCta = 16384;
constexpr int kPoolKpt = kPoolKeysPerCta / kPoolThreads;   // 16 consecutive keys per thread
constexpr int kPoolGather = 8192;                          // threshold-bin keys rank 0 gathers
constexpr int kPoolGpt = kPoolGather / kPoolThreads;       // 8 per thread (two 16-byte loads)

struct PoolFinal {
  uint32_t prefix, mask;   // the selection: masked bits above prefix, ties on it
  int base;                // output rank of this CTA's first selection
  int quota;               // ties this CTA takes (lowest block ids first)
  int total;               // selections of the cluster
};

struct PoolSmem {
  union {
    uint32_t keys[kPoolKeysPerCta];   // general path: the cluster select's keys
    uint32_t cand[kPoolKeysPerCta];   // this CTA's keys in the threshold's bin, padded with zeros to 4
  };
  SelectSmem sel;
  BlockSelectSmem bsel;               // rank 0: the select inside the bin
  SelectStart start;
  int bin_count;                      // keys in the threshold's bin (histogram)
  int n_cand, n_gt;                   // this CTA's keys in / above the bin, read remotely
  int hist_ok;                        // the counts agree with the histogram
  int cbase[kMaxCluster + 1];         // rank 0: first gathered slot of each rank (padded lists)
  int gt_above[kMaxCluster];          // rank 0: per rank, keys above the bin
  int gt_bin[kMaxCluster], eq_bin[kMaxCluster];   // rank 0: per rank, bin keys above / on the final prefix
  PoolFinal fin;                      // written by rank 0
  uint32_t wsum[32];                  // per warp: selections (low 16 bits) and ties (high)
};

// One cluster per request; CTA `rank` holds block maxima [j0, j0 + nloc) as
// order keys, 16 consecutive ones per thread.
//
// With `hist` (the scan's per-request histogram of the leading 12 bits of the
// block-max order keys), every CTA reads it and finds the bin T that holds
// the pool's threshold, the keys above it (all selected) and how many of T's
// keys are still needed.  Every CTA counts its keys above T and in T; when T
// holds at most ~8,100 keys (the maxima crowd into few bins: 2-6 % of a
// request's blocks fall in the threshold's bin on the bench workload) it also
// compacts its keys in T into shared memory.  After one cluster barrier every
// CTA checks all ranks' counts against the histogram; the rank-0 CTA gathers
// T's keys through distributed shared memory (16-byte loads), finds the exact
// threshold among them with the block radix select (10-bit digits, block
// barriers only), counts per rank the keys above it and on it, and writes
// every CTA its output base and its share of the ties; after a second barrier
// every CTA writes its selections in block order (one block prefix sum of
// packed selection and tie counts).  Without a histogram, or with one that
// does not describe these keys (stale, foreign), the general cluster radix
// select runs over every key; with a larger bin it starts from the verified
// bin.  The CTAs zero their slices of the histogram for the next scan.
// Every step costs instructions in all 32 warps, so each is a handful of
// instructions per thread: warp-aggregated atomics, 16-byte loads, one scan.
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
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t lt = (1u << lane) - 1u;

  // this thread's 4 histogram bins, highest first (thread order is descending
  // bin order)
  constexpr int kNB = kPoolHistBins / kPoolThreads;   // 4
  static_assert(kNB == 4, "one 16-byte load of bins per thread");
  const int hbase = kNB * (kPoolThreads - 1 - tid);
  uint4 hv = make_uint4(0u, 0u, 0u, 0u);
  if (hist != nullptr) hv = *reinterpret_cast<const uint4*>(hist + static_cast<long long>(b) * kPoolHistBins + hbase);

  // Slices of the request's block-max row by its capacity (a multiple of 4
  // blocks each: every slice starts 16-byte aligned when the row does), so
  // that the keys' loads need not wait for the length; keys past the length
  // are masked once it arrives.
  const long long capacity = static_cast<long long>(cache.max_pages_per_req) * cache.page_size;
  const int stride = static_cast<int>(capacity / kBlock);   // <= 16 x 16,384 (checked on the host)
  const int per = (((stride + C - 1) / C) + 3) & ~3;
  const int j0 = min(rank * per, stride);
  const int ncap = min(per, stride - j0);
  int32_t* out = pool + static_cast<long long>(b) * P;

  // ---- keys [16 tid, 16 tid + 16): all loads in flight at once ----
  uint32_t key[kPoolKpt];
  const int i0 = kPoolKpt * tid;
  int n;
  {
    const float* src = blockmax + static_cast<long long>(b) * stride + j0;
    const bool vec = (reinterpret_cast<uintptr_t>(src) & 15u) == 0u;
    float f[kPoolKpt];
    if (vec && i0 + kPoolKpt <= ncap) {
#pragma unroll
      for (int u = 0; u < kPoolKpt / 4; ++u) {
        const float4 v = *reinterpret_cast<const float4*>(src + i0 + 4 * u);
        f[4 * u] = v.x;
        f[4 * u + 1] = v.y;
        f[4 * u + 2] = v.z;
        f[4 * u + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < kPoolKpt; ++j) f[j] = i0 + j < ncap ? src[i0 + j] : 0.0f;
    }
    n = max(0, checked_ctx_len(cache, b, capacity, kKPoolSelect, rank == 0 && tid == 0));
#pragma unroll
    for (int j = 0; j < kPoolKpt; ++j) key[j] = order_key(f[j]);
  }
  const int nblk = (n + kBlock - 1) / kBlock;
  const int nloc = max(0, min(ncap, nblk - j0));   // valid keys of this CTA
#pragma unroll
  for (int j = 0; j < kPoolKpt; ++j) key[j] = i0 + j < nloc ? key[j] : 0u;

  // ---- head start from the histogram (the same in every CTA) ----
  bool head = false;
  if (hist != nullptr) {
    const uint32_t c[kNB] = {hv.w, hv.z, hv.y, hv.x};
    if (tid == 0) S.bin_count = kPoolGather + 1;
    head = hist_head_start<kPoolThreads, kNB>(c, hbase + kNB - 1, kPoolHistBits, nblk, P, S.sel.warp_tmp, &S.start,
                                              &S.bin_count);
  }
  if (tid == 0) {
    S.n_cand = 0;
    S.n_gt = 0;
  }
  __syncthreads();   // the head start, the counters
  const bool all_selected = head && S.start.done && S.start.mask == 0u;   // nblk <= P
  const bool counted = head && !all_selected;
  // the padded lists of all ranks fit the gather (each pads at most 3 zeros)
  const bool compact = counted && S.bin_count <= kPoolGather - 3 * C;
  const uint32_t t_prefix = S.start.prefix, t_mask = S.start.mask;

  if (counted) {
    // this CTA's keys above the bin and in it: one atomic per warp each
    int gt = 0, nc = 0;
#pragma unroll
    for (int j = 0; j < kPoolKpt; ++j) {
      const uint32_t km = key[j] & t_mask;
      gt += (key[j] != 0u && km > t_prefix) ? 1 : 0;
      nc += (key[j] != 0u && km == t_prefix) ? 1 : 0;
    }
    int incl = nc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int wbase = 0;
    if (lane == 31 && incl != 0) wbase = atomicAdd(&S.n_cand, incl);
    wbase = __shfl_sync(0xffffffffu, wbase, 31);
    gt = __reduce_add_sync(0xffffffffu, gt);
    if (lane == 0 && gt != 0) atomicAdd(&S.n_gt, gt);
    if (compact && nc != 0) {   // slots < 16384: at most one per key of this CTA
      int slot = wbase + incl - nc;
#pragma unroll
      for (int j = 0; j < kPoolKpt; ++j)
        if (key[j] != 0u && (key[j] & t_mask) == t_prefix) S.cand[slot++] = key[j];
    }
    __syncthreads();
    if (compact && tid < 3) {   // zeros up to a multiple of 4 (no key is 0)
      const int nc_all = S.n_cand;
      const int pad = (nc_all + 3) & ~3;
      if (nc_all + tid < pad) S.cand[nc_all + tid] = 0u;
    }
  }
  cluster.sync();   // #1: every CTA's counts and bin keys; every CTA has read the histogram

  if (hist != nullptr) {   // zero this CTA's slice of the histogram for the next scan
    const int hper = kPoolHistBins / C;
    uint4* hz = reinterpret_cast<uint4*>(hist + static_cast<long long>(b) * kPoolHistBins + rank * hper);
    for (int i = tid; i < hper / 4; i += kPoolThreads) hz[i] = make_uint4(0u, 0u, 0u, 0u);
  }

  if (all_selected) {   // every block is in the pool, in block order
#pragma unroll
    for (int j = 0; j < kPoolKpt; ++j) {
      const int i = kPoolKpt * tid + j;
      if (i < nloc) out[j0 + i] = j0 + i;
    }
    if (rank == 0)
      for (int r = nblk + tid; r < P; r += kPoolThreads) out[r] = -1;
    return;   // no shared memory of this CTA is read remotely on this path
  }

  bool hist_ok = false;
  if (counted) {
    // the counts of all ranks against the histogram (every CTA reads them)
    if (warp == 0) {
      const int nc = lane < C ? cluster.map_shared_rank(&S.n_cand, lane)[0] : 0;
      const int ng = lane < C ? cluster.map_shared_rank(&S.n_gt, lane)[0] : 0;
      const int ncp = (nc + 3) & ~3;   // padded list
      int incl = ncp;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int sum_c = __reduce_add_sync(0xffffffffu, nc);
      const int sum_g = __reduce_add_sync(0xffffffffu, ng);
      if (lane < C) {
        S.cbase[lane] = incl - ncp;
        S.gt_above[lane] = ng;
        S.gt_bin[lane] = 0;
        S.eq_bin[lane] = 0;
      }
      if (lane == C - 1) S.cbase[C] = incl;
      if (lane == 0) S.hist_ok = (sum_c == S.bin_count && sum_g == P - S.start.need) ? 1 : 0;
    }
    __syncthreads();
    hist_ok = S.hist_ok != 0;
  }

  if (!(hist_ok && compact)) {
    // ---- general path: cluster radix select over every key ----
#pragma unroll
    for (int u = 0; u < kPoolKpt / 4; ++u)
      *reinterpret_cast<uint4*>(&S.keys[kPoolKpt * tid + 4 * u]) =
          make_uint4(key[4 * u], key[4 * u + 1], key[4 * u + 2], key[4 * u + 3]);
    __syncthreads();
    // the head start only from a histogram whose threshold bin and the bins
    // above it hold exactly the keys it says (a start from a bin without the
    // keys it claims would leave the radix passes nothing to select)
    const SelectStart* start = hist_ok ? &S.start : nullptr;
    cluster_topk<kPoolThreads>(
        S.keys, nloc, P, S.sel, [&](int i, int r) { out[r] = j0 + i; }, [&](int r) { out[r] = -1; }, start);
    return;
  }

  // ---- rank 0: the threshold inside the bin, and every rank's share ----
  if (rank == 0) {
    const int M = S.cbase[C];   // padded total <= kPoolGather
    constexpr int kQ = kPoolGpt / 4;   // 16-byte loads per thread
    uint32_t g[kPoolGpt];
    int rq[kQ];
    {
      int p[kQ];
#pragma unroll
      for (int q = 0; q < kQ; ++q) {
        p[q] = kPoolGpt * tid + 4 * q;
        rq[q] = 0;
      }
      for (int r = 1; r < C; ++r) {   // rank of each load: independent shared-memory reads
        const int cb = S.cbase[r];
#pragma unroll
        for (int q = 0; q < kQ; ++q) rq[q] = cb <= p[q] ? r : rq[q];
      }
      uint4 v[kQ];
#pragma unroll
      for (int q = 0; q < kQ; ++q)
        v[q] = (!S.start.done && p[q] < M)
                   ? *reinterpret_cast<const uint4*>(cluster.map_shared_rank(&S.cand[0], rq[q]) + (p[q] - S.cbase[rq[q]]))
                   : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int q = 0; q < kQ; ++q) {
        g[4 * q] = v[q].x;
        g[4 * q + 1] = v[q].y;
        g[4 * q + 2] = v[q].z;
        g[4 * q + 3] = v[q].w;
      }
    }
    block_select_prefix(g, S.start.need, S.bsel, &S.start);   // ends with a barrier
    const uint32_t f_prefix = S.bsel.prefix, f_mask = S.bsel.mask;
    const int f_need = S.bsel.need;
    if (!S.start.done) {
      // per rank: the bin's keys above the final prefix and on it (one atomic
      // per group of lanes whose loads came from the same rank)
#pragma unroll
      for (int q = 0; q < kQ; ++q) {
        int ga = 0, eq = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t k = g[4 * q + e], km = k & f_mask;
          ga += (k != 0u && km > f_prefix) ? 1 : 0;
          eq += (k != 0u && km == f_prefix) ? 1 : 0;
        }
        const uint32_t same = __match_any_sync(0xffffffffu, rq[q]);
        ga = __reduce_add_sync(same, ga);
        eq = __reduce_add_sync(same, eq);
        if ((same & lt) == 0u) {   // the group's lowest lane
          if (ga != 0) atomicAdd(&S.gt_bin[rq[q]], ga);
          if (eq != 0) atomicAdd(&S.eq_bin[rq[q]], eq);
        }
      }
    }
    __syncthreads();
    if (warp == 0) {
      // whole bin taken: every bin key ties on the bin's prefix
      const int eq = lane < C ? (S.start.done ? cluster.map_shared_rank(&S.n_cand, lane)[0] : S.eq_bin[lane]) : 0;
      const int above = lane < C ? S.gt_above[lane] + S.gt_bin[lane] : 0;
      int eq_incl = eq;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, eq_incl, o);
        if (lane >= o) eq_incl += y;
      }
      const int quota = max(0, min(f_need - (eq_incl - eq), eq));
      const int sel = above + quota;
      int sel_incl = sel;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, sel_incl, o);
        if (lane >= o) sel_incl += y;
      }
      const int total = __shfl_sync(0xffffffffu, sel_incl, 31);
      if (lane < C)
        *cluster.map_shared_rank(&S.fin, lane) = PoolFinal{f_prefix, f_mask, sel_incl - sel, quota, total};
    }
  }
  cluster.sync();   // #2: every CTA's share is written; no remote reads after this

  // ---- this CTA's selections, in block order (thread order) ----
  const PoolFinal fin = S.fin;
  uint32_t c = 0;   // selections (low 16 bits) and ties (high 16 bits) of this thread's keys
#pragma unroll
  for (int j = 0; j < kPoolKpt; ++j) {
    const uint32_t km = key[j] & fin.mask;
    c += (key[j] != 0u && km > fin.prefix) ? 1u : 0u;
    c += (key[j] != 0u && km == fin.prefix) ? 0x10000u : 0u;
  }
  uint32_t incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) S.wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t v = S.wsum[lane];
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    S.wsum[lane] = x - v;
  }
  __syncthreads();
  if (c != 0u) {
    const uint32_t run = S.wsum[warp] + incl - c;
    int sel_b = static_cast<int>(run & 0xFFFFu), tie_b = static_cast<int>(run >> 16);
#pragma unroll
    for (int j = 0; j < kPoolKpt; ++j) {
      const uint32_t km = key[j] & fin.mask;
      const int i = kPoolKpt * tid + j;
      if (key[j] != 0u && km > fin.prefix) {
        out[fin.base + sel_b + min(tie_b, fin.quota)] = j0 + i;
        ++sel_b;
      } else if (key[j] != 0u && km == fin.prefix) {
        if (tie_b < fin.quota) out[fin.base + sel_b + tie_b] = j0 + i;
        ++tie_b;
      }
    }
  }
  if (rank == 0)
    for (int r = fin.total + tid; r < P; r += kPoolThreads) out[r] = -1;
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
