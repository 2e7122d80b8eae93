// Full-mode indexer scan (first stage of the Hierarchical Sparse Indexer):
// every visible position of every request is scored against that request's
// indexer query, and the max of each block of 8 positions is written out
// [4sapi blog, section 四; alphalab analysis, section 2 CSA2: the first Full
// layer scans the whole visible context].
//
// Design (sm_100a), one persistent CTA per SM; the concatenated work units of
// all requests (256 positions each) are split into contiguous ranges, one per
// CTA:
//   * warp 0: producer.  Every 32 units the warp finds their cache rows in
//     parallel (one unit per lane: request, page-table entry, row; the
//     page-table loads of the next 32 are in flight while lane 0 issues the
//     current 32), so that the issuing lane does no address arithmetic and
//     waits on no global load.  Per unit, lane 0 issues one TMA load of the
//     256-row unit (128 FP8 bytes per row, 128-byte swizzle; two 128-row
//     loads when a page holds an odd number of 128-row tiles) and one bulk
//     copy of its 256 exponent bytes into one stage of a kStages ring.  The
//     issuing lane is the scan's pacing resource: it shares its SM
//     sub-partition with two epilogue warps, and every instruction it saves
//     is time the copies spend in flight;
//   * warp 1 (one lane): tcgen05.mma kind::f8f6f4, M = 128 positions, N = 32
//     heads, K = 128 in 4 steps, per sub-tile, into an accumulator pair (one of
//     kAcc) in TMEM; the stage is released by the MMAs' completion together
//     with the epilogue warps' reads of its exponent bytes;
//   * warps 2..9: two epilogue warpgroups taking alternate units, one thread
//     per position of each sub-tile: tcgen05.ld of the 32 head dot products,
//     score, block max over 8 lanes, stores.  The exponent bytes come from
//     the stage (per-thread byte loads from global memory put their latency
//     and address arithmetic on the epilogue warps, which share issue slots
//     with the producer).  Group 0 also quantises each
//     request's query into the B-operand tile (three buffers) for the MMA.
//     With a histogram buffer, each block max also adds one count to its
//     request's histogram of leading order-key bits (in shared memory, flushed
//     once per CTA: the maxima crowd into few bins, and global atomics on them
//     would serialise), from which the pool selection finds its threshold's
//     leading bits without a pass.
// Per 256 positions the handshake is one stage and one accumulator pair: the
// scan streams at the HBM rate instead of the rate of barrier round trips.
// Every mbarrier wait is bounded; a wait that runs out records
// CSA2_ERR_TIMEOUT and the CTA leaves its loops, drains, frees TMEM, returns.
#include <cub/block/block_scan.cuh>

#include "index_common.cuh"
#include "launch.h"
#include "scan_units.cuh"

namespace csa2 {

namespace {

constexpr int kUnit = kScanUnit;           // positions per work unit (two MMA sub-tiles)
constexpr int kStages = 6;                 // unit ring (32 KB each)
constexpr int kAcc = 4;                    // TMEM accumulator pairs (2 x 32 columns each)
constexpr int kEpiGroups = 2;
constexpr int kQBufs = 3;                  // query-code buffers (segments in flight)
constexpr int kThreads = 64 + kEpiGroups * 128;
constexpr int kMaxBatchScan = 1024;
constexpr int kScanItems = (kMaxBatchScan + kThreads - 1) / kThreads;
constexpr uint32_t kTmemCols = kAcc * 2 * kAccCols;   // 256

struct __align__(1024) IndexSmem {
  uint8_t tiles[kStages][2][kTileBytes];
  uint8_t q[kQBufs][kQBytes];
  union {
    struct {
      uint8_t exps[kStages][kUnit];    // exponent bytes of the stage's unit
      int rowq[32][2];                 // cache rows of the producer's current 32 units (-1: none)
    };
    cub::BlockScan<int, kThreads>::TempStorage scan_tmp;   // the prologue's prefix sum only
  };
  int prefix[kMaxBatchScan + 1];       // units before request b
  uint64_t full[kStages];
  uint64_t empty[kStages];             // the MMAs' completion + the 4 epilogue warps of the unit
  uint64_t acc_full[kAcc];
  uint64_t acc_empty[kAcc];
  uint64_t q_full[kQBufs];
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort_flag;
  // block-max histogram of the CTA's first two requests (slot = request -
  // first request), two 16-bit counts per word; flushed to global memory once
  uint32_t hist[2][kPoolHistBins / 2];
};

__global__ void __launch_bounds__(kThreads, 1)
    index_full_kernel(const csa2_cache cache, const float* __restrict__ q, const float* __restrict__ w,
                      float* __restrict__ blockmax, float* __restrict__ scores, uint32_t* __restrict__ hist,
                      const __grid_constant__ CUtensorMap ik_map, int whole_units, uint64_t wait_ns) {
  extern __shared__ uint8_t smem_raw[];
  IndexSmem& S = *reinterpret_cast<IndexSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int B = cache.batch;
  const long long capacity = static_cast<long long>(cache.max_pages_per_req) * cache.page_size;
  const uint32_t page_size = static_cast<uint32_t>(cache.page_size);

  pdl_wait();                 // the cache rows of a preceding append are complete
  pdl_launch_dependents();    // the pool selection may be launched (it waits for this grid)

  // ---- tiles per request, prefix sums ----
  {
    using Scan = cub::BlockScan<int, kThreads>;
    int items[kScanItems];
#pragma unroll
    for (int i = 0; i < kScanItems; ++i) {
      const int b = tid * kScanItems + i;
      int n = 0;
      if (b < B) n = max(0, checked_ctx_len(cache, b, capacity, kKIndexFull, blockIdx.x == 0));
      items[i] = (n + kUnit - 1) / kUnit;
    }
    int total;
    Scan(S.scan_tmp).ExclusiveSum(items, items, total);
#pragma unroll
    for (int i = 0; i < kScanItems; ++i) {
      const int b = tid * kScanItems + i;
      if (b <= B) S.prefix[b] = items[i];
    }
    if (tid == 0) S.prefix[B] = total;
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 5);
    }
    for (int a = 0; a < kAcc; ++a) {
      mbar_init(&S.acc_full[a], 1);
      mbar_init(&S.acc_empty[a], 4);
    }
    for (int k = 0; k < kQBufs; ++k) mbar_init(&S.q_full[k], 4);   // the 4 warps of epilogue group 0
    mbar_init(&S.drain, 1);
    S.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) tma_prefetch_map(&ik_map);
  if (hist != nullptr)
    for (int i = tid; i < kPoolHistBins; i += kThreads) (&S.hist[0][0])[i] = 0u;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const int total = S.prefix[B];
  const int G = gridDim.x;
  const int t_begin = static_cast<int>((static_cast<long long>(total) * blockIdx.x) / G);
  const int t_end = static_cast<int>((static_cast<long long>(total) * (blockIdx.x + 1)) / G);
  const int n_tiles = t_end - t_begin;
  const uint32_t tmem = S.tmem_base;
  // The histogram counts of this CTA's first two requests go to shared
  // memory (16-bit counts: at most 32 blocks per unit, so fewer than 2^16 per
  // bin while the CTA has fewer than 2048 units); other requests', or all
  // when the CTA has more units, straight to global memory.
  int hist_b0 = 0;
  {
    TileIter first;
    first.init(S.prefix, B, t_begin);
    hist_b0 = first.b;
  }
  const bool hist_smem = n_tiles < 2048;

  if (n_tiles > 0) {
    if (warp == 0) {
      // ================= producer =================
      const uint64_t policy = l2_policy_evict_first();
      const uint32_t full_mask = 0xffffffffu;
      UnitRows next;   // this lane's unit of the next 32
      next.fetch(cache, S.prefix, B, t_begin + lane, lane < n_tiles, capacity, page_size);
      int issued = 0;   // lane 0
      bool stop = false;
      for (int i0 = 0; i0 < n_tiles && !stop; i0 += 32) {
        int r[2];
        next.rows(cache, capacity, kKIndexFull, r);
        S.rowq[lane][0] = r[0];
        S.rowq[lane][1] = r[1];
        // the next 32 units' page-table loads are in flight while lane 0 issues
        next.fetch(cache, S.prefix, B, t_begin + i0 + 32 + lane, i0 + 32 + lane < n_tiles, capacity, page_size);
        __syncwarp();
        if (lane == 0) {
          const int n = min(32, n_tiles - i0);
          for (int k = 0; k < n; ++k) {
            const int i = i0 + k, s = i % kStages;
            if (!mbar_wait(&S.empty[s], ((i / kStages) & 1) ^ 1, wait_ns)) {
              report_error(cache.err_word, CSA2_ERR_TIMEOUT, kKIndexFull, -1, i);
              S.abort_flag = 1;
            }
            if (S.abort_flag) {
              stop = true;
              break;
            }
            const int r0 = S.rowq[k][0], r1 = S.rowq[k][1];
            // rows are multiples of 128, so the exponent copies start 16-byte aligned
            if (whole_units && r0 >= 0) {   // the unit's 256 rows are consecutive
              mbar_arrive_expect_tx(&S.full[s], 2 * kTileBytes + kUnit);
              tma_load_2d(S.tiles[s][0], &ik_map, &S.full[s], 0, r0, policy);
              bulk_load_1d(S.exps[s], cache.ik_exp + r0, kUnit, &S.full[s], policy);
            } else {
              mbar_arrive_expect_tx(&S.full[s], (r0 >= 0) * (kTileBytes + kTile) + (r1 >= 0) * (kTileBytes + kTile));
              if (r0 >= 0) {
                tma_load_2d(S.tiles[s][0], &ik_map, &S.full[s], 0, r0, policy);
                bulk_load_1d(S.exps[s], cache.ik_exp + r0, kTile, &S.full[s], policy);
              }
              if (r1 >= 0) {
                tma_load_2d(S.tiles[s][1], &ik_map, &S.full[s], 0, r1, policy);
                bulk_load_1d(S.exps[s] + kTile, cache.ik_exp + r1, kTile, &S.full[s], policy);
              }
            }
            ++issued;
          }
        }
        stop = __shfl_sync(full_mask, stop, 0);
        __syncwarp();
      }
      if (lane == 0) {
        // copies still in flight (only after an abort): wait for the last one of each stage
        for (int i = issued > kStages ? issued - kStages : 0; i < issued; ++i)
          (void)mbar_wait(&S.full[i % kStages], (i / kStages) & 1, kWaitLimitNs / 2);
      }
    } else if (warp == 1) {
      // ================= MMA issuer =================
      // The issuing lane is on the scan's critical path (its instructions share
      // an SM sub-partition with two epilogue warps): descriptors come from
      // one base by adding stage offsets, the query's only when the request
      // changes, and a count of the request's remaining units replaces the
      // unit walker.
      if (lane == 0) {
        TileIter it;
        it.init(S.prefix, B, t_begin);
        int seg = 0, cur_b = it.b;
        int left = S.prefix[cur_b + 1] - S.prefix[cur_b] - it.j;   // units of this request from here
        bool ok = mbar_wait(&S.q_full[0], 0, wait_ns);
        const uint64_t adesc0 = sw128_kmajor_desc(smem_u32(S.tiles[0][0]));
        uint64_t bdesc = sw128_kmajor_desc(smem_u32(S.q[0]));
        int s = 0, a = 0;                  // i % kStages, i % kAcc
        uint32_t ph_s = 0, ph_a = 0;       // (i / kStages) & 1, (i / kAcc) & 1
        for (int i = 0; ok && i < n_tiles; ++i) {
          if (left == 0) {   // the next request with units: the next query buffer
            cur_b = next_request_with_tiles(S.prefix, B, cur_b);
            left = S.prefix[cur_b + 1] - S.prefix[cur_b];
            ++seg;
            if (!mbar_wait(&S.q_full[seg % kQBufs], (seg / kQBufs) & 1, wait_ns)) { ok = false; break; }
            bdesc = sw128_kmajor_desc(smem_u32(S.q[seg % kQBufs]));
          }
          --left;
          if (!mbar_wait(&S.acc_empty[a], ph_a ^ 1, wait_ns) || !mbar_wait(&S.full[s], ph_s, wait_ns)) {
            ok = false;
            break;
          }
          if (S.abort_flag) break;
          tc_fence_after();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            // start-address field: bits 0..13 of the descriptor (address / 16)
            const uint64_t adesc = adesc0 + static_cast<uint64_t>(((2 * s + h) * kTileBytes) >> 4);
#pragma unroll
            for (int k = 0; k < kIndexDim / 32; ++k)
              umma_f8f6f4(tmem + (2 * a + h) * kAccCols, adesc + 2 * k, bdesc + 2 * k, kIdesc, k > 0 ? 1u : 0u);
          }
          umma_commit(&S.empty[s]);
          umma_commit(&S.acc_full[a]);
          if (++s == kStages) {
            s = 0;
            ph_s ^= 1u;
          }
          if (++a == kAcc) {
            a = 0;
            ph_a ^= 1u;
          }
        }
        if (!ok) {
          report_error(cache.err_word, CSA2_ERR_TIMEOUT, kKIndexFull, cur_b, -1);
          S.abort_flag = 1;
        }
        umma_commit(&S.drain);                       // all MMAs issued above are complete
        (void)mbar_wait(&S.drain, 0, kWaitLimitNs);
      }
    } else {
      // ================= epilogue groups (warps 2..5, 6..9) =================
      const int group = (warp - 2) >> 2;
      const int ew = (warp - 2) & 3;           // 0..3: this warp's share of the query codes
      const int quarter = warp & 3;            // TMEM lane quarter of this warp
      const int toff = quarter * 32 + lane;    // position inside the tile
      auto timed_out = [&](int where) {
        if (lane == 0) {
          report_error(cache.err_word, CSA2_ERR_TIMEOUT, kKIndexFull, -1, where);
          S.abort_flag = 1;
        }
      };
      // Query codes (group 0 only): segment x goes to buffer x % 3.  Writing
      // segment x needs the MMAs of segment x - 3 complete, which holds once
      // group 0 has seen an accumulator of segment x - 2 or later.  Group 0
      // keeps the codes two segments ahead of its current one: between two of
      // its tiles at most two segments begin, so the MMA never waits for codes
      // that group 0 would write only after an accumulator it cannot get.
      int prep_b = 0, prep_x = 0;
      auto prepare = [&]() {
        prepare_query_codes(q + static_cast<long long>(prep_b) * kIndexHeads * kIndexDim, S.q[prep_x % kQBufs], ew,
                            lane);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.q_full[prep_x % kQBufs]);
        prep_b = next_request_with_tiles(S.prefix, B, prep_b);
        ++prep_x;
      };
      TileIter it;
      it.init(S.prefix, B, t_begin);
      int seg = 0, cur_b = it.b;
      if (group == 0) {
        prep_b = cur_b;
        for (int k = 0; k < kQBufs && prep_b < B && S.prefix[prep_b] < t_end; ++k) prepare();
      }
      float ws[32];
      load_head_weights(q + static_cast<long long>(cur_b) * kIndexHeads * kIndexDim, w + cur_b * kIndexHeads, ws,
                        lane);
      int nb = cache.ctx_len[cur_b];
      if (group == 1) it.advance();


      for (int i = group; i < n_tiles; i += kEpiGroups) {
        if (it.b != cur_b) {
          // count the segments passed; group 0 keeps the codes two segments ahead
          for (int b = cur_b; b != it.b; b = next_request_with_tiles(S.prefix, B, b)) ++seg;
          cur_b = it.b;
          load_head_weights(q + static_cast<long long>(cur_b) * kIndexHeads * kIndexDim, w + cur_b * kIndexHeads,
                            ws, lane);
          nb = cache.ctx_len[cur_b];
        }
        const int a = i % kAcc, s = i % kStages;
        const int j = it.j;
        TileIter nx = it;
        nx.advance();
        nx.advance();

        // The stage's copies completed before the MMAs were issued; the wait
        // on its full barrier (the phase of this unit: the stage is not
        // refilled before this warp releases it) makes them visible here.
        if (!mbar_wait_warp(&S.acc_full[a], (i / kAcc) & 1, wait_ns) ||
            !mbar_wait_warp(&S.full[s], (i / kStages) & 1, wait_ns)) {
          timed_out(j);
          break;
        }
        tc_fence_after();
        uint32_t acc0[32], acc1[32];
        tmem_ld_32x32b_x32(tmem + (2 * a) * kAccCols + (static_cast<uint32_t>(quarter * 32) << 16), acc0);
        tmem_ld_32x32b_x32(tmem + (2 * a + 1) * kAccCols + (static_cast<uint32_t>(quarter * 32) << 16), acc1);
        const uint32_t ex[2] = {S.exps[s][toff], S.exps[s][kTile + toff]};
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&S.acc_empty[a]);
          mbar_arrive(&S.empty[s]);
        }
        // Group 0 writes the codes of up to two segments ahead only after this
        // unit's accumulator: the buffer it reuses held the previous segment,
        // whose last unit may be group 1's and issued after group 0's previous
        // accumulator.
        if (group == 0)
          while (prep_x <= seg + 2 && prep_b < B && S.prefix[prep_b] < t_end) prepare();

#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int p = j * kUnit + h * kTile + toff;
          const bool valid = p < nb;
          const float sc = score_from_acc(h == 0 ? acc0 : acc1, ws, ex[h]);
          float bm = valid ? sc : -INFINITY;
          bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
          bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
          bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
          if ((lane & 7) == 0 && valid) {
            blockmax[static_cast<long long>(cur_b) * (capacity / kBlock) + p / kBlock] = bm;
            // one count per block in the request's histogram of leading key bits
            if (hist != nullptr) {
              const uint32_t bin = order_key(bm) >> (32 - kPoolHistBits);
              const int slot = cur_b - hist_b0;
              if (hist_smem && slot < 2) atomicAdd(&S.hist[slot][bin >> 1], 1u << (16 * (bin & 1)));
              else atomicAdd(&hist[static_cast<long long>(cur_b) * kPoolHistBins + bin], 1u);
            }
          }
          if (scores != nullptr && valid) scores[static_cast<long long>(cur_b) * capacity + p] = sc;
        }
        if (warp_flag(&S.abort_flag)) break;
        it = nx;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (hist != nullptr && hist_smem) {   // flush the non-zero counts of the two slots
    for (int i = tid; i < kPoolHistBins; i += kThreads) {
      const int slot = i / (kPoolHistBins / 2), w2 = i % (kPoolHistBins / 2);
      const int b = hist_b0 + slot;
      const uint32_t v = S.hist[slot][w2];
      if (v == 0u || b >= B) continue;
      uint32_t* g = hist + static_cast<long long>(b) * kPoolHistBins + 2 * w2;
      if (v & 0xFFFFu) atomicAdd(g, v & 0xFFFFu);
      if (v >> 16) atomicAdd(g + 1, v >> 16);
    }
  }
}

}  // namespace

// 227 KB per block with no static shared memory (the prefix sum's scratch is
// in the union above), 1 KB of it for aligning the struct
static_assert(sizeof(IndexSmem) + 1024 <= 227 * 1024, "the scan's shared memory exceeds one SM");
size_t index_full_smem_bytes() { return sizeof(IndexSmem) + 1024; }

cudaError_t launch_index_full(const csa2_cache& cache, const float* q, const float* w, float* blockmax,
                              float* scores, uint32_t* hist, const CUtensorMap& ik_map, int whole_units, int num_sms,
                              uint64_t wait_ns, cudaStream_t stream) {
  static ContextMemo attrs;
  const size_t smem = index_full_smem_bytes();
  const cudaError_t e = attrs.once([&] {
    return cudaFuncSetAttribute(index_full_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  });
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, index_full_kernel, cache, q, w, blockmax, scores, hist, ik_map, whole_units, wait_ns);
}

}  // namespace csa2
