// Full-mode indexer scan over an FP4 indexer K, and its quantise-on-append
// [animattoys article, section 把精度降到4比特: V4 kept the indexer's Q and K
// in FP4].  Reading (the pages give no format): the main-KV format on the
// indexer's 128-element rows, E2M1 codes with one E4M3 scale per 16 elements,
// s = E4M3(amax / 6), no row scale, for the cached keys and for each query
// head; score s_t = sum_h w_h * ReLU(<q~_h, k~_t>) over the dequantised values.
// A position costs 72 bytes (64 code bytes + 8 scales) against the FP8
// indexer's 129.
//
// Cache layout of the FP4 indexer K (csa2_ik4): codes [rows][64], element 2i
// in the low nibble of byte i; scales in 1 KB blocks per 128-row tile, in the
// order the tensor core reads block scales (block_scale_offset), so that a
// tile's scales reach tensor memory with one bulk copy and two tcgen05.cp.
//
// index_full_fp4_kernel follows the FP8 scan (one persistent CTA per SM,
// 256-position units split into contiguous CTA ranges, two epilogue
// warpgroups on alternate units), with:
//   * two TMA producer warps, one for the even and one for the odd units;
//   * stages of two 128-row code tiles (64-byte rows, 64-byte swizzle, 8 KB
//     each) and their two 1 KB scale blocks: with pages of whole units, one
//     256-row TMA load and one 2 KB bulk copy per unit (else one of each per
//     tile), issued from cache rows the producer warp resolved 32 units at a
//     time (UnitRows);
//   * two MMA-issuing threads, one per 128-row tile of every unit: tcgen05.cp
//     of the tile's scales to tensor memory, then two tcgen05.mma
//     kind::mxf4nvf4 (K = 64 each, E4M3 block scales, M = 128 positions,
//     N = 32 heads) into the tile's accumulator, one commit per unit each;
//     the epilogue frees the stage once the accumulator pair is complete;
//   * epilogue group 0 quantises each request's query (32 heads) into FP4
//     codes and scales; each issuer copies the query's scales to its own
//     tensor-memory columns once per request segment.
// Every wait is bounded (CSA2_ERR_TIMEOUT, drain, free tensor memory, return).
#include <cub/block/block_scan.cuh>

#include "fp4.cuh"
#include "launch.h"
#include "scan_units.cuh"

namespace csa2 {

namespace {

constexpr int kUnit = kScanUnit;
constexpr int kStages = 10;
constexpr int kAcc = 4;                    // accumulator pairs
constexpr int kEpiGroups = 2;
constexpr int kQBufs = 3;
constexpr int kIssuers = 2;                 // one per 128-row tile of a unit
constexpr int kProducers = 2;               // warps 0 and 3: even and odd units
constexpr int kEpiWarp0 = kProducers + kIssuers;   // first epilogue warp
constexpr int kThreads = 32 * kEpiWarp0 + kEpiGroups * 128;
constexpr int kMaxBatchScan = 1024;
constexpr int kScanItems = (kMaxBatchScan + kThreads - 1) / kThreads;
constexpr int kCodeBytes = CSA2_IK4_CODE_BYTES;          // 64 per row
constexpr int kTileCodeBytes = kTile * kCodeBytes;       // 8 KB
constexpr int kTileScaleBytes = 1024;                    // 128 rows x 8 scales
constexpr int kQCodeBytes = kIndexHeads * kCodeBytes;    // 2 KB
constexpr int kAccCols = 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfaCol = kAcc * 2 * kAccCols;        // 256: 4 cols per (acc pair, tile, K half)
constexpr uint32_t kSfbCol = kSfaCol + kAcc * 2 * 2 * 4; // 320: 8 cols per query buffer
constexpr uint32_t kIdesc = idesc_mxf4nvf4(kTile, kIndexHeads);

struct __align__(1024) Fp4Smem {
  uint8_t tiles[kStages][2][kTileCodeBytes];
  uint8_t scales[kStages][2][kTileScaleBytes];
  uint8_t q[kQBufs][kQCodeBytes];
  uint8_t qscales[kQBufs][kTileScaleBytes];
  uint32_t hist[2][kPoolHistBins / 2];
  int rowq[kProducers][32][2];         // cache rows of each producer's current 32 units (-1: none)
  int prefix[kMaxBatchScan + 1];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[kAcc];
  uint64_t acc_empty[kAcc];
  uint64_t q_full[kQBufs];
  uint64_t drain[kIssuers];
  uint32_t tmem_base;
  volatile int abort_flag;
};

__global__ void __launch_bounds__(kThreads, 1)
    index_full_fp4_kernel(const csa2_cache cache, const uint8_t* __restrict__ ik4_scales,
                          const float* __restrict__ q, const float* __restrict__ w, float* __restrict__ blockmax,
                          float* __restrict__ scores, uint32_t* __restrict__ hist,
                          const __grid_constant__ CUtensorMap code_map, int whole_units, uint64_t wait_ns) {
  extern __shared__ uint8_t smem_raw[];
  Fp4Smem& S = *reinterpret_cast<Fp4Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int B = cache.batch;
  const long long capacity = static_cast<long long>(cache.max_pages_per_req) * cache.page_size;
  const uint32_t page_size = static_cast<uint32_t>(cache.page_size);

  pdl_wait();
  pdl_launch_dependents();

  {
    using Scan = cub::BlockScan<int, kThreads>;
    __shared__ typename Scan::TempStorage scan_tmp;
    int items[kScanItems];
#pragma unroll
    for (int i = 0; i < kScanItems; ++i) {
      const int b = tid * kScanItems + i;
      int n = 0;
      if (b < B) n = max(0, checked_ctx_len(cache, b, capacity, kKIndexFull, blockIdx.x == 0));
      items[i] = (n + kUnit - 1) / kUnit;
    }
    int total;
    Scan(scan_tmp).ExclusiveSum(items, items, total);
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
      mbar_init(&S.empty[s], 1);
    }
    for (int a = 0; a < kAcc; ++a) {
      mbar_init(&S.acc_full[a], kIssuers);
      mbar_init(&S.acc_empty[a], 4);
    }
    for (int k = 0; k < kQBufs; ++k) mbar_init(&S.q_full[k], 4);
    for (int k = 0; k < kIssuers; ++k) mbar_init(&S.drain[k], 1);
    S.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) tma_prefetch_map(&code_map);
  // query scale blocks: the lines' bytes 4..15 (heads 32..127) stay zero
  for (int i = tid; i < kQBufs * kTileScaleBytes / 4; i += kThreads) reinterpret_cast<uint32_t*>(S.qscales)[i] = 0u;
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
  int hist_b0 = 0;
  {
    TileIter first;
    first.init(S.prefix, B, t_begin);
    hist_b0 = first.b;
  }
  const bool hist_smem = n_tiles < 2048;

  if (n_tiles > 0) {
    if (warp == 0 || warp == 3) {
      // ================= producers (warps 0, 3) =================
      // Each copies every other unit (the stages alternate with them: an even
      // number of stages), from cache rows its warp resolved 32 units at a
      // time (one unit per lane, the next 32 units' page-table loads in flight
      // while lane 0 issues).
      const int pr = warp == 0 ? 0 : 1;
      const uint64_t policy = l2_policy_evict_first();
      UnitRows next;   // this lane's unit of the next 32
      next.fetch(cache, S.prefix, B, t_begin + pr + 2 * lane, pr + 2 * lane < n_tiles, capacity, page_size);
      int issued = 0;   // lane 0: own units
      bool stop = false;
      for (int i0 = 0; i0 < n_tiles && !stop; i0 += 64) {
        int r[2];
        next.rows(cache, capacity, kKIndexFull, r);
        S.rowq[pr][lane][0] = r[0];
        S.rowq[pr][lane][1] = r[1];
        const int g1 = i0 + 64 + pr + 2 * lane;
        next.fetch(cache, S.prefix, B, t_begin + g1, g1 < n_tiles, capacity, page_size);
        __syncwarp();
        if (lane == 0) {
          for (int k = 0; k < 32; ++k) {
            const int i = i0 + pr + 2 * k, s = i % kStages;
            if (i >= n_tiles) break;
            if (!mbar_wait(&S.empty[s], ((i / kStages) & 1) ^ 1, wait_ns)) {
              report_error(cache.err_word, CSA2_ERR_TIMEOUT, kKIndexFull, -1, i);
              S.abort_flag = 1;
            }
            if (S.abort_flag) {
              stop = true;
              break;
            }
            const int r0 = S.rowq[pr][k][0], r1 = S.rowq[pr][k][1];
            // a tile's scale block is 1 KB at (row / 128) KB: 16-byte aligned
            if (whole_units && r0 >= 0) {   // the unit's 256 rows and two scale blocks are consecutive
              mbar_arrive_expect_tx(&S.full[s], 2 * (kTileCodeBytes + kTileScaleBytes));
              tma_load_2d(S.tiles[s][0], &code_map, &S.full[s], 0, r0, policy);
              bulk_load_1d(S.scales[s][0], ik4_scales + static_cast<long long>(r0 / kTile) * kTileScaleBytes,
                           2 * kTileScaleBytes, &S.full[s], policy);
            } else {
              mbar_arrive_expect_tx(&S.full[s], ((r0 >= 0) + (r1 >= 0)) * (kTileCodeBytes + kTileScaleBytes));
              for (int h = 0; h < 2; ++h) {
                const int rh = h == 0 ? r0 : r1;
                if (rh < 0) continue;
                tma_load_2d(S.tiles[s][h], &code_map, &S.full[s], 0, rh, policy);
                bulk_load_1d(S.scales[s][h], ik4_scales + static_cast<long long>(rh / kTile) * kTileScaleBytes,
                             kTileScaleBytes, &S.full[s], policy);
              }
            }
            ++issued;
          }
        }
        stop = __shfl_sync(0xffffffffu, stop, 0);
        __syncwarp();
      }
      if (lane == 0) {
        // copies still in flight (only after an abort): wait for the last one of each own stage
        for (int m = issued > kStages / 2 ? issued - kStages / 2 : 0; m < issued; ++m) {
          const int i = pr + 2 * m;
          (void)mbar_wait(&S.full[i % kStages], (i / kStages) & 1, kWaitLimitNs / 2);
        }
      }
    } else if (warp < kEpiWarp0) {
      // ================= MMA issuers (lane 0 of warps 1, 2) =================
      // A tensor-core instruction (MMA, scale copy or commit) costs its issuing
      // thread tens of cycles whatever its size, and one thread issuing a
      // unit's ten set the scan's pace: each of two threads issues one
      // 128-row tile of every unit (two scale copies, two MMAs, one commit to
      // the accumulator barrier, which completes on both).  Both walk the same
      // units and segments and keep their own copy of the query's scales in
      // tensor memory.  The issue loop of the FP8 scan otherwise: descriptors
      // from one base, the query's only when the request changes, a unit
      // count instead of the walker.
      if (lane == 0) {
        const int h = warp - 1;   // this thread's tile of every unit
        TileIter it;
        it.init(S.prefix, B, t_begin);
        int seg = 0, cur_b = it.b;
        int left = S.prefix[cur_b + 1] - S.prefix[cur_b] - it.j;
        const uint32_t sfb0 = tmem + kSfbCol + h * (kQBufs * 8);
        bool ok = mbar_wait(&S.q_full[0], 0, wait_ns);
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int kh = 0; kh < 2; ++kh) tmem_cp_scales(sfb0 + kh * 4, smem_u32(S.qscales[0] + kh * 512));
        }
        const uint64_t adesc0 = sw64_kmajor_desc(smem_u32(S.tiles[0][h]));
        const uint32_t scales0 = smem_u32(S.scales[0][h]);
        uint64_t bdesc = sw64_kmajor_desc(smem_u32(S.q[0]));
        uint32_t sfb = sfb0;
        int s = 0, a = 0;
        uint32_t ph_s = 0, ph_a = 0;
        for (int i = 0; ok && i < n_tiles; ++i) {
          if (left == 0) {
            cur_b = next_request_with_tiles(S.prefix, B, cur_b);
            left = S.prefix[cur_b + 1] - S.prefix[cur_b];
            ++seg;
            if (!mbar_wait(&S.q_full[seg % kQBufs], (seg / kQBufs) & 1, wait_ns)) { ok = false; break; }
            tc_fence_after();
            sfb = sfb0 + (seg % kQBufs) * 8;
#pragma unroll
            for (int kh = 0; kh < 2; ++kh)
              tmem_cp_scales(sfb + kh * 4, smem_u32(S.qscales[seg % kQBufs] + kh * 512));
            bdesc = sw64_kmajor_desc(smem_u32(S.q[seg % kQBufs]));
          }
          --left;
          if (!mbar_wait(&S.acc_empty[a], ph_a ^ 1, wait_ns) || !mbar_wait(&S.full[s], ph_s, wait_ns)) {
            ok = false;
            break;
          }
          if (S.abort_flag) break;
          tc_fence_after();
          const uint32_t sfa = tmem + kSfaCol + (2 * a + h) * 8;
          const uint32_t sc = scales0 + static_cast<uint32_t>(s * 2 * kTileScaleBytes);
#pragma unroll
          for (int kh = 0; kh < 2; ++kh) tmem_cp_scales(sfa + kh * 4, sc + kh * 512);
          // start-address field: bits 0..13 of the descriptor (address / 16)
          const uint64_t adesc = adesc0 + static_cast<uint64_t>((s * 2 * kTileCodeBytes) >> 4);
#pragma unroll
          for (int kh = 0; kh < 2; ++kh)
            umma_mxf4nvf4(tmem + (2 * a + h) * kAccCols, adesc + 2 * kh, bdesc + 2 * kh, kIdesc, sfa + kh * 4,
                          sfb + kh * 4, kh > 0 ? 1u : 0u);
          umma_commit(&S.acc_full[a]);   // the epilogue releases the stage once both tiles' MMAs are done
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
        umma_commit(&S.drain[h]);
        (void)mbar_wait(&S.drain[h], 0, kWaitLimitNs);
      }
    } else {
      // ================= epilogue groups (warps 4..7, 8..11) =================
      const int group = (warp - kEpiWarp0) >> 2;
      const int ew = (warp - kEpiWarp0) & 3;
      const int quarter = warp & 3;
      const int toff = quarter * 32 + lane;
      auto timed_out = [&](int where) {
        if (lane == 0) {
          report_error(cache.err_word, CSA2_ERR_TIMEOUT, kKIndexFull, -1, where);
          S.abort_flag = 1;
        }
      };
      // query buffers: the protocol of the FP8 scan (segment x in buffer x % 3,
      // kept at most two segments ahead of group 0's current one)
      int prep_b = 0, prep_x = 0;
      auto prepare = [&]() {
        prepare_query_fp4(q + static_cast<long long>(prep_b) * kIndexHeads * kIndexDim, S.q[prep_x % kQBufs],
                          S.qscales[prep_x % kQBufs], 0, ew, lane);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.q_full[prep_x % kQBufs]);
        prep_b = next_request_with_tiles(S.prefix, B, prep_b);
        ++prep_x;
      };
      // This group's units: a counter walk over (request, unit) two units at
      // a time; `seg` counts the request segments passed.
      TileIter it;
      it.init(S.prefix, B, t_begin);
      int seg = 0, cur_b = it.b, j = it.j;
      int units_b = S.prefix[cur_b + 1] - S.prefix[cur_b];
      auto step = [&](int d) {
        j += d;
        while (j >= units_b) {
          j -= units_b;
          cur_b = next_request_with_tiles(S.prefix, B, cur_b);
          if (cur_b >= B) break;   // past this CTA's last unit
          units_b = S.prefix[cur_b + 1] - S.prefix[cur_b];
          ++seg;
        }
      };
      if (group == 0) {
        prep_b = cur_b;
        for (int k = 0; k < kQBufs && prep_b < B && S.prefix[prep_b] < t_end; ++k) prepare();
      }
      float ws[32];
      auto load_w = [&](int b) {
        const float wl = w[static_cast<long long>(b) * kIndexHeads + lane];
#pragma unroll
        for (int h = 0; h < 32; ++h) ws[h] = __shfl_sync(0xffffffffu, wl, h);
      };
      if (group == 1) step(1);
      int w_b = -1, nb = 0;   // the request whose weights and length are loaded

      for (int i = group; i < n_tiles; i += kEpiGroups) {
        if (cur_b != w_b) {
          w_b = cur_b;
          load_w(cur_b);
          nb = cache.ctx_len[cur_b];
        }
        const int a = i % kAcc;
        if (!mbar_wait_warp(&S.acc_full[a], (i / kAcc) & 1, wait_ns)) {
          timed_out(j);
          break;
        }
        // both tiles' MMAs (and scale copies) are complete: the stage is free
        if (ew == 0 && lane == 0) mbar_arrive(&S.empty[i % kStages]);
        tc_fence_after();
        uint32_t acc0[32], acc1[32];
        tmem_ld_32x32b_x32(tmem + (2 * a) * kAccCols + (static_cast<uint32_t>(quarter * 32) << 16), acc0);
        tmem_ld_32x32b_x32(tmem + (2 * a + 1) * kAccCols + (static_cast<uint32_t>(quarter * 32) << 16), acc1);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.acc_empty[a]);
        // Group 0 writes the codes of up to two segments ahead only after this
        // unit's accumulator: the buffer it reuses held the previous segment,
        // whose last unit may be group 1's and issued after group 0's previous
        // accumulator.
        if (group == 0)
          while (prep_x <= seg + 2 && prep_b < B && S.prefix[prep_b] < t_end) prepare();

        // both tiles' sums side by side (each in head order, as the re-score)
        float sc[2] = {0.0f, 0.0f};
#pragma unroll
        for (int hh = 0; hh < 32; ++hh) {
          sc[0] = fmaf(ws[hh], fmaxf(__uint_as_float(acc0[hh]), 0.0f), sc[0]);
          sc[1] = fmaf(ws[hh], fmaxf(__uint_as_float(acc1[hh]), 0.0f), sc[1]);
        }
        const int p0 = j * kUnit + toff;
        float bm[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) bm[h] = p0 + h * kTile < nb ? sc[h] : -INFINITY;
#pragma unroll
        for (int d = 1; d < 8; d <<= 1) {
          const float o0 = __shfl_xor_sync(0xffffffffu, bm[0], d);
          const float o1 = __shfl_xor_sync(0xffffffffu, bm[1], d);
          bm[0] = fmaxf(bm[0], o0);
          bm[1] = fmaxf(bm[1], o1);
        }
        if ((lane & 7) == 0) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int p = p0 + h * kTile;
            if (p >= nb) continue;
            blockmax[static_cast<long long>(cur_b) * (capacity / kBlock) + p / kBlock] = bm[h];
            if (hist != nullptr) {
              const uint32_t bin = order_key(bm[h]) >> (32 - kPoolHistBits);
              const int slot = cur_b - hist_b0;
              if (hist_smem && slot < 2) atomicAdd(&S.hist[slot][bin >> 1], 1u << (16 * (bin & 1)));
              else atomicAdd(&hist[static_cast<long long>(cur_b) * kPoolHistBins + bin], 1u);
            }
          }
        }
        if (scores != nullptr) {
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (p0 + h * kTile < nb) scores[static_cast<long long>(cur_b) * capacity + p0 + h * kTile] = sc[h];
        }
        // another role's time-out (every 8th unit: the waits above are bounded anyway)
        if ((i & (8 * kEpiGroups - 1)) < kEpiGroups && warp_flag(&S.abort_flag)) break;
        step(kEpiGroups);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (hist != nullptr && hist_smem) {
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

// Quantise-on-append of FP4 indexer keys: one warp per row.
__global__ void __launch_bounds__(256) append_ik4_kernel(csa2_cache cache, uint8_t* __restrict__ codes,
                                                         uint8_t* __restrict__ scales, int n_rows,
                                                         const float* __restrict__ ik_new,
                                                         const int32_t* __restrict__ req,
                                                         const int32_t* __restrict__ pos) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n_rows) return;
  const int b = req ? req[warp] : warp, t = pos[warp];
  const long long capacity = static_cast<long long>(cache.max_pages_per_req) * cache.page_size;
  if (b < 0 || b >= cache.batch || t < 0 || t >= capacity) {
    if (lane == 0) report_error(cache.err_word, CSA2_ERR_DEVICE_BOUNDS, kKAppend, b, t);
    return;
  }
  const int page = cache.page_table[static_cast<long long>(b) * cache.max_pages_per_req + t / cache.page_size];
  if (page < 0 || page >= cache.num_pages) {
    if (lane == 0) report_error(cache.err_word, CSA2_ERR_DEVICE_BOUNDS, kKAppend, b, t);
    return;
  }
  const long long row = static_cast<long long>(page) * cache.page_size + t % cache.page_size;
  const float4 v = reinterpret_cast<const float4*>(ik_new + static_cast<long long>(warp) * kIndexDim)[lane];
  uint32_t sc;
  const uint32_t c = fp4_row_lane(v, &sc);
  reinterpret_cast<uint16_t*>(codes + row * kCodeBytes)[lane] = static_cast<uint16_t>(c);
  if ((lane & 3) == 0)
    scales[(row / kTile) * kTileScaleBytes + block_scale_offset(static_cast<uint32_t>(row % kTile), lane >> 2)] =
        static_cast<uint8_t>(sc);
}

}  // namespace

static_assert(kStages % kProducers == 0, "each producer keeps to its own stages");
static_assert(sizeof(Fp4Smem) + 1024 <= 225 * 1024, "the FP4 scan's shared memory (plus the prefix sum's) exceeds one SM");
static_assert(kSfbCol + kIssuers * kQBufs * 8 <= kTmemCols, "the FP4 scan's tensor-memory columns");
size_t index_full_fp4_smem_bytes() { return sizeof(Fp4Smem) + 1024; }

cudaError_t launch_index_full_fp4(const csa2_cache& cache, const uint8_t* ik4_scales, const float* q, const float* w,
                                  float* blockmax, float* scores, uint32_t* hist, const CUtensorMap& code_map,
                                  int whole_units, int num_sms, uint64_t wait_ns, cudaStream_t stream) {
  static ContextMemo attrs;
  const size_t smem = index_full_fp4_smem_bytes();
  const cudaError_t e = attrs.once([&] {
    return cudaFuncSetAttribute(index_full_fp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(smem));
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
  return cudaLaunchKernelEx(&cfg, index_full_fp4_kernel, cache, ik4_scales, q, w, blockmax, scores, hist, code_map,
                            whole_units, wait_ns);
}

cudaError_t launch_append_ik4(const csa2_cache& cache, uint8_t* codes, uint8_t* scales, int n_rows,
                              const float* ik_new, const int32_t* req, const int32_t* pos, cudaStream_t stream) {
  const int threads = 256;
  const long long blocks = (static_cast<long long>(n_rows) * 32 + threads - 1) / threads;
  append_ik4_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(cache, codes, scales, n_rows, ik_new, req,
                                                                          pos);
  return cudaGetLastError();
}

}  // namespace csa2
