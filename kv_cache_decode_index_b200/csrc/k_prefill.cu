// Causal prefill indexer: for many queries of one request at once, the Top-k
// visible entries by the Full-mode indexer score, with no pool.  On the pages
// this is the encoder group (1 Full + 5 Reuse layers over a sequence
// compressed m = 2: two tokens per entry) [4sapi blog, section 三; indexer
// shape and Top-512, same blog, section 四].  The causal rule on compressed
// indices (entry e covers tokens m*e .. m*e + m - 1 and is visible at token p
// iff m*e + m - 1 <= p) is a reading: the pages state none.
//
// The score matrix (queries x entries) is an FP8 GEMM, n*32 x 128 by
// 128 x entries, followed by a per-query reduction over the 32 heads.  Design
// (sm_100a):
//   * one CTA per 8 queries; their codes form the B operand (N = 256 =
//     8 queries x 32 heads, 32 KB, resident for the CTA's lifetime);
//   * warp 0 (one lane): TMA producer of 128-entry indexer-K tiles (16 KB)
//     into a kPStages ring, and of the tiles' exponent bytes (1-D bulk copy,
//     128 B) into a ring of their own that the epilogue releases; both read
//     with an L2 evict_last hint (every CTA reads the same keys);
//   * warp 1 (one lane): tcgen05.mma kind::f8f6f4, M = 128 entries, N = 256,
//     K = 128 in 4 steps, into one of two 256-column TMEM accumulators;
//   * warps 2..17: epilogue.  Warp e reads TMEM lane quarter (warp % 4) for
//     the two queries 2*(e/4), 2*(e/4)+1: 32 fp32 head dot products per (entry,
//     query), all 64 columns loaded before the accumulator is handed back ->
//     score (ReLU split between the min/max and FMA units, four fp32 FMA
//     chains per query) ->
//     filter against the query's running threshold theta.  Survivors are
//     appended to the query's candidate list in the caller's workspace.  When
//     any list nears its capacity, epilogue warp j compacts the list of query
//     j to the exact k best (warp radix select) and raises its theta, all at
//     the same tile.  Entries arrive in increasing order, so an entry whose
//     key does not exceed theta can never enter the Top-k.
// A second kernel reduces every list to the exact Top-k, sorted ascending.
// Every mbarrier wait is bounded; a wait that runs out records
// CSA2_ERR_TIMEOUT and every role leaves its loop (the epilogue warps leave
// together, decided at their per-tile barrier), drains, frees TMEM and
// returns.
#include <mutex>

#include "index_common.cuh"
#include "launch.h"
#include "warp_select.cuh"

namespace csa2 {

namespace {

constexpr int kPQ = 8;                                 // queries per CTA
constexpr int kPN = kPQ * kIndexHeads;                 // 256: MMA N
constexpr int kPStages = 6;
constexpr int kPExp = 8;                               // exponent-byte ring (slots of 128 B)
constexpr int kPAcc = 2;                               // accumulators of kPN columns
constexpr int kQPW = 2;                                // queries per epilogue warp and tile
constexpr int kPEpiWarps = 4 * kPQ / kQPW;             // 16: four TMEM lane quarters per query group
constexpr int kPThreads = 64 + kPEpiWarps * 32;        // 576
constexpr uint32_t kPTmemCols = kPAcc * kPN;           // 512
constexpr uint32_t kPIdesc = idesc_e4m3_f32(kTile, kPN);
constexpr int kCand = CSA2_PREFILL_CANDIDATES;         // list capacity per query
constexpr int kBarEvery = 8;                           // tiles between the epilogue's barriers
constexpr int kHigh = kCand - kBarEvery * kTile;       // compaction trigger
constexpr int kBarAll = 1;                             // named barrier: all epilogue warps
constexpr int kBarTile = 2;                            // per-tile barrier of the epilogue warps
static_assert(kCand % 4 == 0 && kCand >= 2 * CSA2_PREFILL_MAX_K + 2 * kTile, "candidate capacity");
// a list compacted to k is below the trigger, and one below the trigger has
// room for the kBarEvery tiles until the next check
static_assert(kHigh > CSA2_PREFILL_MAX_K && kHigh + kBarEvery * kTile <= kCand, "compaction trigger");

struct __align__(1024) PrefillSmem {
  uint8_t tiles[kPStages][kTileBytes];
  uint8_t q[kPN * kIndexDim];          // B operand: row 32*j + h = head h of query j
  uint8_t exps[kPExp][kTile];          // exponent bytes of the tiles in flight
  float ws[kPQ][kIndexHeads];          // w_h * sigma^q_h
  uint32_t hist[kPQ][256];             // radix histograms of the compactions
  int vis[kPQ];                        // visible entries of each query
  int cnt[kPQ];                        // list lengths
  uint32_t theta[kPQ];                 // admission thresholds (order keys)
  int epi_abort;                       // the epilogue leaves its loop
  uint64_t full[kPStages];
  uint64_t empty[kPStages];
  uint64_t acc_full[kPAcc];
  uint64_t acc_empty[kPAcc];
  uint64_t exp_full[kPExp];
  uint64_t exp_empty[kPExp];
  uint64_t q_full;
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort_flag;
};

struct Workspace {
  uint32_t* key;   // [n][kCand] order keys
  int32_t* pos;    // [n][kCand] entries
  int32_t* cnt;    // [n] list lengths
};

__host__ __device__ inline Workspace split_workspace(void* ws, long long n) {
  uint8_t* p = static_cast<uint8_t*>(ws);
  Workspace w;
  w.key = reinterpret_cast<uint32_t*>(p);
  w.pos = reinterpret_cast<int32_t*>(p + static_cast<size_t>(n) * kCand * 4);
  w.cnt = reinterpret_cast<int32_t*>(p + static_cast<size_t>(n) * kCand * 8);
  return w;
}

__global__ void __launch_bounds__(kPThreads, 1)
    prefill_scan_kernel(const csa2_cache cache, int req, int n_queries, const int32_t* __restrict__ q_pos, int ratio,
                        const float* __restrict__ q, const float* __restrict__ w, int k, Workspace wsp,
                        const __grid_constant__ CUtensorMap ik_map, uint64_t wait_ns) {
  extern __shared__ uint8_t smem_raw[];
  PrefillSmem& S =
      *reinterpret_cast<PrefillSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int j0 = blockIdx.x * kPQ;
  const long long capacity = static_cast<long long>(cache.max_pages_per_req) * cache.page_size;
  const uint32_t page_size = static_cast<uint32_t>(cache.page_size);
  const int32_t* ptab = cache.page_table + static_cast<long long>(req) * cache.max_pages_per_req;

  if (tid < kPQ) {
    const int j = j0 + tid;
    long long v = 0;
    if (j < n_queries) {
      const long long p = q_pos[j];
      v = p < 0 ? 0 : (p + 1) / ratio;
      const long long n = max(0, checked_ctx_len(cache, req, capacity, kKPrefill, blockIdx.x == 0 && tid == 0));
      v = v < n ? v : n;
    }
    S.vis[tid] = static_cast<int>(v);
    S.cnt[tid] = 0;
    S.theta[tid] = 0u;   // every order key is >= 1
  }
  if (tid == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    for (int a = 0; a < kPAcc; ++a) {
      mbar_init(&S.acc_full[a], 1);
      mbar_init(&S.acc_empty[a], kPEpiWarps);
    }
    for (int x = 0; x < kPExp; ++x) {
      mbar_init(&S.exp_full[x], 1);
      mbar_init(&S.exp_empty[x], kPEpiWarps);
    }
    mbar_init(&S.q_full, kPEpiWarps);
    mbar_init(&S.drain, 1);
    S.epi_abort = 0;
    S.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, kPTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) tma_prefetch_map(&ik_map);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  int vmax = 0;
#pragma unroll
  for (int t = 0; t < kPQ; ++t) vmax = max(vmax, S.vis[t]);
  const int n_tiles = (vmax + kTile - 1) / kTile;
  const uint32_t tmem = S.tmem_base;

  if (warp == 0) {
    // ================= producer =================
    if (lane == 0 && n_tiles > 0) {
      const uint64_t policy = l2_policy_evict_last();
      int issued = 0, page_idx = -1, page = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % kPStages, x = i % kPExp;
        if (!mbar_wait(&S.empty[s], ((i / kPStages) & 1) ^ 1, wait_ns) ||
            !mbar_wait(&S.exp_empty[x], ((i / kPExp) & 1) ^ 1, wait_ns)) {
          report_error(cache.err_word, CSA2_ERR_TIMEOUT, kKPrefill, req, i);
          S.abort_flag = 1;
          break;
        }
        if (S.abort_flag) break;
        const int p0 = i * kTile;   // < vmax <= capacity < 2^31
        const int pidx = static_cast<int>(static_cast<uint32_t>(p0) / page_size);
        if (pidx != page_idx) {
          page_idx = pidx;
          page = ptab[pidx];
          if (page < 0 || page >= cache.num_pages) {
            report_error(cache.err_word, CSA2_ERR_DEVICE_BOUNDS, kKPrefill, req, p0);
            page = 0;   // load a valid page; the call's outputs are flagged invalid
          }
        }
        const int row = page * cache.page_size + (p0 - pidx * cache.page_size);
        mbar_arrive_expect_tx(&S.full[s], kTileBytes);
        tma_load_2d(S.tiles[s], &ik_map, &S.full[s], 0, row, policy);
        // the tile's 128 exponent bytes: 128-byte aligned (row is a multiple of 128)
        mbar_arrive_expect_tx(&S.exp_full[x], kTile);
        bulk_load_1d(S.exps[x], cache.ik_exp + row, kTile, &S.exp_full[x], policy);
        ++issued;
      }
      // copies still in flight (only after an abort)
      for (int i = issued > kPStages ? issued - kPStages : 0; i < issued; ++i)
        (void)mbar_wait(&S.full[i % kPStages], (i / kPStages) & 1, kWaitLimitNs / 2);
      for (int i = issued > kPExp ? issued - kPExp : 0; i < issued; ++i)
        (void)mbar_wait(&S.exp_full[i % kPExp], (i / kPExp) & 1, kWaitLimitNs / 2);
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0 && n_tiles > 0) {
      bool ok = mbar_wait(&S.q_full, 0, wait_ns);
      const uint64_t bdesc = sw128_kmajor_desc(smem_u32(S.q));
      for (int i = 0; ok && i < n_tiles; ++i) {
        const int s = i % kPStages, a = i % kPAcc;
        if (!mbar_wait(&S.acc_empty[a], ((i / kPAcc) & 1) ^ 1, wait_ns) ||
            !mbar_wait(&S.full[s], (i / kPStages) & 1, wait_ns)) {
          ok = false;
          break;
        }
        if (S.abort_flag) break;
        tc_fence_after();
        const uint64_t adesc = sw128_kmajor_desc(smem_u32(S.tiles[s]));
#pragma unroll
        for (int kk = 0; kk < kIndexDim / 32; ++kk)
          umma_f8f6f4(tmem + a * kPN, adesc + 2 * kk, bdesc + 2 * kk, kPIdesc, kk > 0 ? 1u : 0u);
        umma_commit(&S.empty[s]);
        umma_commit(&S.acc_full[a]);
      }
      if (!ok) {
        report_error(cache.err_word, CSA2_ERR_TIMEOUT, kKPrefill, req, -1);
        S.abort_flag = 1;
      }
      umma_commit(&S.drain);
      (void)mbar_wait(&S.drain, 0, kWaitLimitNs);
    }
  } else {
    // ================= epilogue (warps 2..9) =================
    const int e = warp - 2;
    const int grp = e >> 2;                    // queries kQPW*grp .. kQPW*grp + kQPW - 1
    const int own = e;                         // the query whose list this warp compacts (e < kPQ)
    const int quarter = warp & 3;              // TMEM lane quarter
    const int toff = quarter * 32 + lane;      // entry inside the tile

    // Query codes -> B operand rows 32*j + h; each warp quantises
    // 4*kPQ/kPEpiWarps groups of 8 heads.
    {
      constexpr int kParts = 4 * kPQ / kPEpiWarps;
      for (int c = 0; c < kParts; ++c) {
        const int part = e * kParts + c, jq = part >> 2, ew = part & 3;
        const int j = j0 + jq;
        uint8_t* qt = S.q + jq * kIndexHeads * kIndexDim;
        if (j < n_queries) {
          prepare_query_part(q + static_cast<long long>(j) * kIndexHeads * kIndexDim,
                             w + static_cast<long long>(j) * kIndexHeads, qt, S.ws[jq], ew, lane);
        } else {
#pragma unroll
          for (int hh = 0; hh < 8; ++hh) *reinterpret_cast<uint32_t*>(qt + sw128_offset(ew * 8 + hh, 4u * lane)) = 0u;
          if (lane < 8) S.ws[jq][ew * 8 + lane] = 0.0f;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.q_full);
    }
    named_bar_sync(kBarAll, kPEpiWarps * 32);   // ws of all queries written

    int vis_r[kQPW];
    uint32_t theta_r[kQPW];
#pragma unroll
    for (int t = 0; t < kQPW; ++t) {
      vis_r[t] = S.vis[grp * kQPW + t];
      theta_r[t] = 0u;
    }
    const float kDown = exp2i(-25), kUp = exp2i(25);

    bool failed = false, crossed = false;
    for (int i = 0; i < n_tiles; ++i) {
      const int a = i % kPAcc, x = i % kPExp;
      if (!failed) failed = warp_flag(&S.abort_flag);
      if (!failed && (!mbar_wait_warp_backoff(&S.acc_full[a], (i / kPAcc) & 1, wait_ns) ||
                      !mbar_wait_warp(&S.exp_full[x], (i / kPExp) & 1, wait_ns))) {
        failed = true;
        if (lane == 0) report_error(cache.err_word, CSA2_ERR_TIMEOUT, kKPrefill, req, i);
      }
      if (!failed) {
        // All 128 columns of this warp's four queries at once; the
        // accumulator is handed back to the MMA before the arithmetic.
        tc_fence_after();
        const uint32_t tbase =
            tmem + a * kPN + (static_cast<uint32_t>(quarter * 32) << 16) + grp * kQPW * kIndexHeads;
        uint32_t acc[kQPW][32];
#pragma unroll
        for (int t = 0; t < kQPW; ++t) tmem_ld_32x32b_x32(tbase + t * kIndexHeads, acc[t]);
        tmem_ld_wait();
        const uint32_t ex = S.exps[x][toff];
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&S.acc_empty[a]);
          mbar_arrive(&S.exp_empty[x]);
        }
        const float sigma = exp2i(static_cast<int>(ex) - 127);
        const int p = i * kTile + toff;
        // Two queries at a time, each summed in four scalar FMA chains.
#pragma unroll
        for (int t0 = 0; t0 < kQPW; t0 += 2) {
          float sc[2][4];
#pragma unroll
          for (int u = 0; u < 2; ++u) sc[u][0] = sc[u][1] = sc[u][2] = sc[u][3] = 0.0f;
#pragma unroll
          for (int h = 0; h < 8; ++h) {
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              // sum_h ws_h ReLU(acc_h): even heads take ReLU on the FP
              // min/max unit, odd heads on the FMA unit as a saturating
              // multiply by 2^-25 (|acc| < 2^25, so that is ReLU(acc) * 2^-25
              // exactly); the odd sums are scaled back by 2^25 at the end.
              const uint32_t(&ac)[32] = acc[t0 + u];
              const float4 c = reinterpret_cast<const float4*>(S.ws[grp * kQPW + t0 + u])[h];
              float r1, r3;
              asm("mul.rn.sat.f32 %0, %1, %2;" : "=f"(r1) : "f"(__uint_as_float(ac[4 * h + 1])), "f"(kDown));
              asm("mul.rn.sat.f32 %0, %1, %2;" : "=f"(r3) : "f"(__uint_as_float(ac[4 * h + 3])), "f"(kDown));
              sc[u][0] = fmaf(c.x, fmaxf(__uint_as_float(ac[4 * h]), 0.0f), sc[u][0]);
              sc[u][1] = fmaf(c.y, r1, sc[u][1]);
              sc[u][2] = fmaf(c.z, fmaxf(__uint_as_float(ac[4 * h + 2]), 0.0f), sc[u][2]);
              sc[u][3] = fmaf(c.w, r3, sc[u][3]);
            }
          }
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int t = t0 + u;
            const int jl = grp * kQPW + t;
            const float even = sc[u][0] + sc[u][2], odd = sc[u][1] + sc[u][3];
            const uint32_t key = order_key(fmaf(odd, kUp, even) * sigma);
            const bool admit = p < vis_r[t] && key > theta_r[t];
            const uint32_t m = __ballot_sync(0xffffffffu, admit);
            if (m != 0u) {
              int base = 0;
              if (lane == 0) base = atomicAdd(&S.cnt[jl], __popc(m));
              base = __shfl_sync(0xffffffffu, base, 0);
              if (admit) {
                const int idx = base + __popc(m & lanemask_lt());
                const size_t at = static_cast<size_t>(j0 + jl) * kCand + idx;
                wsp.key[at] = key;
                wsp.pos[at] = p;
                crossed |= idx >= kHigh;
              }
            }
          }
        }
      }
      if (failed && lane == 0) {
        S.epi_abort = 1;
        S.abort_flag = 1;
      }
      // A barrier of all epilogue warps every kBarEvery tiles: leave
      // together, or, when any list may lack room for the next kBarEvery
      // tiles, compact every list to its k best at once (one stall per round
      // instead of one per list).
      if ((i % kBarEvery != kBarEvery - 1 && i != n_tiles - 1) ||
          !named_bar_or(kBarTile, kPEpiWarps * 32, crossed || failed))
        continue;
      {
        if (*reinterpret_cast<volatile int*>(&S.epi_abort)) break;
        const int n = own < kPQ ? *reinterpret_cast<volatile int*>(&S.cnt[own]) : 0;
        if (n > k) {
          const size_t at = static_cast<size_t>(j0 + own) * kCand;
          uint32_t th = 0u;
          const int kept = warp_compact_topk(wsp.key + at, wsp.pos + at, n, k, S.hist[own], lane, &th);
          if (lane == 0) {
            S.cnt[own] = kept;
            S.theta[own] = max(S.theta[own], th);
          }
        }
        named_bar_sync(kBarTile, kPEpiWarps * 32);
#pragma unroll
        for (int t = 0; t < kQPW; ++t) theta_r[t] = *reinterpret_cast<volatile uint32_t*>(&S.theta[grp * kQPW + t]);
        crossed = false;
      }
    }
    if (lane == 0 && own < kPQ && j0 + own < n_queries)
      wsp.cnt[j0 + own] = *reinterpret_cast<volatile int*>(&S.cnt[own]);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kPTmemCols);
  }
}

// Per query (one warp): the exact k best of its list, sorted ascending and
// padded with -1.
constexpr int kSelWarps = 4;
constexpr int kSortMax = CSA2_PREFILL_MAX_K;

__global__ void __launch_bounds__(kSelWarps * 32)
    prefill_select_kernel(int n_queries, int k, Workspace wsp, int32_t* __restrict__ topk) {
  __shared__ uint32_t hist[kSelWarps][256];
  __shared__ int32_t sortbuf[kSelWarps][kSortMax];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * kSelWarps + warp;
  if (j >= n_queries) return;
  const size_t at = static_cast<size_t>(j) * kCand;
  int n = wsp.cnt[j];
  n = n < 0 ? 0 : (n > kCand ? kCand : n);
  uint32_t th = 0u;
  n = warp_compact_topk(wsp.key + at, wsp.pos + at, n, k, hist[warp], lane, &th);
  int P = 32;
  while (P < n) P <<= 1;
  int32_t* sb = sortbuf[warp];
  for (int i = lane; i < P; i += 32) sb[i] = i < n ? wsp.pos[at + i] : 0x7fffffff;
  __syncwarp();
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = lane; t < P / 2; t += 32) {
        const int lo = (t / stride) * stride * 2 + (t % stride);
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const int32_t x = sb[lo], y = sb[hi];
        if ((x > y) == up) {
          sb[lo] = y;
          sb[hi] = x;
        }
      }
      __syncwarp();
    }
  }
  int32_t* out = topk + static_cast<size_t>(j) * k;
  for (int i = lane; i < k; i += 32) out[i] = i < n ? sb[i] : -1;
}

}  // namespace

size_t prefill_workspace_bytes(long long n_queries) {
  if (n_queries <= 0) return 0;
  return static_cast<size_t>(n_queries) * kCand * 8 + ((static_cast<size_t>(n_queries) * 4 + 15) & ~size_t(15));
}

cudaError_t launch_prefill_index(const csa2_cache& cache, int req, int n_queries, const int32_t* q_pos, int ratio,
                                 const float* q, const float* w, int k, int32_t* topk, void* workspace,
                                 const CUtensorMap& ik_map, uint64_t wait_ns, cudaStream_t stream) {
  static ContextMemo attrs;
  const size_t smem = sizeof(PrefillSmem) + 1024;
  cudaError_t e = attrs.once([&] {
    return cudaFuncSetAttribute(prefill_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(smem));
  });
  if (e != cudaSuccess) return e;
  const Workspace wsp = split_workspace(workspace, n_queries);
  const int grid = (n_queries + kPQ - 1) / kPQ;
  prefill_scan_kernel<<<grid, kPThreads, smem, stream>>>(cache, req, n_queries, q_pos, ratio, q, w, k, wsp, ik_map,
                                                         wait_ns);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int sgrid = (n_queries + kSelWarps - 1) / kSelWarps;
  prefill_select_kernel<<<sgrid, kSelWarps * 32, 0, stream>>>(n_queries, k, wsp, topk);
  return cudaGetLastError();
}

// ------------------------------------------------- static-scratch variant ----
// Candidate lists of csa2_prefill_index_static: a file-scope device array
// sized for kStaticPrefillMaxQueries queries, so the call needs no
// caller-provided workspace.  Every call on a device uses the same array.
namespace {
constexpr long long kStaticPrefillBytes =
    static_cast<long long>(kStaticPrefillMaxQueries) * kCand * 8 + kStaticPrefillMaxQueries * 4;
__device__ __align__(256) uint8_t g_prefill_scratch[kStaticPrefillBytes];

// Its device address, looked up once per CUDA context (the module, and the
// array with it, is loaded again in a context that is created anew).
ContextMemo g_scratch_addr;
}  // namespace

cudaError_t static_prefill_scratch(void** addr) {
  return g_scratch_addr.get(addr, [](void** out) { return cudaGetSymbolAddress(out, g_prefill_scratch); });
}

}  // namespace csa2
