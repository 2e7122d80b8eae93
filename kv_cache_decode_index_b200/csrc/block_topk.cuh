// Exact top-K over the keys of one CTA of 1024 threads, held in registers.
//
// Thread t holds keys [t*ITEMS, (t+1)*ITEMS) (uint32, order-preserving,
// 0 = not a candidate); that index order decides ties (lower index first) and
// is the output order (ascending).  Radix select with 10-bit digits (one
// 1024-bin histogram in shared memory, one bin per thread for the digit
// search), starting either from the valid keys' common leading bits (count,
// min, max) or from a head start the caller found in a histogram of the keys.
// Then every thread counts its keys above / on the threshold prefix, two block
// prefix sums give each thread its first output rank, and the selected keys
// are emitted in index order.  No cluster, no global memory of its own.
#pragma once

#include "cluster_topk.cuh"

namespace csa2 {

constexpr int kBlockSelectThreads = 1024;

struct BlockSelectSmem {
  uint32_t hist[1024];
  int warp_tmp[64];
  uint32_t wstat[32][3];
  SelectStart start;   // a head start staged by the caller (optional)
  uint32_t prefix, mask;
  int need, hi, done;
};

// Head start of a top-K select from a histogram of the keys' leading `bits`
// bits, read by one block of THREADS threads: thread t holds NB consecutive
// bins, highest first (c[j] is bin top_bin - j), and ascending thread order is
// descending bin order.  `valid` is the number of valid keys.  Returns (in
// every thread) whether the histogram is consistent with it, i.e. holds
// exactly `valid` counts: a stale or foreign histogram makes the caller fall
// back to a select without head start, so it costs time, never correctness.
// The start is written to *out by the thread that finds it (read it after a
// barrier).
// With bin_count, the count of the threshold's bin is stored there too.
// With kLocalValid, `valid` is this thread's count of valid keys, summed over
// the block in the same prefix sum as the bins (warp_tmp: 2 * THREADS / 32).
template <int THREADS, int NB, bool kLocalValid = false>
__device__ bool hist_head_start(const uint32_t (&c)[NB], int top_bin, int bits, int valid, int K, int* warp_tmp,
                                SelectStart* out, int* bin_count = nullptr) {
  int sum = 0;
#pragma unroll
  for (int j = 0; j < NB; ++j) sum += static_cast<int>(c[j]);
  int total, above;
  if constexpr (kLocalValid) {
    int valid_total;
    above = block_exclusive_sum2<THREADS>(sum, valid, warp_tmp, &total, &valid_total).x;
    valid = valid_total;
  } else {
    above = block_exclusive_sum<THREADS>(sum, warp_tmp, &total);
  }
  if (total != valid) return false;
  if (valid <= K) {   // everything valid is selected
    if (threadIdx.x == 0) *out = SelectStart{0u, 0u, valid, -1, 1};
    return true;
  }
  if (above < K && K <= above + sum) {   // exactly one thread holds the threshold bin
    int a = above;
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      const int cj = static_cast<int>(c[j]);
      if (a < K && K <= a + cj) {
        const uint32_t T = static_cast<uint32_t>(top_bin - j);
        *out = SelectStart{T << (32 - bits), 0xFFFFFFFFu << (32 - bits), K - a, 31 - bits, cj == K - a ? 1 : 0};
        if (bin_count != nullptr) *bin_count = cj;
      }
      a += cj;
    }
  }
  return true;
}

// The radix passes of block_topk.  On return (after a barrier) S.prefix,
// S.mask and S.need describe the selection of the K best keys: every valid key
// whose masked bits exceed S.prefix, and the first S.need keys (by index)
// whose masked bits equal it.  start: optional head start (read after a
// barrier; may point into S.start), whose need replaces K.  Called by all
// 1024 threads.
template <int ITEMS>
__device__ void block_select_prefix(const uint32_t (&keys)[ITEMS], int K, BlockSelectSmem& S,
                                    const SelectStart* start) {
  constexpr int THREADS = kBlockSelectThreads;
  constexpr int kWarps = THREADS / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (start != nullptr) {
    __syncthreads();   // a head start staged in shared memory is complete
    if (tid == 0) {
      S.prefix = start->prefix;
      S.mask = start->mask;
      S.need = start->need;
      S.hi = start->hi;
      S.done = start->done;
    }
  } else {
    uint32_t cnt = 0, kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
    for (int i = 0; i < ITEMS; ++i) {
      const uint32_t k = keys[i];
      if (k != 0u) {
        ++cnt;
        kmin = min(kmin, k);
        kmax = max(kmax, k);
      }
    }
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) {
      S.wstat[warp][0] = cnt;
      S.wstat[warp][1] = kmin;
      S.wstat[warp][2] = kmax;
    }
    __syncthreads();
    if (warp == 0) {
      cnt = lane < kWarps ? S.wstat[lane][0] : 0u;
      kmin = lane < kWarps ? S.wstat[lane][1] : 0xFFFFFFFFu;
      kmax = lane < kWarps ? S.wstat[lane][2] : 0u;
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      kmin = __reduce_min_sync(0xffffffffu, kmin);
      kmax = __reduce_max_sync(0xffffffffu, kmax);
      if (lane == 0) {
        if (cnt <= static_cast<uint32_t>(K)) {   // everything valid is selected
          S.prefix = 0u;
          S.mask = 0u;
          S.need = static_cast<int>(cnt);
          S.done = 1;
        } else if (kmin == kmax) {                 // all valid keys tie: the first K by index
          S.prefix = kmin;
          S.mask = 0xFFFFFFFFu;
          S.need = K;
          S.done = 1;
        } else {
          const int top = 31 - __clz(kmin ^ kmax);
          S.mask = top == 31 ? 0u : (0xFFFFFFFFu << (top + 1));
          S.prefix = kmin & S.mask;
          S.need = K;
          S.hi = top;
          S.done = 0;
        }
      }
    }
  }
  __syncthreads();

#pragma unroll 1
  while (!S.done) {
    const int hi = S.hi;
    const int lo = hi >= 9 ? hi - 9 : 0;
    const uint32_t dmask = (hi - lo == 31) ? 0xFFFFFFFFu : (((1u << (hi - lo + 1)) - 1u) << lo);
    const uint32_t prefix = S.prefix, mask = S.mask;
    const int need = S.need;
    S.hist[tid] = 0u;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < ITEMS; ++i) {
      const uint32_t k = keys[i];
      if (k != 0u && (k & mask) == prefix) atomicAdd(&S.hist[(k & dmask) >> lo], 1u);
    }
    __syncthreads();
    // thread t owns digit 1023 - t: an exclusive sum in thread order counts
    // the keys in the digits above
    const int c = static_cast<int>(S.hist[1023 - tid]);
    int total;
    const int above = block_exclusive_sum<THREADS>(c, S.warp_tmp, &total);
    // fewer matching keys than needed (a head start that does not describe
    // the keys): stop with what is above the prefix instead of passing forever
    if (tid == 0 && total < need) {
      S.need = 0;
      S.done = 1;
    }
    if (above < need && need <= above + c) {   // exactly one thread
      const uint32_t d = 1023u - static_cast<uint32_t>(tid);
      S.prefix = prefix | (d << lo);
      S.mask = mask | dmask;
      S.need = need - above;
      S.hi = lo - 1;
      if (c == need - above || lo == 0) S.done = 1;
    }
    __syncthreads();
  }
}

// Select the K best keys of the CTA.  emit(i, r): key index i has output rank
// r (0 <= r < min(K, valid keys)); pad(r) for the ranks past the valid keys.
// start: optional head start (read after a barrier; may point into S.start).
// Called by all 1024 threads.
template <int ITEMS, class Emit, class Pad>
__device__ void block_topk(const uint32_t (&keys)[ITEMS], int K, BlockSelectSmem& S, Emit emit, Pad pad,
                           const SelectStart* start) {
  constexpr int THREADS = kBlockSelectThreads;
  const int tid = threadIdx.x;
  block_select_prefix(keys, K, S, start);

  // ---- keys above the threshold prefix, and ties on it (lower index first) ----
  const uint32_t prefix = S.prefix, mask = S.mask;
  const int need = S.need;
  int gt = 0, eq = 0;
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) {
    const uint32_t k = keys[i], km = k & mask;
    gt += (k != 0u && km > prefix) ? 1 : 0;
    eq += (k != 0u && km == prefix) ? 1 : 0;
  }
  int gt_total, eq_total;
  const int2 before = block_exclusive_sum2<THREADS>(gt, eq, S.warp_tmp, &gt_total, &eq_total);
  const int gt_before = before.x, eq_before = before.y;
  int take = max(0, min(need - eq_before, eq));   // ties this thread takes
  int r = gt_before + min(eq_before, need);
  if (gt + take > 0) {   // most threads select none of their keys
#pragma unroll
    for (int i = 0; i < ITEMS; ++i) {
      const uint32_t k = keys[i], km = k & mask;
      const bool above = k != 0u && km > prefix;
      const bool tie = k != 0u && km == prefix && take > 0;
      if (above || tie) {
        emit(tid * ITEMS + i, r);
        ++r;
        if (tie) --take;
      }
    }
  }
  const int sel_total = gt_total + min(eq_total, need);
  for (int q = sel_total + tid; q < K; q += THREADS) pad(q);
}

}  // namespace csa2
