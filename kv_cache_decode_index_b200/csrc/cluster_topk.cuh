// Exact top-K over keys spread across the CTAs of one thread-block cluster.
//
// Each CTA holds its share of the candidates' keys in shared memory
// (uint32, order-preserving; 0 = not a candidate).  Candidates are ordered by
// (cluster rank, local index); that order is the ascending candidate-id order,
// which decides ties (lower id first) and the output order (ascending).
//
// First the cluster-wide count, minimum and maximum of the valid keys: their
// common leading bits need no pass (scores of one request share their sign and
// most exponent bits), and K >= count selects everything.  A caller that knows
// the threshold's leading bits already (from a histogram of the keys) passes
// them as a SelectStart instead, and that phase is skipped.  Then radix select,
// 8 bits per pass from the first differing bit: every CTA builds the
// histogram of its keys that match the prefix decided so far, the CTAs read
// each other's histograms through distributed shared memory (one cluster
// barrier per pass, two histogram buffers), and all of them derive the same
// next digit.  The passes stop as soon as every key matching the prefix is
// needed.  Then each CTA counts its keys above / on the threshold prefix, the
// counts are exchanged once more, and every CTA writes its selected ids at
// their ranks.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace csa2 {

namespace cg = cooperative_groups;

constexpr int kMaxCluster = 16;

struct SelectSmem {
  uint32_t hist[2][256];
  uint32_t ghist[256];
  int gt_eq[2];              // this CTA's (above, on-threshold) counts, read remotely
  uint32_t stat[3];          // this CTA's (count, min, max) of valid keys, read remotely
  uint32_t wstat[32][3];
  int warp_tmp[32];
  uint32_t prefix, mask;
  int need;
  int done;
  int hi;                    // top bit of the next digit
  int total;                 // valid candidates in the cluster
  int fin[3];                // this CTA's output base, ties taken, cluster total
};

// Head start of a select: the threshold's leading bits (prefix under mask),
// found elsewhere, and the number of keys still needed among the keys that
// match them.  hi is the top bit of the next radix digit; done = 1 when the
// selection is decided already (every matching key is needed, or no bit is
// left).  All keys not matching the prefix are above it or below it.
struct SelectStart {
  uint32_t prefix, mask;
  int need;
  int hi;
  int done;
};

// Exclusive block-wide prefix sum of one int per thread (THREADS multiple of
// 32, <= 1024).  Returns the thread's exclusive prefix; *sum gets the total.
template <int THREADS>
__device__ __forceinline__ int block_exclusive_sum(int v, int* warp_tmp, int* sum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();   // warp_tmp reuse guard
  if (lane == 31) warp_tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = lane < THREADS / 32 ? warp_tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < THREADS / 32) warp_tmp[lane] = t;   // inclusive warp totals
  }
  __syncthreads();
  *sum = warp_tmp[THREADS / 32 - 1];
  return x - v + (warp > 0 ? warp_tmp[warp - 1] : 0);
}

// Two exclusive block-wide prefix sums at once, sharing the barriers of one
// (warp_tmp holds 2 * THREADS / 32 ints).  *sa, *sb get the totals.
template <int THREADS>
__device__ __forceinline__ int2 block_exclusive_sum2(int a, int b, int* warp_tmp, int* sa, int* sb) {
  constexpr int kW = THREADS / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = a, y = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int xa = __shfl_up_sync(0xffffffffu, x, o);
    const int yb = __shfl_up_sync(0xffffffffu, y, o);
    if (lane >= o) {
      x += xa;
      y += yb;
    }
  }
  __syncthreads();   // warp_tmp reuse guard
  if (lane == 31) {
    warp_tmp[warp] = x;
    warp_tmp[kW + warp] = y;
  }
  __syncthreads();
  if (warp == 0) {
    int t = lane < kW ? warp_tmp[lane] : 0, u = lane < kW ? warp_tmp[kW + lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ta = __shfl_up_sync(0xffffffffu, t, o);
      const int ub = __shfl_up_sync(0xffffffffu, u, o);
      if (lane >= o) {
        t += ta;
        u += ub;
      }
    }
    if (lane < kW) {   // inclusive warp totals
      warp_tmp[lane] = t;
      warp_tmp[kW + lane] = u;
    }
  }
  __syncthreads();
  *sa = warp_tmp[kW - 1];
  *sb = warp_tmp[2 * kW - 1];
  return make_int2(x - a + (warp > 0 ? warp_tmp[warp - 1] : 0), y - b + (warp > 0 ? warp_tmp[kW + warp - 1] : 0));
}

// Select the K best of the cluster's candidates.  emit(i, r) is called for the
// local candidate i that has output rank r (0 <= r < min(K, total)); pad(r) for
// r in [total, K) by the cluster's rank-0 CTA.  Must be called by all THREADS
// threads of every CTA of the cluster (it contains cluster barriers).  start:
// an optional head start, the same in every CTA of the cluster.
template <int THREADS, class Emit, class Pad>
__device__ void cluster_topk(const uint32_t* keys, int n_local, int K, SelectSmem& S, Emit emit, Pad pad,
                             const SelectStart* start = nullptr) {
  constexpr int kWarps = THREADS / 32;
  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rounds = (n_local + THREADS - 1) / THREADS;

  if (start != nullptr) {
    for (int i = tid; i < 256; i += THREADS) S.hist[0][i] = 0;
    if (tid == 0) {
      S.prefix = start->prefix;
      S.mask = start->mask;
      S.need = start->need;
      S.hi = start->hi;
      S.done = start->done;
    }
    __syncthreads();
  } else {
    // ---- count, min and max of the valid keys ----
    uint32_t cnt = 0, kmin = 0xFFFFFFFFu, kmax = 0u;
    for (int r = 0; r < rounds; ++r) {
      const int i = r * THREADS + tid;
      const uint32_t k = i < n_local ? keys[i] : 0u;
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
    for (int i = tid; i < 256; i += THREADS) S.hist[0][i] = 0;
    __syncthreads();
    if (warp == 0) {
      cnt = lane < kWarps ? S.wstat[lane][0] : 0u;
      kmin = lane < kWarps ? S.wstat[lane][1] : 0xFFFFFFFFu;
      kmax = lane < kWarps ? S.wstat[lane][2] : 0u;
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      kmin = __reduce_min_sync(0xffffffffu, kmin);
      kmax = __reduce_max_sync(0xffffffffu, kmax);
      if (lane == 0) {
        S.stat[0] = cnt;
        S.stat[1] = kmin;
        S.stat[2] = kmax;
      }
    }
    cluster.sync();   // every CTA's statistics are complete
    if (warp == 0) {
      const uint32_t* st = lane < C ? cluster.map_shared_rank(&S.stat[0], lane) : nullptr;
      cnt = st ? st[0] : 0u;
      kmin = st ? st[1] : 0xFFFFFFFFu;
      kmax = st ? st[2] : 0u;
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      kmin = __reduce_min_sync(0xffffffffu, kmin);
      kmax = __reduce_max_sync(0xffffffffu, kmax);
      if (lane == 0) {
        S.total = static_cast<int>(cnt);
        if (cnt <= static_cast<uint32_t>(K)) {   // everything valid is selected
          S.prefix = 0u;
          S.mask = 0u;
          S.need = static_cast<int>(cnt);
          S.done = 1;
        } else if (kmin == kmax) {                 // all valid keys tie: the first K by id
          S.prefix = kmin;
          S.mask = 0xFFFFFFFFu;
          S.need = K;
          S.done = 1;
        } else {
          const int top = 31 - __clz(kmin ^ kmax);   // highest bit where the keys differ
          S.mask = top == 31 ? 0u : (0xFFFFFFFFu << (top + 1));
          S.prefix = kmin & S.mask;
          S.need = K;
          S.hi = top;
          S.done = 0;
        }
      }
    }
    __syncthreads();
  }

#pragma unroll 1
  for (int pass = 0; !S.done; ++pass) {
    const int hi = S.hi;
    const int lo = hi >= 7 ? hi - 7 : 0;
    const uint32_t dmask = (hi - lo == 31) ? 0xFFFFFFFFu : (((1u << (hi - lo + 1)) - 1u) << lo);
    const int buf = pass & 1;
    const uint32_t prefix = S.prefix, mask = S.mask;
    for (int r = 0; r < rounds; ++r) {
      const int i = r * THREADS + tid;
      const uint32_t k = i < n_local ? keys[i] : 0u;
      if (k != 0u && (k & mask) == prefix) atomicAdd(&S.hist[buf][(k & dmask) >> lo], 1u);
    }
    cluster.sync();   // every CTA's histogram of this pass is complete
    for (int d = tid; d < 256; d += THREADS) {
      uint32_t part[kMaxCluster];   // remote reads issued together
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r) part[r] = r < C ? cluster.map_shared_rank(&S.hist[buf][0], r)[d] : 0u;
      uint32_t g = 0;
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r) g += part[r];
      S.ghist[d] = g;
      S.hist[buf ^ 1][d] = 0;   // next pass's buffer (last read remotely before this barrier)
    }
    __syncthreads();
    if (tid < 32) {
      // lane l owns digits 255-8l .. 248-8l (descending)
      uint32_t local[8];
      uint32_t sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        local[i] = S.ghist[255 - 8 * tid - i];
        sum += local[i];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      const uint32_t need = static_cast<uint32_t>(S.need);
      uint32_t above = incl - sum;   // keys in digits above this lane's range
      // fewer matching keys than needed: only a head start that does not
      // describe the keys does that; stop with what is above the prefix
      // rather than pass forever (the caller's start is verified)
      if (__shfl_sync(0xffffffffu, incl, 31) < need && tid == 0) {
        S.need = 0;
        S.done = 1;
      }
      if (above < need && need <= incl) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (above < need && need <= above + local[i]) {
            const uint32_t d = 255u - 8u * tid - i;
            S.prefix = prefix | (d << lo);
            S.mask = mask | dmask;
            S.need = static_cast<int>(need - above);
            S.hi = lo - 1;
            // all keys with this prefix are taken, or no bit is left to split them
            if (local[i] == need - above || lo == 0) S.done = 1;
          }
          above += local[i];
        }
      }
    }
    __syncthreads();
  }

  // ---- final: keys above the threshold prefix, and keys on it (ties) ----
  // Warp w owns the contiguous local range [wbeg, wend); lanes read it
  // interleaved and rank their selections with ballots, so the output keeps
  // the ascending candidate order.
  const uint32_t prefix = S.prefix, mask = S.mask;
  const int need = S.need;
  const int wper = (((n_local + kWarps - 1) / kWarps) + 31) & ~31;
  const int wbeg = min(warp * wper, n_local), wend = min(wbeg + wper, n_local);
  const uint32_t lt = (1u << lane) - 1u;
  int gt_w = 0, eq_w = 0;
  for (int base = wbeg; base < wend; base += 32) {
    const int i = base + lane;
    const uint32_t k = i < wend ? keys[i] : 0u;
    const uint32_t km = k & mask;
    gt_w += __popc(__ballot_sync(0xffffffffu, k != 0u && km > prefix));
    eq_w += __popc(__ballot_sync(0xffffffffu, k != 0u && km == prefix));
  }
  // per-warp totals -> CTA totals and this warp's position among them
  int local_gt, local_eq;
  const int eq_before_w = block_exclusive_sum<THREADS>(lane == 0 ? eq_w : 0, S.warp_tmp, &local_eq);
  const int gt_before_w = block_exclusive_sum<THREADS>(lane == 0 ? gt_w : 0, S.warp_tmp, &local_gt);
  if (tid == 0) {
    S.gt_eq[0] = local_gt;
    S.gt_eq[1] = local_eq;
  }
  cluster.sync();   // counts visible cluster-wide
  // one warp reads the C ranks' counts (lane r: rank r) and derives this
  // CTA's output base, its share of the ties and the total selected
  if (warp == 0) {
    const int g = lane < C ? cluster.map_shared_rank(&S.gt_eq[0], lane)[0] : 0;
    const int e = lane < C ? cluster.map_shared_rank(&S.gt_eq[0], lane)[1] : 0;
    int ties_incl = e;   // inclusive prefix of the tie counts over the ranks
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, ties_incl, o);
      if (lane >= o) ties_incl += y;
    }
    const int take = max(0, min(need - (ties_incl - e), e));
    int sel_incl = g + take;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, sel_incl, o);
      if (lane >= o) sel_incl += y;
    }
    if (lane == rank) {
      S.fin[0] = sel_incl - (g + take);   // selections of the lower ranks
      S.fin[1] = take;
    }
    if (lane == 31) S.fin[2] = sel_incl;
  }
  __syncthreads();
  const int out_base = S.fin[0], take_local = S.fin[1], sel_total = S.fin[2];
  // ties taken by this warp, and the output rank of its first selection
  const int eqb = __shfl_sync(0xffffffffu, eq_before_w, 0);
  const int gtb = __shfl_sync(0xffffffffu, gt_before_w, 0);
  const int take_w = max(0, min(take_local - eqb, eq_w));
  const int ties_taken_before_w = max(0, min(take_local, eqb));
  int sel_rank = out_base + gtb + ties_taken_before_w;
  int ties_seen = 0;
  for (int base = wbeg; base < wend; base += 32) {
    const int i = base + lane;
    const uint32_t k = i < wend ? keys[i] : 0u;
    const uint32_t km = k & mask;
    const bool above = k != 0u && km > prefix;
    const bool tie = k != 0u && km == prefix;
    const uint32_t tie_bal = __ballot_sync(0xffffffffu, tie);
    const bool take = above || (tie && ties_seen + __popc(tie_bal & lt) < take_w);
    const uint32_t sel_bal = __ballot_sync(0xffffffffu, take);
    if (take) emit(i, sel_rank + __popc(sel_bal & lt));
    sel_rank += __popc(sel_bal);
    ties_seen += __popc(tie_bal);
  }
  if (rank == 0)
    for (int r = sel_total + tid; r < K; r += THREADS) pad(r);
  cluster.sync();   // no CTA leaves while its shared memory may still be read
}

}  // namespace csa2
