// Exact top-K over keys spread across the CTAs of one thread-block cluster.
//
// Each CTA holds its share of the candidates' keys in shared memory
// (uint32, order-preserving; 0 = not a candidate).  Candidates are ordered by
// (cluster rank, local index); that order is the ascending candidate-id order,
// which decides ties (lower id first) and the output order (ascending).
//
// Radix select, 8 bits per pass from the top: every CTA builds the histogram
// of its keys that match the prefix decided so far, the CTAs read each other's
// histograms through distributed shared memory (one cluster barrier per pass,
// two histogram buffers), and all of them derive the same next digit.  The
// passes stop as soon as every key matching the prefix is needed.  Then each
// CTA counts its keys above / on the threshold prefix, the counts are
// exchanged once more, and every CTA writes its selected ids at their ranks.
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
  int warp_tmp[32];
  uint32_t prefix, mask;
  int need;
  int done;
  int total;                 // valid candidates in the cluster
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

// Select the K best of the cluster's candidates.  emit(i, r) is called for the
// local candidate i that has output rank r (0 <= r < min(K, total)); pad(r) for
// r in [total, K) by the cluster's rank-0 CTA.  Must be called by all THREADS
// threads of every CTA of the cluster (it contains cluster barriers).
template <int THREADS, class Emit, class Pad>
__device__ void cluster_topk(const uint32_t* keys, int n_local, int K, SelectSmem& S, Emit emit, Pad pad) {
  constexpr int kWarps = THREADS / 32;
  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rounds = (n_local + THREADS - 1) / THREADS;

  if (tid == 0) {
    S.prefix = 0;
    S.mask = 0;
    S.done = 0;
  }
  for (int i = tid; i < 256; i += THREADS) S.hist[0][i] = 0;
  __syncthreads();

#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const int buf = pass & 1;
    const uint32_t prefix = S.prefix, mask = S.mask;
    // Keys of one request concentrate in a few bins in the first passes, so
    // increments are aggregated per warp: one atomic per distinct bin.
    for (int r = 0; r < rounds; ++r) {
      const int i = r * THREADS + tid;
      const uint32_t k = i < n_local ? keys[i] : 0u;
      const bool counted = k != 0u && (k & mask) == prefix;
      const uint32_t bin = counted ? ((k >> shift) & 255u) : 256u;
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (counted && lane == __ffs(peers) - 1) atomicAdd(&S.hist[buf][bin], __popc(peers));
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
      const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
      if (pass == 0 && tid == 0) {
        S.total = static_cast<int>(total);
        if (total <= static_cast<uint32_t>(K)) {   // everything valid is selected
          S.need = static_cast<int>(total);
          S.done = 1;
        } else {
          S.need = K;
        }
      }
      __syncwarp();
      if (!S.done) {
        const uint32_t need = static_cast<uint32_t>(S.need);
        uint32_t above = incl - sum;   // keys in digits above this lane's range
        if (above < need && need <= incl) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (above < need && need <= above + local[i]) {
              const uint32_t d = 255u - 8u * tid - i;
              S.prefix = prefix | (d << shift);
              S.mask = mask | (255u << shift);
              S.need = static_cast<int>(need - above);
              if (local[i] == need - above) S.done = 1;   // all keys with this prefix are taken
            }
            above += local[i];
          }
        }
      }
    }
    __syncthreads();
    if (S.done) break;
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
  int rg[kMaxCluster], re[kMaxCluster];   // remote reads issued together
#pragma unroll
  for (int r = 0; r < kMaxCluster; ++r) {
    rg[r] = r < C ? cluster.map_shared_rank(&S.gt_eq[0], r)[0] : 0;
    re[r] = r < C ? cluster.map_shared_rank(&S.gt_eq[0], r)[1] : 0;
  }
  int out_base = 0, take_local = 0, sel_total = 0, ties_before = 0;
#pragma unroll
  for (int r = 0; r < kMaxCluster; ++r) {
    if (r >= C) break;
    const int g = rg[r], e = re[r];
    const int take = max(0, min(need - ties_before, e));
    if (r < rank) out_base += g + take;
    if (r == rank) take_local = take;
    sel_total += g + take;
    ties_before += e;
  }
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
