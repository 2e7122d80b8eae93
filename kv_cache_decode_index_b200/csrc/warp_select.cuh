// Exact Top-k of a candidate list by ONE warp: radix select over 32-bit keys
// (8-bit digits from the top bit, lane-aggregated shared-memory histogram),
// ties at the k-th key broken by the lower position, then an in-place,
// order-preserving compaction.  The list lives in global memory as two arrays
// (order keys, positions), 16-byte aligned; positions are distinct.
//
// Ranking rule [reading of the indexer's Top-512, 4sapi blog, section 四]: a
// larger score first, the lower position on equal scores.
#pragma once

#include "common.cuh"

namespace csa2 {

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Four consecutive entries [base, base + 4) of a 16-byte aligned array of
// 32-bit values with n valid entries and room for at least
// round_up(n, 4) entries: one vector load, entries at or past n flagged
// invalid.
__device__ __forceinline__ void load4(const uint32_t* a, int base, int n, uint32_t (&v)[4], bool (&ok)[4]) {
  uint4 x = make_uint4(0u, 0u, 0u, 0u);
  if (base < n) x = *reinterpret_cast<const uint4*>(a + base);
  v[0] = x.x;
  v[1] = x.y;
  v[2] = x.z;
  v[3] = x.w;
#pragma unroll
  for (int e = 0; e < 4; ++e) ok[e] = base + e < n;
}

constexpr int kSelBatch = 8;   // vector loads per lane in flight in the selection passes

struct KthResult {
  uint32_t thr;   // k-th largest value, or the lower edge of its digit bin
  int need;       // entries equal to thr still to take (exact case)
  bool exact;     // false: every participant >= thr is taken (exactly kk of them)
};

// The kk-th largest (kk >= 1, kk <= number of participants) of the values
// that `fetch(base, v, ok)` delivers four at a time for base = 0, 4, 8, ... < n.
// If the digit bin holding the kk-th value holds exactly the entries still
// needed, stops there: then the participants >= thr are exactly kk.
// Otherwise returns the exact value thr with `need` = how many of the entries
// equal to thr belong to the kk largest (the rest of them do not).
template <class Fetch>
__device__ KthResult warp_kth_largest(Fetch fetch, int n, int kk, uint32_t* hist, int lane) {
  uint32_t prefix = 0, pmask = 0;
  int need = kk;
  for (int hi = 31; hi >= 0;) {
    const int lo = hi >= 7 ? hi - 7 : 0;
    const uint32_t dmask = (2u << (hi - lo)) - 1u;
#pragma unroll
    for (int t = 0; t < 8; ++t) hist[lane * 8 + t] = 0u;
    __syncwarp();
    for (int base0 = 0; base0 < n; base0 += 128 * kSelBatch) {
      uint32_t v[kSelBatch][4];
      bool ok[kSelBatch][4];
#pragma unroll
      for (int c = 0; c < kSelBatch; ++c) fetch(base0 + c * 128 + lane * 4, v[c], ok[c]);
#pragma unroll
      for (int c = 0; c < kSelBatch; ++c)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool act = ok[c][e] && (v[c][e] & pmask) == prefix;
          const uint32_t d = (v[c][e] >> lo) & dmask;
          const uint32_t am = __ballot_sync(0xffffffffu, act);
          if (act) {
            const uint32_t peers = __match_any_sync(am, d);
            if ((__ffs(peers) - 1) == lane) atomicAdd(&hist[d], static_cast<uint32_t>(__popc(peers)));
          }
        }
    }
    __syncwarp();
    uint32_t c[8], lsum = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      c[t] = hist[lane * 8 + t];
      lsum += c[t];
    }
    uint32_t suf = lsum;   // participants in the bins of lanes >= this lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_down_sync(0xffffffffu, suf, o);
      if (lane + o < 32) suf += t;
    }
    const uint32_t above_lane = suf - lsum;
    const bool mine = above_lane < static_cast<uint32_t>(need) && static_cast<uint32_t>(need) <= suf;
    const int L = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    uint32_t d = 0, above = 0, in_bin = 0;
    if (lane == L) {
      uint32_t acc = above_lane;
#pragma unroll
      for (int t = 7; t >= 0; --t) {
        if (in_bin == 0u && acc + c[t] >= static_cast<uint32_t>(need)) {
          d = static_cast<uint32_t>(lane * 8 + t);
          above = acc;
          in_bin = c[t];
        }
        acc += c[t];
      }
    }
    d = __shfl_sync(0xffffffffu, d, L);
    above = __shfl_sync(0xffffffffu, above, L);
    in_bin = __shfl_sync(0xffffffffu, in_bin, L);
    need -= static_cast<int>(above);
    prefix |= d << lo;
    pmask |= dmask << lo;
    __syncwarp();   // the histogram is cleared again by the next pass
    if (static_cast<int>(in_bin) == need) return KthResult{prefix, need, false};
    hi = lo - 1;
  }
  return KthResult{prefix, need, true};
}

// Keep the k best entries (larger key first, lower position on equal keys) of
// keys[0, n) / pos[0, n), moved to the front in their original order.  Both
// arrays must have room for round_up(n, 4) entries.
// Returns the number kept (min(n, k)) and in *theta a key threshold such that
// an entry with a key <= *theta and a position above every kept one can never
// enter the k best.  n > k is required for *theta to be written.
__device__ __forceinline__ int warp_compact_topk(uint32_t* keys, int32_t* pos, int n, int k, uint32_t* hist,
                                                 int lane, uint32_t* theta) {
  if (n <= k) return n;
  auto fetch_keys = [&](int base, uint32_t (&v)[4], bool (&ok)[4]) { load4(keys, base, n, v, ok); };
  const KthResult r = warp_kth_largest(fetch_keys, n, k, hist, lane);
  // Entries equal to r.thr in an exact result: take the r.need lowest positions
  // (the r.need largest complemented positions).
  bool all_ties = !r.exact;
  uint32_t pos_cut = 0;
  if (r.exact) {
    auto fetch_ties = [&](int base, uint32_t (&v)[4], bool (&ok)[4]) {
      uint32_t kv[4];
      load4(keys, base, n, kv, ok);
      uint32_t pv[4];
      bool pok[4];
      load4(reinterpret_cast<const uint32_t*>(pos), base, n, pv, pok);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        ok[e] = ok[e] && kv[e] == r.thr;
        v[e] = ~pv[e];
      }
    };
    const KthResult t = warp_kth_largest(fetch_ties, n, r.need, hist, lane);
    pos_cut = t.thr;   // positions are distinct, so t is exact or a bin edge: take ~pos >= cut
  }
  // In-place, order-preserving: a batch is read completely before any of its
  // survivors is written, and survivors never move to a higher index.
  constexpr int kCB = kSelBatch / 2;
  int out = 0;
  for (int base0 = 0; base0 < n; base0 += 128 * kCB) {
    uint32_t kv[kCB][4], pv[kCB][4];
    bool ok[kCB][4], pok[kCB][4];
#pragma unroll
    for (int c = 0; c < kCB; ++c) {
      load4(keys, base0 + c * 128 + lane * 4, n, kv[c], ok[c]);
      load4(reinterpret_cast<const uint32_t*>(pos), base0 + c * 128 + lane * 4, n, pv[c], pok[c]);
    }
    __syncwarp();
#pragma unroll
    for (int c = 0; c < kCB; ++c) {
      bool keep[4];
      int cnt = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        keep[e] = ok[c][e] && (kv[c][e] > r.thr || (kv[c][e] == r.thr && (all_ties || ~pv[c][e] >= pos_cut)));
        cnt += keep[e] ? 1 : 0;
      }
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      int at = out + incl - cnt;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (keep[e]) {
          keys[at] = kv[c][e];
          pos[at] = static_cast<int32_t>(pv[c][e]);
          ++at;
        }
      out += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  __syncwarp();
  *theta = r.thr;
  return out;
}

}  // namespace csa2
