// Work units of the Full scans (FP8 and FP4 indexer): the visible positions
// of all requests, in request order, cut into units of 256 positions; a
// CTA owns a contiguous range of the concatenated units.  prefix[b] is the
// number of units before request b (prefix[batch] = all units).
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kScanUnit = 2 * kTile;   // positions per unit (two 128-row MMA tiles)

// Walks a CTA's units in order: request b, unit j inside it.
struct TileIter {
  const int* prefix;
  int batch;
  int b, j;
  __device__ void init(const int* pre, int nb, int g) {
    prefix = pre;
    batch = nb;
    int lo = 0, hi = nb - 1;   // last b with prefix[b] <= g
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pre[mid] <= g) lo = mid;
      else hi = mid - 1;
    }
    b = lo;
    j = g - pre[lo];
    skip_empty();
  }
  __device__ void skip_empty() {
    while (b < batch && j >= prefix[b + 1] - prefix[b]) {
      j = 0;
      ++b;
    }
  }
  __device__ void advance() {
    ++j;
    skip_empty();
  }
};

__device__ __forceinline__ int next_request_with_tiles(const int* prefix, int batch, int b) {
  ++b;
  while (b < batch && prefix[b + 1] == prefix[b]) ++b;
  return b;
}

// Cache rows of one unit's two 128-row tiles, found in two steps so that a
// warp can resolve 32 units at once (one per lane) and keep the page-table
// loads in flight while it does other work: fetch() issues the loads,
// rows() uses them.  The issuing lane of a scan's producer then does no
// address arithmetic and waits on no global load per unit.
struct UnitRows {
  int b;         // request, or -1: no unit
  int p0;        // first position of the unit
  int pidx;      // page index of tile 0
  int page[2];   // page-table entries (page[1] = -2: tile 1 is on tile 0's page, or absent)
  int n;         // the request's visible positions (a page-table slot past them need not be valid)

  // Unit g (global index among all units; g < prefix[batch] or the slot is
  // empty).  Positions are below 2^31 (checked on the host): 32-bit
  // arithmetic.
  __device__ void fetch(const csa2_cache& cache, const int* prefix, int batch, int g, bool valid,
                        long long capacity, uint32_t page_size) {
    b = -1;
    page[0] = page[1] = 0;
    if (!valid) return;
    int lo = 0, hi = batch - 1;   // last request with prefix <= g: the request of unit g
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= g) lo = mid;
      else hi = mid - 1;
    }
    b = lo;
    n = cache.ctx_len[lo];   // in flight with the page-table loads
    p0 = (g - prefix[lo]) * kScanUnit;
    pidx = static_cast<int>(static_cast<uint32_t>(p0) / page_size);
    const int32_t* pt = cache.page_table + static_cast<long long>(lo) * cache.max_pages_per_req;
    page[0] = pt[pidx];
    const int p1 = p0 + kTile;
    page[1] = (p1 < capacity && static_cast<uint32_t>(p1) / page_size != static_cast<uint32_t>(pidx)) ? pt[pidx + 1]
                                                                                                      : -2;
  }

  // r[h]: cache row of tile h, or -1 when the tile starts past the request's
  // visible positions (its page-table slot need not hold a page).  A page id
  // outside [0, num_pages) is reported (CSA2_ERR_DEVICE_BOUNDS) and replaced
  // by page 0, so that the copy stays in bounds; the results of that tile
  // are flagged invalid by the report.
  __device__ void rows(const csa2_cache& cache, long long capacity, int kernel, int (&r)[2]) const {
    r[0] = r[1] = -1;
    if (b < 0) return;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int p = p0 + h * kTile;
      if (p >= capacity || p >= n) continue;
      const bool own_page = h == 1 && page[1] != -2;
      int pg = own_page ? page[1] : page[0];
      if (pg < 0 || pg >= cache.num_pages) {
        report_error(cache.err_word, CSA2_ERR_DEVICE_BOUNDS, kernel, b, p);
        pg = 0;
      }
      r[h] = pg * cache.page_size + (p - (pidx + own_page) * cache.page_size);
    }
  }
};

}  // namespace csa2
