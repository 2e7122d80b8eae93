// Pool of a context-sharded request: a 1M-position context split into
// consecutive slices, one per device, each scanned and pooled on its own
// device [alphalab analysis, limits section: a context this long may have to
// be sharded across machines, at the price of the exchange between them].
//
//   pool_candidates_kernel: a slice's local pool as (block max, global block
//     id) pairs, the 8 bytes per pool entry that the devices exchange (16 KB
//     per request for a 2048-block pool);
//   pool_merge_kernel: one CTA of 1024 threads per request holds the G slices'
//     candidates (G x 2048 keys) in registers and selects the exact top
//     pool_blocks, ties to the lower global block id: the slices come in
//     ascending order and each list is ascending, so candidate order is global
//     id order.  A block of the whole request's pool has fewer than
//     pool_blocks blocks ahead of it in its own slice, so its slice kept it:
//     the merge equals the pool of the unsharded request.
#include "block_topk.cuh"
#include "launch.h"

namespace csa2 {

namespace {

__global__ void pool_candidates_kernel(const csa2_cache cache, const float* __restrict__ blockmax,
                                       const int32_t* __restrict__ pool, int P, int block_offset,
                                       float* __restrict__ values, int32_t* __restrict__ ids) {
  pdl_wait();   // the slice's pool of the preceding launch is complete
  pdl_launch_dependents();
  const long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  if (i >= static_cast<long long>(cache.batch) * P) return;
  const int b = static_cast<int>(i / P);
  const long long capacity = static_cast<long long>(cache.max_pages_per_req) * cache.page_size;
  const int n = max(0, checked_ctx_len(cache, b, capacity, kKPoolSelect, i % P == 0));
  const int nblk = (n + kBlock - 1) / kBlock;
  const int j = pool[i];
  float v = 0.0f;
  int id = -1;
  if (j >= 0 && j < nblk) {
    v = blockmax[static_cast<long long>(b) * (capacity / kBlock) + j];
    id = j + block_offset;
  } else if (j >= nblk || j < -1) {
    report_error(cache.err_word, CSA2_ERR_DEVICE_BOUNDS, kKPoolSelect, b, j);
  }
  values[i] = v;
  ids[i] = id;
}

// values / ids: [G][batch][P]; pool: [batch][P]
template <int ITEMS>
__global__ void __launch_bounds__(kBlockSelectThreads, 1)
    pool_merge_kernel(int G, int batch, int P, const float* __restrict__ values, const int32_t* __restrict__ ids,
                      int32_t* __restrict__ pool) {
  __shared__ BlockSelectSmem S;
  const int b = blockIdx.x, tid = threadIdx.x;
  const int n = G * P;
  pdl_wait();   // the candidates (copied or gathered before this launch) are complete
  pdl_launch_dependents();
  auto at = [&](int i) { return (static_cast<long long>(i / P) * batch + b) * P + i % P; };
  uint32_t k[ITEMS];
#pragma unroll
  for (int j = 0; j < ITEMS; ++j) {
    const int i = tid * ITEMS + j;
    k[j] = 0u;
    if (i < n) {
      const long long a = at(i);
      if (ids[a] >= 0) k[j] = order_key(values[a]);
    }
  }
  int32_t* out = pool + static_cast<long long>(b) * P;
  block_topk<ITEMS>(
      k, P, S, [&](int i, int r) { out[r] = ids[at(i)]; }, [&](int r) { out[r] = -1; }, nullptr);
}

}  // namespace

cudaError_t launch_pool_candidates(const csa2_cache& cache, const float* blockmax, const int32_t* pool, int P,
                                   int block_offset, float* values, int32_t* ids, cudaStream_t stream) {
  const long long total = static_cast<long long>(cache.batch) * P;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.stream = stream;
  cfg.blockDim = dim3(256);
  cfg.gridDim = dim3(static_cast<unsigned>((total + 255) / 256));
  return cudaLaunchKernelEx(&cfg, pool_candidates_kernel, cache, blockmax, pool, P, block_offset, values, ids);
}

cudaError_t launch_pool_merge(int n_shards, int batch, int P, const float* values, const int32_t* ids, int32_t* pool,
                              cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.stream = stream;
  cfg.blockDim = dim3(kBlockSelectThreads);
  cfg.gridDim = dim3(batch);
  const long long n = static_cast<long long>(n_shards) * P;
  if (n <= 16LL * kBlockSelectThreads)
    return cudaLaunchKernelEx(&cfg, pool_merge_kernel<16>, n_shards, batch, P, values, ids, pool);
  return cudaLaunchKernelEx(&cfg, pool_merge_kernel<32>, n_shards, batch, P, values, ids, pool);
}

}  // namespace csa2
