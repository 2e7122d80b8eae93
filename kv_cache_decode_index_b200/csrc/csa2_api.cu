// C ABI of libcsa2.so (declared in include/csa2.h): host-side validation,
// TMA tensor maps, launches.  No allocation, no synchronisation except in
// csa2_get_error.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace {

thread_local char g_msg[512] = "";

csa2_status fail(csa2_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

csa2_status cuda_fail(cudaError_t e, const char* what) {
  return fail(CSA2_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr int kMaxBatch = 1024;
constexpr int kMaxK = 4096;
constexpr int kMaxPool = 4096;
constexpr long long kMaxFlatPositions = 65536;        // Top-k without a pool
constexpr long long kMaxPoolSelectBlocks = 16LL * 16384;
constexpr int kMaxPrefillQueries = 1 << 20;

uint64_t g_wait_limit_ns = csa2::kWaitLimitNs;

// Device properties, cached per device ordinal.
struct DeviceInfo {
  int sms = 0;
  int major = 0;
};
std::mutex g_dev_mu;
DeviceInfo g_dev[64];

csa2_status device_info(DeviceInfo* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(CSA2_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_dev[dev].sms == 0) {
    int sms = 0, major = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    g_dev[dev].sms = sms;
    g_dev[dev].major = major;
  }
  *out = g_dev[dev];
  if (out->major != 10) return fail(CSA2_ERR_UNSUPPORTED, "needs an sm_100 (B200-class) device, found sm_%d", out->major * 10);
  return CSA2_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point.
using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

csa2_status encode_rows_map(void* base, long long rows, int row_bytes, int box_rows, CUtensorMapSwizzle swizzle,
                            CUtensorMap* map);

csa2_status encode_ik_map(const csa2_cache* c, int box_rows, CUtensorMap* map) {
  return encode_rows_map(c->ik_codes, static_cast<long long>(c->num_pages) * c->page_size, csa2::kIndexDim, box_rows,
                         CU_TENSOR_MAP_SWIZZLE_128B, map);
}

// 2-D map over `rows` rows of `row_bytes` bytes (uint8), box of box_rows
// full rows.
csa2_status encode_rows_map(void* base, long long rows, int row_bytes, int box_rows, CUtensorMapSwizzle swizzle,
                            CUtensorMap* map) {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  if (fn == nullptr) return fail(CSA2_ERR_UNSUPPORTED, "cuTensorMapEncodeTiled is not available");
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(row_bytes), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CSA2_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return CSA2_OK;
}

csa2_status check_ik4(const csa2_ik4* ik4) {
  if (ik4 == nullptr || ik4->codes == nullptr || ik4->scales == nullptr || !aligned(ik4->codes, 16) ||
      !aligned(ik4->scales, 16))
    return fail(CSA2_ERR_ARG, "ik4, ik4.codes and ik4.scales must be set and 16-byte aligned");
  return CSA2_OK;
}

long long capacity_of(const csa2_cache* c) {
  return static_cast<long long>(c->max_pages_per_req) * c->page_size;
}

csa2_status check_cache(const csa2_cache* c, bool need_kv, bool need_ik) {
  if (c == nullptr) return fail(CSA2_ERR_ARG, "cache is NULL");
  if (c->page_table == nullptr || c->ctx_len == nullptr || c->err_word == nullptr)
    return fail(CSA2_ERR_ARG, "cache.page_table, ctx_len and err_word must be set");
  if (c->batch < 1 || c->batch > kMaxBatch) return fail(CSA2_ERR_SHAPE, "batch %d outside [1, %d]", c->batch, kMaxBatch);
  if (c->page_size <= 0 || c->page_size % csa2::kTile != 0)
    return fail(CSA2_ERR_SHAPE, "page_size %d must be a positive multiple of 128", c->page_size);
  if (c->num_pages < 1 || c->max_pages_per_req < 1)
    return fail(CSA2_ERR_SHAPE, "num_pages and max_pages_per_req must be >= 1");
  if (static_cast<long long>(c->num_pages) * c->page_size >= (1LL << 31))
    return fail(CSA2_ERR_SHAPE, "num_pages * page_size must stay below 2^31 rows");
  if (capacity_of(c) >= (1LL << 31)) return fail(CSA2_ERR_SHAPE, "max_pages_per_req * page_size must stay below 2^31");
  if (need_kv && (c->kv_codes == nullptr || c->kv_scales == nullptr || !aligned(c->kv_codes, 16) ||
                  !aligned(c->kv_scales, 16)))
    return fail(CSA2_ERR_ARG, "kv_codes and kv_scales must be set and 16-byte aligned");
  if (need_ik && (c->ik_codes == nullptr || c->ik_exp == nullptr || !aligned(c->ik_codes, 16) ||
                  !aligned(c->ik_exp, 16)))
    return fail(CSA2_ERR_ARG, "ik_codes and ik_exp must be set and 16-byte aligned");
  return CSA2_OK;
}

#define CSA2_TRY(expr)                 \
  do {                                 \
    const csa2_status s_ = (expr);     \
    if (s_ != CSA2_OK) return s_;      \
  } while (0)

csa2_status sparse_attn_impl(const csa2_cache* cache, int32_t n_layers, int32_t n_queries, const int32_t* q_req,
                             const int32_t* const* topk, int32_t k, const uint16_t* const* q, int32_t H, float scale,
                             uint16_t* const* out, void* stream, void* workspace = nullptr,
                             size_t workspace_bytes = 0) {
  CSA2_TRY(check_cache(cache, true, false));
  if (n_layers < 1 || n_layers > CSA2_ATTN_MAX_LAYERS)
    return fail(CSA2_ERR_SHAPE, "n_layers %d outside [1, %d]", n_layers, CSA2_ATTN_MAX_LAYERS);
  if (n_queries < 0) return fail(CSA2_ERR_SHAPE, "n_queries %d < 0", n_queries);
  if (n_queries == 0) return CSA2_OK;
  if (q_req == nullptr && n_queries > cache->batch)
    return fail(CSA2_ERR_SHAPE, "without q_req, n_queries (%d) must not exceed batch (%d)", n_queries, cache->batch);
  if (H != 16 && H != 32 && H != 64) return fail(CSA2_ERR_SHAPE, "H %d not in {16, 32, 64}", H);
  if (k < 1 || k > kMaxK) return fail(CSA2_ERR_SHAPE, "k %d outside [1, %d]", k, kMaxK);
  if (static_cast<long long>(n_layers) * n_queries * 4 >= (1LL << 31))
    return fail(CSA2_ERR_SHAPE, "n_layers * n_queries too large");
  if (topk == nullptr || q == nullptr || out == nullptr) return fail(CSA2_ERR_ARG, "topk, q and out must be set");
  for (int l = 0; l < n_layers; ++l)
    if (topk[l] == nullptr || q[l] == nullptr || out[l] == nullptr || !aligned(q[l], 16) || !aligned(out[l], 16))
      return fail(CSA2_ERR_ARG, "layer %d: topk, q and out (16-byte aligned) must be set", l);
  if (workspace != nullptr) {
    if (!aligned(workspace, 16)) return fail(CSA2_ERR_ARG, "workspace must be 16-byte aligned");
    const size_t need = csa2::attn_workspace_bytes(n_layers, n_queries, H);
    if (workspace_bytes < need)
      return fail(CSA2_ERR_SHAPE, "workspace_bytes %zu < %zu (csa2_attn_workspace_bytes)", workspace_bytes, need);
  }
  DeviceInfo d;
  CSA2_TRY(device_info(&d));
  const cudaError_t e = csa2::launch_sparse_attn(*cache, n_layers, n_queries, q_req, topk, k, q, H, scale, out,
                                                 static_cast<cudaStream_t>(stream), nullptr, nullptr, nullptr, 0,
                                                 workspace);
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "sparse_attn launch");
}

}  // namespace

extern "C" {

csa2_status csa2_append_kv(const csa2_cache* cache, int32_t n_rows, const float* kv_new, const float* ik_new,
                           const int32_t* req, const int32_t* pos, void* stream) {
  CSA2_TRY(check_cache(cache, true, true));
  if (n_rows < 0) return fail(CSA2_ERR_SHAPE, "n_rows %d < 0", n_rows);
  if (n_rows == 0) return CSA2_OK;
  if (kv_new == nullptr || ik_new == nullptr || pos == nullptr || !aligned(kv_new, 16) || !aligned(ik_new, 16))
    return fail(CSA2_ERR_ARG, "kv_new, ik_new (16-byte aligned) and pos must be set");
  if (req == nullptr && n_rows > cache->batch)
    return fail(CSA2_ERR_SHAPE, "without req, n_rows (%d) must not exceed batch (%d)", n_rows, cache->batch);
  DeviceInfo d;
  CSA2_TRY(device_info(&d));
  const cudaError_t e = csa2::launch_append(*cache, n_rows, kv_new, ik_new, req, pos, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "append_kv launch");
}

csa2_status csa2_compress_append(const csa2_cache* cache, int32_t n_entries, int32_t m, const float* kv_tok,
                                 const float* ik_tok, const int32_t* req, const int32_t* pos, void* stream) {
  CSA2_TRY(check_cache(cache, true, true));
  if (n_entries < 0) return fail(CSA2_ERR_SHAPE, "n_entries %d < 0", n_entries);
  if (m != 1 && m != 2 && m != 4 && m != 8) return fail(CSA2_ERR_SHAPE, "m %d not in {1, 2, 4, 8}", m);
  if (n_entries == 0) return CSA2_OK;
  if (kv_tok == nullptr || ik_tok == nullptr || pos == nullptr || !aligned(kv_tok, 16) || !aligned(ik_tok, 16))
    return fail(CSA2_ERR_ARG, "kv_tok, ik_tok (16-byte aligned) and pos must be set");
  if (static_cast<long long>(n_entries) * m >= (1LL << 31))
    return fail(CSA2_ERR_SHAPE, "n_entries * m must stay below 2^31");
  DeviceInfo d;
  CSA2_TRY(device_info(&d));
  const cudaError_t e = csa2::launch_compress_append(*cache, n_entries, m, kv_tok, ik_tok, req, pos,
                                                     static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "compress_append launch");
}

csa2_status csa2_index_full(const csa2_cache* cache, const float* q, const float* w, float* blockmax, float* scores,
                            uint32_t* hist, void* stream) {
  CSA2_TRY(check_cache(cache, false, true));
  if (q == nullptr || w == nullptr || blockmax == nullptr || !aligned(q, 16))
    return fail(CSA2_ERR_ARG, "q (16-byte aligned), w and blockmax must be set");
  if (hist != nullptr && !aligned(hist, 16)) return fail(CSA2_ERR_ARG, "hist must be 16-byte aligned");
  DeviceInfo d;
  CSA2_TRY(device_info(&d));
  // With pages of whole 256-position units, one TMA box covers a unit.
  const int whole_units = cache->page_size % (2 * csa2::kTile) == 0;
  CUtensorMap map;
  CSA2_TRY(encode_ik_map(cache, whole_units ? 2 * csa2::kTile : csa2::kTile, &map));
  const cudaError_t e = csa2::launch_index_full(*cache, q, w, blockmax, scores, hist, map, whole_units, d.sms,
                                                g_wait_limit_ns,
                                                static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "index_full launch");
}

csa2_status csa2_append_ik4(const csa2_cache* cache, const csa2_ik4* ik4, int32_t n_rows, const float* ik_new,
                            const int32_t* req, const int32_t* pos, void* stream) {
  CSA2_TRY(check_cache(cache, false, false));
  CSA2_TRY(check_ik4(ik4));
  if (n_rows < 0) return fail(CSA2_ERR_SHAPE, "n_rows %d < 0", n_rows);
  if (n_rows == 0) return CSA2_OK;
  if (ik_new == nullptr || pos == nullptr || !aligned(ik_new, 16))
    return fail(CSA2_ERR_ARG, "ik_new (16-byte aligned) and pos must be set");
  if (req == nullptr && n_rows > cache->batch)
    return fail(CSA2_ERR_SHAPE, "without req, n_rows (%d) must not exceed batch (%d)", n_rows, cache->batch);
  DeviceInfo d;
  CSA2_TRY(device_info(&d));
  const cudaError_t e = csa2::launch_append_ik4(*cache, ik4->codes, ik4->scales, n_rows, ik_new, req, pos,
                                                static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "append_ik4 launch");
}

csa2_status csa2_index_full_fp4(const csa2_cache* cache, const csa2_ik4* ik4, const float* q, const float* w,
                                float* blockmax, float* scores, uint32_t* hist, void* stream) {
  CSA2_TRY(check_cache(cache, false, false));
  CSA2_TRY(check_ik4(ik4));
  if (q == nullptr || w == nullptr || blockmax == nullptr || !aligned(q, 16))
    return fail(CSA2_ERR_ARG, "q (16-byte aligned), w and blockmax must be set");
  if (hist != nullptr && !aligned(hist, 16)) return fail(CSA2_ERR_ARG, "hist must be 16-byte aligned");
  DeviceInfo d;
  CSA2_TRY(device_info(&d));
  const int whole_units = cache->page_size % (2 * csa2::kTile) == 0;   // one TMA box per unit
  CUtensorMap map;
  CSA2_TRY(encode_rows_map(ik4->codes, static_cast<long long>(cache->num_pages) * cache->page_size,
                           CSA2_IK4_CODE_BYTES, whole_units ? 2 * csa2::kTile : csa2::kTile,
                           CU_TENSOR_MAP_SWIZZLE_64B, &map));
  const cudaError_t e = csa2::launch_index_full_fp4(*cache, ik4->scales, q, w, blockmax, scores, hist, map,
                                                    whole_units, d.sms, g_wait_limit_ns,
                                                    static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "index_full_fp4 launch");
}

csa2_status csa2_pool_select(const csa2_cache* cache, const float* blockmax, uint32_t* hist, int32_t pool_blocks,
                             int32_t* pool, void* stream) {
  CSA2_TRY(check_cache(cache, false, false));
  if (blockmax == nullptr || pool == nullptr) return fail(CSA2_ERR_ARG, "blockmax and pool must be set");
  if (hist != nullptr && !aligned(hist, 16)) return fail(CSA2_ERR_ARG, "hist must be 16-byte aligned");
  if (pool_blocks < 1 || pool_blocks > kMaxPool)
    return fail(CSA2_ERR_SHAPE, "pool_blocks %d outside [1, %d]", pool_blocks, kMaxPool);
  const long long nblk = (capacity_of(cache) + csa2::kBlock - 1) / csa2::kBlock;
  if (nblk > kMaxPoolSelectBlocks)
    return fail(CSA2_ERR_SHAPE, "request capacity %lld positions exceeds the pool-select limit of %lld",
                capacity_of(cache), kMaxPoolSelectBlocks * csa2::kBlock);
  DeviceInfo d;
  CSA2_TRY(device_info(&d));
  // Without a histogram the radix passes scan every key: 16 CTAs above
  // 524,288 positions halve the keys per CTA.  With one, the passes only
  // touch the keys of the threshold's bin, and 8 CTAs (up to 16,384 keys
  // each) halve the cost of each pass's exchange instead.
  const long long per_cta = 16384;
  const int cluster = (nblk <= 4LL * per_cta || (hist != nullptr && nblk <= 8LL * per_cta)) ? 8 : 16;
  const cudaError_t e = csa2::launch_pool_select(*cache, blockmax, hist, pool_blocks, pool, cluster,
                                                 static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "pool_select launch");
}

csa2_status csa2_reindex(const csa2_cache* cache, csa2_mode mode, const int32_t* pool, int32_t pool_blocks,
                         const float* q, const float* w, const float* full_scores, const int32_t* prev_topk,
                         int32_t k, int32_t* topk, void* stream) {
  CSA2_TRY(check_cache(cache, false, mode != CSA2_REUSE));
  if (k < 1 || k > kMaxK) return fail(CSA2_ERR_SHAPE, "k %d outside [1, %d]", k, kMaxK);
  if (topk == nullptr) return fail(CSA2_ERR_ARG, "topk must be set");
  if (mode != CSA2_FULL && mode != CSA2_REINDEX && mode != CSA2_REUSE)
    return fail(CSA2_ERR_ARG, "unknown mode %d", static_cast<int>(mode));
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (mode == CSA2_REUSE) {
    if (prev_topk == nullptr) return fail(CSA2_ERR_ARG, "REUSE needs prev_topk");
    if (prev_topk == topk) return CSA2_OK;
    DeviceInfo d;
    CSA2_TRY(device_info(&d));
    const cudaError_t e = csa2::launch_copy_topk(prev_topk, topk, static_cast<long long>(cache->batch) * k, s);
    return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "reuse copy launch");
  }
  const float* stored = mode == CSA2_FULL ? full_scores : nullptr;
  if (stored == nullptr && (q == nullptr || w == nullptr || !aligned(q, 16)))
    return fail(CSA2_ERR_ARG, "re-scoring needs q (16-byte aligned) and w");
  int max_blocks;
  if (pool != nullptr) {
    if (pool_blocks < 1 || pool_blocks > kMaxPool)
      return fail(CSA2_ERR_SHAPE, "pool_blocks %d outside [1, %d]", pool_blocks, kMaxPool);
    max_blocks = (pool_blocks + csa2::kReindexPoolCluster - 1) / csa2::kReindexPoolCluster;
  } else {
    if (capacity_of(cache) > kMaxFlatPositions)
      return fail(CSA2_ERR_SHAPE, "Top-k without a pool supports request capacity <= %lld positions (got %lld)",
                  kMaxFlatPositions, capacity_of(cache));
    const long long nblk = (capacity_of(cache) + csa2::kBlock - 1) / csa2::kBlock;
    max_blocks = static_cast<int>((nblk + 7) / 8);
  }
  DeviceInfo d;
  CSA2_TRY(device_info(&d));
  CUtensorMap map;
  CSA2_TRY(encode_ik_map(cache, csa2::kBlock, &map));
  const cudaError_t e = csa2::launch_reindex(*cache, pool, pool_blocks, q, w, stored, k, topk, map, max_blocks,
                                             g_wait_limit_ns, s);
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "reindex launch");
}

size_t csa2_reindex_layers_workspace_bytes(int32_t batch, int32_t n_layers, int32_t pool_blocks) {
  return csa2::rescore_workspace_bytes(batch, n_layers, pool_blocks);
}

static csa2_status reindex_layers_impl(const csa2_cache* cache, const csa2_ik4* ik4, int32_t n_layers, const int32_t* pool,
                                int32_t pool_blocks, const float* const* q, const float* const* w, int32_t k,
                                int32_t* const* topk, void* workspace, size_t workspace_bytes, void* stream) {
  CSA2_TRY(check_cache(cache, false, ik4 == nullptr));
  if (ik4 != nullptr) CSA2_TRY(check_ik4(ik4));
  const int max_layers = ik4 != nullptr ? 4 : CSA2_MAX_SCORE_LAYERS;
  if (n_layers < 1 || n_layers > max_layers)
    return fail(CSA2_ERR_SHAPE, "n_layers %d outside [1, %d]", n_layers, max_layers);
  if (pool_blocks < 1 || pool_blocks > kMaxPool)
    return fail(CSA2_ERR_SHAPE, "pool_blocks %d outside [1, %d]", pool_blocks, kMaxPool);
  if (k < 1 || k > kMaxK) return fail(CSA2_ERR_SHAPE, "k %d outside [1, %d]", k, kMaxK);
  if (pool == nullptr || q == nullptr || w == nullptr || topk == nullptr)
    return fail(CSA2_ERR_ARG, "pool, q, w and topk must be set");
  for (int l = 0; l < n_layers; ++l)
    if (q[l] == nullptr || w[l] == nullptr || topk[l] == nullptr || !aligned(q[l], 16))
      return fail(CSA2_ERR_ARG, "layer %d: q (16-byte aligned), w and topk must be set", l);
  if (workspace == nullptr || !aligned(workspace, 16))
    return fail(CSA2_ERR_ARG, "workspace must be set and 16-byte aligned");
  const size_t need = csa2::rescore_workspace_bytes(cache->batch, n_layers, pool_blocks);
  if (workspace_bytes < need)
    return fail(CSA2_ERR_SHAPE, "workspace_bytes %zu < %zu (csa2_reindex_layers_workspace_bytes)", workspace_bytes,
                need);
  DeviceInfo d;
  CSA2_TRY(device_info(&d));
  CUtensorMap map;
  if (ik4 != nullptr)
    CSA2_TRY(encode_rows_map(ik4->codes, static_cast<long long>(cache->num_pages) * cache->page_size,
                             CSA2_IK4_CODE_BYTES, csa2::kBlock, CU_TENSOR_MAP_SWIZZLE_64B, &map));
  else
    CSA2_TRY(encode_ik_map(cache, csa2::kBlock, &map));
  const cudaError_t e =
      csa2::launch_rescore_layers(*cache, ik4 != nullptr ? ik4->scales : nullptr, n_layers, pool, pool_blocks, q, w, k,
                                  topk, workspace, map, d.sms, g_wait_limit_ns, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "reindex_layers launch");
}

csa2_status csa2_reindex_layers(const csa2_cache* cache, int32_t n_layers, const int32_t* pool, int32_t pool_blocks,
                                const float* const* q, const float* const* w, int32_t k, int32_t* const* topk,
                                void* workspace, size_t workspace_bytes, void* stream) {
  return reindex_layers_impl(cache, nullptr, n_layers, pool, pool_blocks, q, w, k, topk, workspace, workspace_bytes,
                             stream);
}

csa2_status csa2_reindex_layers_fp4(const csa2_cache* cache, const csa2_ik4* ik4, int32_t n_layers,
                                    const int32_t* pool, int32_t pool_blocks, const float* const* q,
                                    const float* const* w, int32_t k, int32_t* const* topk, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  if (ik4 == nullptr) return fail(CSA2_ERR_ARG, "ik4 must be set");
  return reindex_layers_impl(cache, ik4, n_layers, pool, pool_blocks, q, w, k, topk, workspace, workspace_bytes,
                             stream);
}

csa2_status csa2_pool_candidates(const csa2_cache* shard, const float* blockmax, const int32_t* pool,
                                 int32_t pool_blocks, int32_t block_offset, float* values, int32_t* ids,
                                 void* stream) {
  CSA2_TRY(check_cache(shard, false, false));
  if (blockmax == nullptr || pool == nullptr || values == nullptr || ids == nullptr)
    return fail(CSA2_ERR_ARG, "blockmax, pool, values and ids must be set");
  if (pool_blocks < 1 || pool_blocks > kMaxPool)
    return fail(CSA2_ERR_SHAPE, "pool_blocks %d outside [1, %d]", pool_blocks, kMaxPool);
  if (block_offset < 0 ||
      static_cast<long long>(block_offset) + (capacity_of(shard) + csa2::kBlock - 1) / csa2::kBlock >= (1LL << 31))
    return fail(CSA2_ERR_SHAPE, "block_offset %d: global block ids must lie in [0, 2^31)", block_offset);
  DeviceInfo d;
  CSA2_TRY(device_info(&d));
  const cudaError_t e = csa2::launch_pool_candidates(*shard, blockmax, pool, pool_blocks, block_offset, values, ids,
                                                     static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "pool_candidates launch");
}

csa2_status csa2_pool_merge(int32_t n_shards, int32_t batch, int32_t pool_blocks, const float* values,
                            const int32_t* ids, int32_t* pool, void* stream) {
  if (n_shards < 1 || n_shards > CSA2_MAX_SHARDS)
    return fail(CSA2_ERR_SHAPE, "n_shards %d outside [1, %d]", n_shards, CSA2_MAX_SHARDS);
  if (batch < 1 || batch > kMaxBatch) return fail(CSA2_ERR_SHAPE, "batch %d outside [1, %d]", batch, kMaxBatch);
  if (pool_blocks < 1 || pool_blocks > kMaxPool)
    return fail(CSA2_ERR_SHAPE, "pool_blocks %d outside [1, %d]", pool_blocks, kMaxPool);
  if (static_cast<long long>(n_shards) * pool_blocks > 32768)
    return fail(CSA2_ERR_SHAPE, "n_shards * pool_blocks = %lld exceeds 32768 candidates",
                static_cast<long long>(n_shards) * pool_blocks);
  if (values == nullptr || ids == nullptr || pool == nullptr)
    return fail(CSA2_ERR_ARG, "values, ids and pool must be set");
  DeviceInfo d;
  CSA2_TRY(device_info(&d));
  const cudaError_t e =
      csa2::launch_pool_merge(n_shards, batch, pool_blocks, values, ids, pool, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "pool_merge launch");
}

csa2_status csa2_sparse_attn(const csa2_cache* cache, int32_t n_queries, const int32_t* q_req, const int32_t* topk,
                             int32_t k, const uint16_t* q, int32_t H, float scale, uint16_t* out, void* stream) {
  const uint16_t* qs[1] = {q};
  uint16_t* os[1] = {out};
  const int32_t* ts[1] = {topk};
  return sparse_attn_impl(cache, 1, n_queries, q_req, ts, k, qs, H, scale, os, stream);
}

csa2_status csa2_swa_append(const csa2_cache* cache, int32_t window, uint8_t* swa_codes, uint8_t* swa_exp,
                            int32_t n_rows, const float* x, const int32_t* req, const int32_t* pos, void* stream) {
  CSA2_TRY(check_cache(cache, false, false));
  if (window < 1 || window > CSA2_SWA_MAX_WINDOW)
    return fail(CSA2_ERR_SHAPE, "window %d outside [1, %d]", window, CSA2_SWA_MAX_WINDOW);
  if (n_rows < 0) return fail(CSA2_ERR_SHAPE, "n_rows %d < 0", n_rows);
  if (n_rows == 0) return CSA2_OK;
  if (swa_codes == nullptr || swa_exp == nullptr || x == nullptr || pos == nullptr || !aligned(swa_codes, 16) ||
      !aligned(x, 16))
    return fail(CSA2_ERR_ARG, "swa_codes (16-byte aligned), swa_exp, x (16-byte aligned) and pos must be set");
  if (req == nullptr && n_rows > cache->batch)
    return fail(CSA2_ERR_SHAPE, "without req, n_rows (%d) must not exceed batch (%d)", n_rows, cache->batch);
  DeviceInfo d;
  CSA2_TRY(device_info(&d));
  const cudaError_t e = csa2::launch_swa_append(*cache, window, swa_codes, swa_exp, n_rows, x, req, pos,
                                                static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "swa_append launch");
}

csa2_status csa2_sparse_attn_swa(const csa2_cache* cache, int32_t n_queries, const int32_t* q_req,
                                 const int32_t* topk, int32_t k, const uint8_t* swa_codes, const uint8_t* swa_exp,
                                 int32_t window, const int32_t* q_pos, const uint16_t* q, int32_t H, float scale,
                                 uint16_t* out, void* stream) {
  CSA2_TRY(check_cache(cache, true, false));
  if (window < 1 || window > CSA2_SWA_MAX_WINDOW)
    return fail(CSA2_ERR_SHAPE, "window %d outside [1, %d]", window, CSA2_SWA_MAX_WINDOW);
  if (swa_codes == nullptr || swa_exp == nullptr || q_pos == nullptr || !aligned(swa_codes, 16))
    return fail(CSA2_ERR_ARG, "swa_codes (16-byte aligned), swa_exp and q_pos must be set");
  if (n_queries < 0) return fail(CSA2_ERR_SHAPE, "n_queries %d < 0", n_queries);
  if (n_queries == 0) return CSA2_OK;
  if (q_req == nullptr && n_queries > cache->batch)
    return fail(CSA2_ERR_SHAPE, "without q_req, n_queries (%d) must not exceed batch (%d)", n_queries, cache->batch);
  if (H != 16 && H != 32 && H != 64) return fail(CSA2_ERR_SHAPE, "H %d not in {16, 32, 64}", H);
  if (k < 1 || k > kMaxK) return fail(CSA2_ERR_SHAPE, "k %d outside [1, %d]", k, kMaxK);
  if (topk == nullptr || q == nullptr || out == nullptr || !aligned(q, 16) || !aligned(out, 16))
    return fail(CSA2_ERR_ARG, "topk, q and out (16-byte aligned) must be set");
  DeviceInfo d;
  CSA2_TRY(device_info(&d));
  const uint16_t* qs[1] = {q};
  uint16_t* os[1] = {out};
  const int32_t* ts[1] = {topk};
  const cudaError_t e = csa2::launch_sparse_attn(*cache, 1, n_queries, q_req, ts, k, qs, H, scale, os,
                                                 static_cast<cudaStream_t>(stream), swa_codes, swa_exp, q_pos,
                                                 window);
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "sparse_attn_swa launch");
}

csa2_status csa2_sparse_attn_layers(const csa2_cache* cache, int32_t n_layers, int32_t n_queries,
                                    const int32_t* q_req, const int32_t* const* topk, int32_t k, const uint16_t* const* q,
                                    int32_t H, float scale, uint16_t* const* out, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  return sparse_attn_impl(cache, n_layers, n_queries, q_req, topk, k, q, H, scale, out, stream, workspace,
                          workspace_bytes);
}

size_t csa2_attn_workspace_bytes(int32_t n_layers, int32_t n_queries, int32_t H) {
  if (n_layers < 0 || n_queries < 0 || H < 0) return 0;
  return csa2::attn_workspace_bytes(n_layers, n_queries, H);
}

size_t csa2_prefill_workspace_bytes(int32_t n_queries) { return csa2::prefill_workspace_bytes(n_queries); }

csa2_status csa2_prefill_index(const csa2_cache* cache, int32_t req, int32_t n_queries, const int32_t* q_pos,
                               int32_t ratio, const float* q, const float* w, int32_t k, int32_t* topk,
                               void* workspace, size_t workspace_bytes, void* stream) {
  CSA2_TRY(check_cache(cache, false, true));
  if (req < 0 || req >= cache->batch) return fail(CSA2_ERR_SHAPE, "req %d outside [0, %d)", req, cache->batch);
  if (n_queries < 0 || n_queries > kMaxPrefillQueries)
    return fail(CSA2_ERR_SHAPE, "n_queries %d outside [0, %d]", n_queries, kMaxPrefillQueries);
  if (n_queries == 0) return CSA2_OK;
  if (ratio < 1) return fail(CSA2_ERR_SHAPE, "ratio %d < 1", ratio);
  if (k < 1 || k > CSA2_PREFILL_MAX_K) return fail(CSA2_ERR_SHAPE, "k %d outside [1, %d]", k, CSA2_PREFILL_MAX_K);
  if (q_pos == nullptr || q == nullptr || w == nullptr || topk == nullptr || !aligned(q, 16))
    return fail(CSA2_ERR_ARG, "q_pos, q (16-byte aligned), w and topk must be set");
  if (workspace == nullptr || !aligned(workspace, 16))
    return fail(CSA2_ERR_ARG, "workspace must be set and 16-byte aligned");
  if (workspace_bytes < csa2::prefill_workspace_bytes(n_queries))
    return fail(CSA2_ERR_SHAPE, "workspace of %zu bytes, %zu needed", workspace_bytes,
                csa2::prefill_workspace_bytes(n_queries));
  DeviceInfo d;
  CSA2_TRY(device_info(&d));
  CUtensorMap map;
  CSA2_TRY(encode_ik_map(cache, csa2::kTile, &map));
  const cudaError_t e = csa2::launch_prefill_index(*cache, req, n_queries, q_pos, ratio, q, w, k, topk, workspace,
                                                   map, g_wait_limit_ns, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "prefill_index launch");
}

csa2_status csa2_prefill_index_static(const csa2_cache* cache, int32_t req, int32_t n_queries,
                                      const int32_t* q_pos, int32_t ratio, const float* q, const float* w,
                                      int32_t k, int32_t* topk, void* stream) {
  if (n_queries > CSA2_PREFILL_STATIC_MAX_QUERIES)
    return fail(CSA2_ERR_SHAPE, "n_queries %d above the static scratch limit of %d", n_queries,
                CSA2_PREFILL_STATIC_MAX_QUERIES);
  if (n_queries <= 0) return csa2_prefill_index(cache, req, n_queries, q_pos, ratio, q, w, k, topk, nullptr, 0, stream);
  // the host-side checks of csa2_prefill_index, before the device is touched
  CSA2_TRY(check_cache(cache, false, true));
  if (req < 0 || req >= cache->batch) return fail(CSA2_ERR_SHAPE, "req %d outside [0, %d)", req, cache->batch);
  if (ratio < 1) return fail(CSA2_ERR_SHAPE, "ratio %d < 1", ratio);
  if (k < 1 || k > CSA2_PREFILL_MAX_K) return fail(CSA2_ERR_SHAPE, "k %d outside [1, %d]", k, CSA2_PREFILL_MAX_K);
  if (q_pos == nullptr || q == nullptr || w == nullptr || topk == nullptr || !aligned(q, 16))
    return fail(CSA2_ERR_ARG, "q_pos, q (16-byte aligned), w and topk must be set");
  DeviceInfo d;
  CSA2_TRY(device_info(&d));
  void* scratch = nullptr;
  const cudaError_t e = csa2::static_prefill_scratch(&scratch);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(prefill scratch)");
  return csa2_prefill_index(cache, req, n_queries, q_pos, ratio, q, w, k, topk, scratch,
                            csa2::prefill_workspace_bytes(n_queries), stream);
}

csa2_status csa2_get_error(const csa2_cache* cache, int32_t* out, void* stream) {
  if (cache == nullptr || cache->err_word == nullptr || out == nullptr)
    return fail(CSA2_ERR_ARG, "cache, cache.err_word and out must be set");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  e = cudaMemcpy(out, cache->err_word, 4 * sizeof(int32_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(err_word)");
  return static_cast<csa2_status>(out[0]);
}

const char* csa2_status_string(csa2_status s) {
  switch (s) {
    case CSA2_OK: return "ok";
    case CSA2_ERR_ARG: return "invalid argument";
    case CSA2_ERR_SHAPE: return "unsupported shape";
    case CSA2_ERR_CUDA: return "CUDA runtime error";
    case CSA2_ERR_DEVICE_BOUNDS: return "out-of-range page or position found on the device";
    case CSA2_ERR_TIMEOUT: return "a pipeline wait on the device gave up";
    case CSA2_ERR_UNSUPPORTED: return "unsupported device or feature";
  }
  return "unknown status";
}

const char* csa2_last_error_message(void) { return g_msg; }

void csa2_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns = ns; }

}  // extern "C"
