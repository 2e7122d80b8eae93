// Host-side launchers of the CSA2 kernels (internal to libcsa2.so).  Each
// returns the launch's cudaError_t; argument validation happens before, in
// csa2_api.cu.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

#include "../../include/csa2.h"

namespace csa2 {

// Unique id of the calling thread's current CUDA context (the current
// device's primary context is made current first when none is).
cudaError_t current_context_id(unsigned long long* id);

// Set-up that belongs to one CUDA context (kernel attributes, the address of a
// __device__ array), run once in each context the library is used in.
class ContextMemo {
 public:
  // *value = the value stored for the current context; make(value) computes
  // and stores it the first time.
  template <class Make>
  cudaError_t get(void** value, Make make) {
    unsigned long long id = 0;
    bool found = false;
    cudaError_t e = lookup(&id, &found, value);
    if (e != cudaSuccess || found) return e;
    e = make(value);
    if (e == cudaSuccess) store(id, *value);
    return e;
  }
  // run() once per context (set-up without a value).
  template <class Run>
  cudaError_t once(Run run) {
    void* v = nullptr;
    return get(&v, [&](void** out) {
      *out = nullptr;
      return run();
    });
  }

 private:
  cudaError_t lookup(unsigned long long* id, bool* found, void** value);
  void store(unsigned long long id, void* value);
  static constexpr int kSlots = 64;
  std::mutex mu_;
  unsigned long long ids_[kSlots] = {};
  void* vals_[kSlots] = {};
  int n_ = 0, next_ = 0;
};

cudaError_t launch_append(const csa2_cache& cache, int n_rows, const float* kv_new, const float* ik_new,
                          const int32_t* req, const int32_t* pos, cudaStream_t stream);

cudaError_t launch_compress_append(const csa2_cache& cache, int n_entries, int m, const float* kv_tok,
                                   const float* ik_tok, const int32_t* req, const int32_t* pos, cudaStream_t stream);

size_t index_full_smem_bytes();
cudaError_t launch_index_full(const csa2_cache& cache, const float* q, const float* w, float* blockmax,
                              float* scores, uint32_t* hist, const CUtensorMap& ik_map, int whole_units, int num_sms,
                              uint64_t wait_ns, cudaStream_t stream);

// FP4 indexer: scan and quantise-on-append.
size_t index_full_fp4_smem_bytes();
cudaError_t launch_index_full_fp4(const csa2_cache& cache, const uint8_t* ik4_scales, const float* q, const float* w,
                                  float* blockmax, float* scores, uint32_t* hist, const CUtensorMap& code_map,
                                  int whole_units, int num_sms, uint64_t wait_ns, cudaStream_t stream);
cudaError_t launch_append_ik4(const csa2_cache& cache, uint8_t* codes, uint8_t* scales, int n_rows,
                              const float* ik_new, const int32_t* req, const int32_t* pos, cudaStream_t stream);

cudaError_t launch_pool_select(const csa2_cache& cache, const float* blockmax, uint32_t* hist, int pool_blocks,
                               int32_t* pool, int cluster, cudaStream_t stream);

// Top-k of n_layers layers over the pool: one scoring launch (every pool
// block gathered once, all layers in one MMA) and one select launch.
size_t rescore_workspace_bytes(long long batch, int n_layers, int pool_blocks);
// ik4_scales != nullptr: the FP4 indexer (blk_map over its codes, n_layers <= 4).
cudaError_t launch_rescore_layers(const csa2_cache& cache, const uint8_t* ik4_scales, int n_layers,
                                  const int32_t* pool, int pool_blocks, const float* const* q, const float* const* w,
                                  int k, int32_t* const* topk, void* workspace, const CUtensorMap& blk_map,
                                  int num_sms, uint64_t wait_ns, cudaStream_t stream);

constexpr int kReindexPoolCluster = 16;   // CTAs per request when re-scoring a pool
cudaError_t launch_reindex(const csa2_cache& cache, const int32_t* pool, int pool_blocks, const float* q,
                           const float* w, const float* full_scores, int k, int32_t* topk,
                           const CUtensorMap& ik_blk_map, int cands_per_cta, uint64_t wait_ns, cudaStream_t stream);

size_t prefill_workspace_bytes(long long n_queries);
constexpr int kStaticPrefillMaxQueries = CSA2_PREFILL_STATIC_MAX_QUERIES;
// Device address (current device) of the static candidate-list array of
// csa2_prefill_index_static; looked up once per device.
cudaError_t static_prefill_scratch(void** addr);
cudaError_t launch_prefill_index(const csa2_cache& cache, int req, int n_queries, const int32_t* q_pos, int ratio,
                                 const float* q, const float* w, int k, int32_t* topk, void* workspace,
                                 const CUtensorMap& ik_map, uint64_t wait_ns, cudaStream_t stream);

// Sharded pool: a slice's (block max, global id) candidates, and the exact
// merge of G slices' candidates ([G][batch][P] each).
cudaError_t launch_pool_candidates(const csa2_cache& cache, const float* blockmax, const int32_t* pool, int P,
                                   int block_offset, float* values, int32_t* ids, cudaStream_t stream);
cudaError_t launch_pool_merge(int n_shards, int batch, int P, const float* values, const int32_t* ids, int32_t* pool,
                              cudaStream_t stream);

cudaError_t launch_copy_topk(const int32_t* src, int32_t* dst, long long n, cudaStream_t stream);

// topk[l] / q[l] / out[l] (host arrays of device pointers): Top-k, query and
// output of layer l of n_layers layers (layers may share a Top-k).
// swa_codes == nullptr: no sliding window; else the window of `window`
// tokens ending at q_pos[i] is merged into query i's softmax.
cudaError_t launch_sparse_attn(const csa2_cache& cache, int n_layers, int n_queries, const int32_t* q_req,
                               const int32_t* const* topk, int k, const uint16_t* const* q, int H, float scale,
                               uint16_t* const* out, cudaStream_t stream, const uint8_t* swa_codes = nullptr,
                               const uint8_t* swa_exp = nullptr, const int32_t* q_pos = nullptr, int window = 0,
                               void* xchg = nullptr);
size_t attn_workspace_bytes(long long n_layers, long long n_queries, int H);
cudaError_t launch_swa_append(const csa2_cache& cache, int window, uint8_t* swa_codes, uint8_t* swa_exp, int n_rows,
                              const float* x, const int32_t* req, const int32_t* pos, cudaStream_t stream);

}  // namespace csa2
