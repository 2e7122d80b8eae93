// Host-side bookkeeping per CUDA context.  Kernel attributes (dynamic shared
// memory size, cluster sizes) and the addresses of the library's __device__
// arrays belong to one context: a process that uses several devices, or whose
// context is destroyed and created again (cudaDeviceReset, a framework
// releasing the primary context), must set them up again in the new one.
// Contexts are told apart by the driver's unique context id, which is never
// reused within a process (a recreated context can get the old handle value,
// never the old id).
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "launch.h"

namespace csa2 {

namespace {
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_get_current = nullptr;
CtxGetIdFn g_get_id = nullptr;
std::once_flag g_once;

void* driver_entry(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return p;
}
}  // namespace

cudaError_t current_context_id(unsigned long long* id) {
  std::call_once(g_once, [] {
    g_get_current = reinterpret_cast<CtxGetCurrentFn>(driver_entry("cuCtxGetCurrent"));
    g_get_id = reinterpret_cast<CtxGetIdFn>(driver_entry("cuCtxGetId"));
  });
  if (g_get_current == nullptr || g_get_id == nullptr) return cudaErrorNotSupported;
  CUcontext ctx = nullptr;
  if (g_get_current(&ctx) != CUDA_SUCCESS) return cudaErrorInitializationError;
  if (ctx == nullptr) {
    // no context current on this thread yet: make the device's primary
    // context current, as the runtime's first call on the device would
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaSetDevice(dev);
    if (e != cudaSuccess) return e;
    if (g_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorInitializationError;
  }
  return g_get_id(ctx, id) == CUDA_SUCCESS ? cudaSuccess : cudaErrorInitializationError;
}

cudaError_t ContextMemo::lookup(unsigned long long* id, bool* found, void** value) {
  const cudaError_t e = current_context_id(id);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu_);
  *found = false;
  for (int i = 0; i < n_; ++i)
    if (ids_[i] == *id) {
      *found = true;
      *value = vals_[i];
      break;
    }
  return cudaSuccess;
}

void ContextMemo::store(unsigned long long id, void* value) {
  std::lock_guard<std::mutex> lk(mu_);
  for (int i = 0; i < n_; ++i)
    if (ids_[i] == id) {
      vals_[i] = value;
      return;
    }
  int slot;
  if (n_ < kSlots) {
    slot = n_++;
  } else {   // full: replace the oldest entry
    slot = next_;
    next_ = (next_ + 1) % kSlots;
  }
  ids_[slot] = id;
  vals_[slot] = value;
}

}  // namespace csa2
