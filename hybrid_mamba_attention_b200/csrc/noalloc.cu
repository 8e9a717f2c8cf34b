// Scratch of hspec_attn_paged_block_noalloc: a fixed device array, so that callers
// that cannot allocate device memory still get the split-KV partials somewhere.
//
// The array lives in this file's module alone.  Under CUDA's lazy module loading
// (the default) the module, and with it the array's HSPEC_NOALLOC_SCRATCH_BYTES of
// device memory, is loaded the first time this file's address lookup runs on a
// device, i.e. at the first allocation-free call there; with
// CUDA_MODULE_LOADING=EAGER it is loaded when the context is created.  Either way it
// stays until the context is destroyed.
//
// On the host, `g_noalloc_scratch` names a host-side shadow, not device memory, so
// host code never passes it to a kernel: the device address is looked up below, once
// per CUDA context, with the caller's device current.
#include <mutex>
#include <vector>

#include "../../include/hspec.h"
#include "common.cuh"

static __device__ __align__(256) unsigned char g_noalloc_scratch[HSPEC_NOALLOC_SCRATCH_BYTES];

namespace hspec {

void* current_context();

// Device address of g_noalloc_scratch in the current context; NULL (message
// recorded) if the lookup fails.  The first call in a context does the lookup.
void* noalloc_scratch_address() {
  struct Entry {
    void* ctx;
    void* addr;
  };
  static std::mutex mu;
  static std::vector<Entry> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    set_error("allocation-free attention: no current CUDA device");
    return nullptr;
  }
  void* ctx = current_context();
  std::lock_guard<std::mutex> lock(mu);
  if (ctx)
    for (const Entry& e : cache)
      if (e.ctx == ctx) return e.addr;
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) {
    cudaGetLastError();
    if (e == cudaErrorMemoryAllocation)
      set_error("allocation-free attention: device %d has no room for the library's %zu-byte static scratch "
                "(reserved when its module loads; make the first call before handing the memory to a KV pool, "
                "or load modules eagerly): %s",
                dev, (size_t)HSPEC_NOALLOC_SCRATCH_BYTES, cudaGetErrorString(e));
    else
      set_error("allocation-free attention: cudaGetSymbolAddress(scratch) failed on device %d: %s", dev,
                cudaGetErrorString(e));
    return nullptr;
  }
  if (!ctx) ctx = current_context();  // the lookup made the device's primary context current
  if (ctx) cache.push_back({ctx, p});
  return p;
}

}  // namespace hspec
