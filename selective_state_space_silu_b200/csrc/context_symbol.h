// Device address of a file-scope __device__ variable in the calling thread's current CUDA
// context.  The address belongs to a context, not to a device: a second context on the same
// device (cuCtxCreate) or a context re-created after a reset has its own copy of the module
// and so its own address.  Lookups (cudaGetSymbolAddress, a host-side query that allocates
// nothing) are cached per (context, variable), keyed by the context's unique id (cuCtxGetId:
// unique for the life of the process, never reused).  In host code the variable's name is
// only a host-side stand-in, never a device address.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

namespace mm_host {

using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

inline CtxGetIdFn ctx_get_id_fn() {
  static CtxGetIdFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<CtxGetIdFn>(nullptr);
    return reinterpret_cast<CtxGetIdFn>(p);
  }();
  return fn;
}

// Looks up (or finds cached) `symbol`'s device address in the current context; the lookup
// makes the device's primary context current on a thread that has none.  Returns 0, or a
// nonzero code with the reason (prefixed by `who`) in `why`.
inline int symbol_in_context(const void* symbol, void** out, const char* who, char* why,
                             size_t why_len) {
  struct Entry {
    unsigned long long ctx_id;
    const void* symbol;
    void* ptr;
  };
  constexpr int kEntries = 64;
  static Entry cache[kEntries] = {};
  static int next = 0;
  static std::mutex mu;
  const CtxGetIdFn get_id = ctx_get_id_fn();
  unsigned long long id = 0;
  bool have_id = get_id && get_id(nullptr, &id) == CUDA_SUCCESS;
  if (have_id) {
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& e : cache)
      if (e.ptr && e.ctx_id == id && e.symbol == symbol) {
        *out = e.ptr;
        return 0;
      }
  }
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, symbol);
  if (e != cudaSuccess || !p) {
    snprintf(why, why_len, "%s: cudaGetSymbolAddress failed: %s", who,
             e != cudaSuccess ? cudaGetErrorString(e) : "null address");
    return 1;
  }
  if (!have_id) have_id = get_id && get_id(nullptr, &id) == CUDA_SUCCESS;
  if (have_id) {
    std::lock_guard<std::mutex> lock(mu);
    cache[next] = Entry{id, symbol, p};
    next = (next + 1) % kEntries;
  }
  *out = p;
  return 0;
}

}  // namespace mm_host
