// mamba_mixer_fwd_noalloc: the fused forward for callers that cannot allocate device
// memory, with its scratch space held in this file's static device array.
//
// Some callers have no way to hand the library a workspace: plugin hosts that pass in the
// input and output buffers but expose no allocator, code running inside an allocator's
// own callback (where calling cudaMalloc would re-enter it), and latency-critical paths
// that must not call cudaMalloc because it can synchronize the whole device.  This entry
// point takes the same inputs and outputs as mamba_mixer_fwd and uses instead a
// library-owned scratch array of kNoAllocScratchBytes per device (held by every GPU that
// loads the library, until the process exits).  It allocates nothing.
// mamba_mixer_noalloc_check reads and clears that array's status word.

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "mamba_mixer.h"

namespace mm_internal {
void set_last_error(const char* msg);  // mamba_mixer.cu: the message mamba_last_error returns
}

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(2) << 20;  // 2 MiB per device

// Scratch for the forward's workspace: a 256-byte header (status word) followed by the
// carry aggregates of the time chunks.  Zero at module load; the forward writes every
// aggregate before reading it, so nothing has to be cleared between calls.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// The array's device address belongs to a CUDA context, not to a device: a second context
// on the same device (cuCtxCreate) or a context re-created after a reset has its own copy
// of the module and so its own address.  The lookup is therefore cached per context, keyed
// by the context's unique id (cuCtxGetId: unique for the life of the process, never reused).
// In host code the symbol itself is only a host-side stand-in, never a device address.
struct CtxEntry {
  unsigned long long ctx_id;
  void* ptr;
};
constexpr int kCacheEntries = 64;
CtxEntry g_cache[kCacheEntries] = {};
int g_cache_next = 0;
std::mutex g_cache_mu;

using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

CtxGetIdFn ctx_get_id_fn() {
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

int noalloc_fail(int code, const char* msg) {
  mm_internal::set_last_error(msg);
  return code;
}

// Looks up (or finds cached) the scratch array's address in the current context.  The
// lookup itself (cudaGetSymbolAddress) makes the device's primary context current when the
// thread has none yet.  On failure writes the reason to `why`.
int scratch_for_current_context(void** out, const char* who, char* why, size_t why_len) {
  const CtxGetIdFn get_id = ctx_get_id_fn();
  unsigned long long id = 0;
  bool have_id = get_id && get_id(nullptr, &id) == CUDA_SUCCESS;
  if (have_id) {
    std::lock_guard<std::mutex> lock(g_cache_mu);
    for (const CtxEntry& e : g_cache)
      if (e.ptr && e.ctx_id == id) {
        *out = e.ptr;
        return MAMBA_OK;
      }
  }
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || !p) {
    snprintf(why, why_len, "%s: cudaGetSymbolAddress of the scratch array failed: %s", who,
             e != cudaSuccess ? cudaGetErrorString(e) : "null address");
    return MAMBA_ERR_CUDA;
  }
  // the lookup may just have made a primary context current: take its id now
  if (!have_id) have_id = get_id && get_id(nullptr, &id) == CUDA_SUCCESS;
  if (have_id) {
    std::lock_guard<std::mutex> lock(g_cache_mu);
    g_cache[g_cache_next] = CtxEntry{id, p};
    g_cache_next = (g_cache_next + 1) % kCacheEntries;
  }
  *out = p;
  return MAMBA_OK;
}

}  // namespace

extern "C" MAMBA_API int mamba_mixer_fwd_noalloc(
    const mamba_dims* dims, const void* xp, const void* z, const void* dt_raw, const void* B,
    const void* C, const float* A_log, const float* D, const float* conv_w, const float* conv_b,
    const float* dt_bias, void* y, float* h_out, void* conv_state_out, void* cuda_stream) {
  const size_t need = mamba_mixer_fwd_workspace_bytes(dims);
  if (need == 0)  // unsupported dims: let the full entry point report why
    return mamba_mixer_fwd(dims, xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, y,
                           h_out, conv_state_out, nullptr, 0, cuda_stream);
  if (need > kNoAllocScratchBytes) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "mamba_mixer_fwd_noalloc: these sizes need %zu bytes of scratch, more than its "
             "fixed %zu; use mamba_mixer_fwd with a caller-allocated workspace",
             need, kNoAllocScratchBytes);
    return noalloc_fail(MAMBA_ERR_WORKSPACE, msg);
  }
  void* scratch = nullptr;
  char why[256];
  if (scratch_for_current_context(&scratch, "mamba_mixer_fwd_noalloc", why, sizeof(why)) != MAMBA_OK)
    return noalloc_fail(MAMBA_ERR_CUDA, why);
  return mamba_mixer_fwd(dims, xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, y, h_out,
                         conv_state_out, scratch, kNoAllocScratchBytes, cuda_stream);
}

extern "C" MAMBA_API int mamba_mixer_noalloc_check(void* cuda_stream) {
  void* scratch = nullptr;
  char why[256];
  if (scratch_for_current_context(&scratch, "mamba_mixer_noalloc_check", why, sizeof(why)) != MAMBA_OK)
    return noalloc_fail(MAMBA_ERR_CUDA, why);
  return mamba_mixer_check(scratch, cuda_stream);
}
