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

#include "context_symbol.h"
#include "mamba_mixer.h"

namespace mm_internal {
void set_last_error(const char* msg);  // mamba_mixer.cu: the message mamba_last_error returns
}

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(2) << 20;  // 2 MiB per device

// Scratch for the forward's workspace: a 256-byte header (status word, chunk-unit counter)
// followed by the carried states of the time chunks and their flags.  The forward resets
// the counter and flags itself (cudaMemsetAsync on the stream, no allocation) and writes
// every carried state before reading it, so nothing else has to be cleared between calls.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

int noalloc_fail(int code, const char* msg) {
  mm_internal::set_last_error(msg);
  return code;
}

// The scratch array's device address in the current context (looked up once per context).
int scratch_for_current_context(void** out, const char* who, char* why, size_t why_len) {
  return mm_host::symbol_in_context(reinterpret_cast<const void*>(&g_noalloc_scratch), out, who,
                                    why, why_len) == 0 ? MAMBA_OK : MAMBA_ERR_CUDA;
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
