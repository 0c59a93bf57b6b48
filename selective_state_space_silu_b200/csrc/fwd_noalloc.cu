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

#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "mamba_mixer.h"

namespace mm_internal {
void set_last_error(const char* msg);  // mamba_mixer.cu: the message mamba_last_error returns
}

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(2) << 20;  // 2 MiB per device
constexpr int kMaxDevices = 64;

// Scratch for the forward's workspace: a 256-byte header (status word) followed by the
// carry aggregates of the time chunks.  Zero at module load; the forward writes every
// aggregate before reading it, so nothing has to be cleared between calls.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on each device, looked up once per device with that
// device current.  In host code the symbol itself is only a host-side stand-in.
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

int noalloc_fail(int code, const char* msg) {
  mm_internal::set_last_error(msg);
  return code;
}

int scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MAMBA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) return MAMBA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
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
  if (scratch_for_current_device(&scratch) != MAMBA_OK)
    return noalloc_fail(MAMBA_ERR_CUDA,
                        "mamba_mixer_fwd_noalloc: cudaGetSymbolAddress of the scratch failed");
  return mamba_mixer_fwd(dims, xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, y, h_out,
                         conv_state_out, scratch, kNoAllocScratchBytes, cuda_stream);
}
