// mamba2_ssd_fwd: host side of the Mamba2 scan (argument checks and the launch).

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>

#include "context_symbol.h"
#include "mamba2_ssd.h"
#include "ssd_kernel.cuh"
#include "ssd_step.cuh"
#include "ssd_layer.cuh"
#include "ssd_tc_kernel.cuh"

namespace mm_internal {
void set_last_error(const char* msg);  // mamba_mixer.cu: the message mamba_last_error returns
bool make_map4d_sw128(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                      uint64_t d3, uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3);
}

// The Mamba2 scan's status word: its tensor-core main pass waits on its own copies and
// products (bounded), and a wait that runs out is recorded here (one word per context;
// mamba2_ssd_check reads and clears it).
static __device__ __align__(256) int g_ssd_status[64];

namespace {

int ssd_fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  mm_internal::set_last_error(buf);
  return code;
}

int ssd_ok() {
  mm_internal::set_last_error("");
  return MAMBA_OK;
}

int need(const void* p, const char* name, bool required, size_t align) {
  if (!p) return required ? ssd_fail(MAMBA_ERR_INVALID_ARGUMENT, "%s is NULL", name) : MAMBA_OK;
  if (reinterpret_cast<uintptr_t>(p) % align)
    return ssd_fail(MAMBA_ERR_ALIGNMENT, "%s is not %zu-byte aligned", name, align);
  return MAMBA_OK;
}

struct Range {
  const void* p;
  size_t bytes;
  const char* name;
};

bool overlap(const Range& a, const Range& b) {
  if (!a.p || !b.p || !a.bytes || !b.bytes) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a.p), b0 = reinterpret_cast<uintptr_t>(b.p);
  return a0 < b0 + b.bytes && b0 < a0 + a.bytes;
}

// Time segments: with few (batch row, head) pairs, each pair's chunks are cut into
// segments that run as separate CTAs (a state pass over segments 0 .. nseg - 2 first).
// Measured (B200, 24 heads x 64, d_state 128): 8 x 2048 steps -> 1 segment, 125 us (2: 131,
// 3: 138); 2 x 8192 -> 6 segments, 129 us (3: 139, 8: 160).
struct SegPlan {
  int nseg, cps;
};

constexpr int64_t kSms = 148;

// Rows without document resets take the tensor-core passes (main pass: one CTA per SM, 10
// warps, 170 KB of shared memory for d_state 128 and 512 TMEM columns).
bool use_tc(const int32_t* seq_idx) { return seq_idx == nullptr; }

// Time segments.  One plan serves both passes (the workspace query does not know whether
// document ids will be given); it is set by the tensor-core passes, which take every row
// without document resets.  Their cost, measured on B200 (d_state 128, 64-step chunks): a
// main-pass CTA (one per SM) takes about (5.3 + c) x 1.675 us for c chunks, a state-pass CTA
// (two per SM) about c x 1.5 us.  The plan minimises the waves of both passes times those
// costs over 1..16 segments, the fewest segments on a tie.
SegPlan seg_plan(int64_t Bt, int64_t L, int64_t H) {
  const int64_t nchunks = (L + ssd::kQ - 1) / ssd::kQ;
  const int64_t pairs = Bt * H;
  if (nchunks <= 1 || pairs <= 0) return {1, int(nchunks > 0 ? nchunks : 1)};
  double best_cost = -1.0;
  int64_t best_n = 1, best_cps = nchunks;
  for (int64_t n = 1; n <= 16 && n <= nchunks; ++n) {
    const int64_t cps = (nchunks + n - 1) / n;
    const int64_t n_eff = (nchunks + cps - 1) / cps;
    const int64_t main_waves = (pairs * n_eff + kSms - 1) / kSms;
    const int64_t state_waves = n_eff > 1 ? (pairs * (n_eff - 1) + 2 * kSms - 1) / (2 * kSms) : 0;
    const double cost = double(main_waves) * (5.3 + double(cps)) * 1.675 +
                        double(state_waves) * double(cps) * 1.5;
    if (best_cost < 0.0 || cost < best_cost - 1e-9) {
      best_cost = cost;
      best_n = n_eff;
      best_cps = cps;
    }
  }
  return {int(best_n), int(best_cps)};
}

// nseg state slots per (row, head) -- nseg - 1 segment end states and the copy of h_in --
// then nseg - 1 floats per (row, head)
size_t ws_h_bytes(int64_t Bt, int64_t H, int64_t N, const SegPlan& sp) {
  return size_t(Bt * H) * size_t(sp.nseg) * size_t(ssd::kP * N) * 4;
}

size_t ws_bytes_for(int64_t Bt, int64_t H, int64_t N, const SegPlan& sp) {
  if (sp.nseg <= 1) return 0;
  const size_t nA = size_t(Bt * H) * size_t(sp.nseg - 1);
  return ws_h_bytes(Bt, H, N, sp) + ((nA * 4 + 255) / 256) * 256;
}

template <int N, bool kGate, bool kPre, bool kSeq>
cudaError_t launch_one(const ssd::SsdArgs& a, int64_t batch, int nz, cudaStream_t st) {
  auto kern = ssd::ssd_fwd_kernel<N, kGate, kPre, kSeq>;
  constexpr int smem = ssd::SsdSmem<N, kPre>::kBytes;
  static bool attr_set = false;   // the attribute is set once per instantiation
  if (!attr_set) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  kern<<<dim3(unsigned(a.H), unsigned(batch), unsigned(nz)), ssd::kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <int N, bool kGate, bool kSeq>
cudaError_t launch(const ssd::SsdArgs& a, int64_t batch, cudaStream_t st) {
  if (a.nseg > 1) {
    cudaError_t e = launch_one<N, false, true, kSeq>(a, batch, a.nseg - 1, st);
    if (e != cudaSuccess) return e;
  }
  return launch_one<N, kGate, false, kSeq>(a, batch, a.nseg, st);
}

// The tensor-core passes (no document resets): the state pass when the rows are cut into
// segments, then the main pass.
template <int N>
cudaError_t launch_tc_state(const ssd::SsdArgs& a, int64_t batch, const CUtensorMap* maps,
                            int* status, cudaStream_t st) {
  using S = ssd::tc::StateSmem<N>;
  auto kern = ssd::tc::ssd_tc_state_kernel<N>;
  static bool attr_set = false;
  if (!attr_set) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               S::kDynamic);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  kern<<<dim3(unsigned(a.H), unsigned(batch), unsigned(a.nseg - 1)), ssd::tc::kThreads,
         S::kDynamic, st>>>(maps[1], maps[2], a, status);
  return cudaGetLastError();
}

template <int N, bool kGate>
cudaError_t launch_tc(const ssd::SsdArgs& a, int64_t batch, const CUtensorMap* maps, int* status,
                      cudaStream_t st) {
  using S = ssd::tc::Smem<N>;
  if (a.nseg > 1) {
    cudaError_t e = launch_tc_state<N>(a, batch, maps, status, st);
    if (e != cudaSuccess) return e;
  }
  auto kern = ssd::tc::ssd_tc_kernel<N, kGate>;
  static bool attr_set = false;
  if (!attr_set) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               S::kDynamic);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  kern<<<dim3(unsigned(a.H), unsigned(batch), unsigned(a.nseg)), ssd::tc::kThreads, S::kDynamic,
         st>>>(maps[0], maps[1], maps[2], a, status);
  return cudaGetLastError();
}

template <int N>
cudaError_t launch_n(const ssd::SsdArgs& a, int64_t batch, cudaStream_t st) {
  if (a.z)
    return a.seq_idx ? launch<N, true, true>(a, batch, st) : launch<N, true, false>(a, batch, st);
  return a.seq_idx ? launch<N, false, true>(a, batch, st) : launch<N, false, false>(a, batch, st);
}

int check_dims(const mamba2_dims* dims) {
  if (!dims) return ssd_fail(MAMBA_ERR_INVALID_ARGUMENT, "dims is NULL");
  if (dims->reserved != 0) return ssd_fail(MAMBA_ERR_INVALID_ARGUMENT, "dims.reserved must be 0");
  const int64_t Bt = dims->batch, L = dims->seqlen, H = dims->nheads, P = dims->headdim,
                N = dims->d_state, G = dims->ngroups;
  if (Bt < 0 || L < 0 || H < 0 || P < 0 || N < 0 || G < 0)
    return ssd_fail(MAMBA_ERR_INVALID_ARGUMENT, "negative size in dims");
  if (dims->io_dtype != MAMBA_BF16)
    return ssd_fail(MAMBA_ERR_UNSUPPORTED, "io_dtype %d: only MAMBA_BF16 is supported", dims->io_dtype);
  if (P != ssd::kP) return ssd_fail(MAMBA_ERR_UNSUPPORTED, "headdim %lld: only 64 is supported", (long long)P);
  if (N != 64 && N != 128)
    return ssd_fail(MAMBA_ERR_UNSUPPORTED, "d_state %lld: only 64 and 128 are supported", (long long)N);
  if (G < 1 || (H > 0 && H % G))
    return ssd_fail(MAMBA_ERR_INVALID_ARGUMENT, "ngroups %lld must be >= 1 and divide nheads %lld",
                    (long long)G, (long long)H);
  if (Bt > 65535) return ssd_fail(MAMBA_ERR_UNSUPPORTED, "batch %lld > 65535", (long long)Bt);
  if (H > 0x7fffffff) return ssd_fail(MAMBA_ERR_UNSUPPORTED, "nheads too large");
  const double act_d = double(Bt) * double(L) * double(H) * double(P);
  const double bc_d = double(Bt) * double(L) * double(G) * double(N);
  if (act_d * 2 > 9e18 || bc_d * 2 > 9e18) return ssd_fail(MAMBA_ERR_INVALID_ARGUMENT, "sizes overflow");
  return MAMBA_OK;
}

}  // namespace

extern "C" MAMBA_API size_t mamba2_ssd_fwd_workspace_bytes(const mamba2_dims* dims) {
  if (check_dims(dims) != MAMBA_OK) return 0;
  const SegPlan sp = seg_plan(dims->batch, dims->seqlen, dims->nheads);
  return ws_bytes_for(dims->batch, dims->nheads, dims->d_state, sp);
}

extern "C" MAMBA_API int mamba2_ssd_check(void* cuda_stream) {
  void* word = nullptr;
  char why[256];
  if (mm_host::symbol_in_context(reinterpret_cast<const void*>(&g_ssd_status), &word,
                                 "mamba2_ssd_check", why, sizeof(why)) != 0)
    return ssd_fail(MAMBA_ERR_CUDA, "%s", why);
  return mamba_mixer_check(word, cuda_stream);
}

extern "C" MAMBA_API int mamba2_ssd_fwd(const mamba2_dims* dims, const void* x, const void* dt_raw,
                                        const float* A_log, const void* B, const void* C,
                                        const float* D, const float* dt_bias, const void* z,
                                        const int32_t* seq_idx, const float* h_in, void* y,
                                        float* h_out,
                                        void* workspace, size_t workspace_bytes,
                                        void* cuda_stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  const int64_t Bt = dims->batch, L = dims->seqlen, H = dims->nheads, P = dims->headdim,
                N = dims->d_state, G = dims->ngroups;
  const size_t act = size_t(Bt * L * H * P), bc = size_t(Bt * L * G * N), dtn = size_t(Bt * L * H);
  const size_t state = size_t(Bt * H * P * N);
  const bool any = act > 0;
  if ((rc = need(x, "x", any, 16)) || (rc = need(dt_raw, "dt_raw", any, 2)) ||
      (rc = need(A_log, "A_log", H > 0, 4)) || (rc = need(B, "B", any, 16)) ||
      (rc = need(C, "C", any, 16)) || (rc = need(D, "D", H > 0, 4)) ||
      (rc = need(dt_bias, "dt_bias", H > 0, 4)) || (rc = need(z, "z", false, 16)) ||
      (rc = need(seq_idx, "seq_idx", false, 4)) ||
      (rc = need(h_in, "h_in", false, 16)) || (rc = need(y, "y", any, 16)) ||
      (rc = need(h_out, "h_out", false, 16)))
    return rc;
  const Range ins[] = {{x, act * 2, "x"},         {dt_raw, dtn * 2, "dt_raw"}, {A_log, size_t(H) * 4, "A_log"},
                       {B, bc * 2, "B"},          {C, bc * 2, "C"},            {D, size_t(H) * 4, "D"},
                       {dt_bias, size_t(H) * 4, "dt_bias"}, {z, act * 2, "z"},
                       {seq_idx, size_t(Bt * L) * 4, "seq_idx"}};
  const Range y_r{y, act * 2, "y"}, hin_r{h_in, state * 4, "h_in"}, hout_r{h_out, state * 4, "h_out"};
  for (const Range& i : ins) {
    if (overlap(y_r, i) || overlap(hout_r, i))
      return ssd_fail(MAMBA_ERR_INVALID_ARGUMENT, "an output overlaps %s", i.name);
  }
  if (overlap(y_r, hout_r) || overlap(y_r, hin_r))
    return ssd_fail(MAMBA_ERR_INVALID_ARGUMENT, "y overlaps a state buffer");
  if (overlap(hout_r, hin_r) && h_out != h_in)
    return ssd_fail(MAMBA_ERR_INVALID_ARGUMENT, "h_out partially overlaps h_in");
  const bool tc = use_tc(seq_idx) && L > 0;   // an empty sequence only passes h_in through
  const SegPlan sp = seg_plan(Bt, L, H);
  const size_t need = ws_bytes_for(Bt, H, N, sp);
  if (need > 0) {
    if (!workspace || workspace_bytes < need)
      return ssd_fail(MAMBA_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", workspace_bytes, need);
    if (reinterpret_cast<uintptr_t>(workspace) % 256)
      return ssd_fail(MAMBA_ERR_ALIGNMENT, "workspace is not 256-byte aligned");
    const Range ws_r{workspace, need, "workspace"};
    for (const Range& i : ins)
      if (overlap(ws_r, i)) return ssd_fail(MAMBA_ERR_INVALID_ARGUMENT, "workspace overlaps %s", i.name);
    if (overlap(ws_r, y_r) || overlap(ws_r, hin_r) || overlap(ws_r, hout_r))
      return ssd_fail(MAMBA_ERR_INVALID_ARGUMENT, "workspace overlaps an output or the state");
  }
  if (Bt == 0 || H == 0) return ssd_ok();

  ssd::SsdArgs a{};
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.dt = static_cast<const __nv_bfloat16*>(dt_raw);
  a.A_log = A_log;
  a.B = static_cast<const __nv_bfloat16*>(B);
  a.C = static_cast<const __nv_bfloat16*>(C);
  a.D = D;
  a.dt_bias = dt_bias;
  a.z = static_cast<const __nv_bfloat16*>(z);
  a.h_in = h_in;
  a.seq_idx = seq_idx;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.h_out = h_out;
  a.L = L;
  a.H = int(H);
  a.G = int(G);
  a.nseg = sp.nseg;
  a.cps = sp.cps;
  if (sp.nseg > 1) {
    a.ws_H = static_cast<float*>(workspace);
    a.ws_A = reinterpret_cast<float*>(static_cast<unsigned char*>(workspace) + ws_h_bytes(Bt, H, N, sp));
  }
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t e;
  if (tc) {
    CUtensorMap maps[3];
    if (!mm_internal::make_map4d_sw128(&maps[0], C, uint64_t(N), uint64_t(G), uint64_t(L),
                                       uint64_t(Bt), 64, 1, uint32_t(ssd::kQ), 1) ||
        !mm_internal::make_map4d_sw128(&maps[1], B, uint64_t(N), uint64_t(G), uint64_t(L),
                                       uint64_t(Bt), 64, 1, uint32_t(ssd::kQ), 1) ||
        !mm_internal::make_map4d_sw128(&maps[2], x, uint64_t(P), uint64_t(H), uint64_t(L),
                                       uint64_t(Bt), 64, 1, uint32_t(ssd::kQ), 1))
      return ssd_fail(MAMBA_ERR_CUDA, "cuTensorMapEncodeTiled failed or is unavailable");
    void* word = nullptr;
    char why[256];
    if (mm_host::symbol_in_context(reinterpret_cast<const void*>(&g_ssd_status), &word,
                                   "mamba2_ssd_fwd", why, sizeof(why)) != 0)
      return ssd_fail(MAMBA_ERR_CUDA, "%s", why);
    int* status = static_cast<int*>(word);
    if (N == 128)
      e = z ? launch_tc<128, true>(a, Bt, maps, status, st) : launch_tc<128, false>(a, Bt, maps, status, st);
    else
      e = z ? launch_tc<64, true>(a, Bt, maps, status, st) : launch_tc<64, false>(a, Bt, maps, status, st);
  } else {
    e = N == 128 ? launch_n<128>(a, Bt, st) : launch_n<64>(a, Bt, st);
  }
  if (e != cudaSuccess) return ssd_fail(MAMBA_ERR_CUDA, "ssd launch failed: %s", cudaGetErrorString(e));
  return ssd_ok();
}

extern "C" MAMBA_API int mamba2_ssd_step(const mamba2_dims* dims, const void* x, const void* dt_raw,
                                         const float* A_log, const void* B, const void* C,
                                         const float* D, const float* dt_bias, const void* z,
                                         const float* h_in, void* y, float* h_out,
                                         void* cuda_stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  const int64_t Bt = dims->batch, H = dims->nheads, P = dims->headdim, N = dims->d_state,
                G = dims->ngroups;
  if (dims->seqlen != 1)
    return ssd_fail(MAMBA_ERR_INVALID_ARGUMENT, "seqlen %lld: the step takes one token",
                    (long long)dims->seqlen);
  const size_t rows = size_t(Bt * H * P), state = rows * size_t(N);
  const bool any = rows > 0;
  if ((rc = need(x, "x", any, 16)) || (rc = need(dt_raw, "dt_raw", any, 2)) ||
      (rc = need(A_log, "A_log", H > 0, 4)) || (rc = need(B, "B", any, 16)) ||
      (rc = need(C, "C", any, 16)) || (rc = need(D, "D", H > 0, 4)) ||
      (rc = need(dt_bias, "dt_bias", H > 0, 4)) || (rc = need(z, "z", false, 16)) ||
      (rc = need(h_in, "h_in", any, 16)) || (rc = need(y, "y", any, 16)) ||
      (rc = need(h_out, "h_out", any, 16)))
    return rc;
  const size_t bc = size_t(Bt * G * N);
  const Range ins[] = {{x, rows * 2, "x"},       {dt_raw, size_t(Bt * H) * 2, "dt_raw"},
                       {A_log, size_t(H) * 4, "A_log"}, {B, bc * 2, "B"}, {C, bc * 2, "C"},
                       {D, size_t(H) * 4, "D"},  {dt_bias, size_t(H) * 4, "dt_bias"},
                       {z, rows * 2, "z"}};
  const Range y_r{y, rows * 2, "y"}, hin_r{h_in, state * 4, "h_in"}, hout_r{h_out, state * 4, "h_out"};
  for (const Range& i : ins)
    if (overlap(y_r, i) || overlap(hout_r, i))
      return ssd_fail(MAMBA_ERR_INVALID_ARGUMENT, "an output overlaps %s", i.name);
  if (overlap(y_r, hout_r) || overlap(y_r, hin_r))
    return ssd_fail(MAMBA_ERR_INVALID_ARGUMENT, "y overlaps a state buffer");
  if (overlap(hout_r, hin_r) && h_out != h_in)
    return ssd_fail(MAMBA_ERR_INVALID_ARGUMENT, "h_out partially overlaps h_in");
  if (!any) return ssd_ok();
  if (H > (int64_t(0x7fffffff) / 4))
    return ssd_fail(MAMBA_ERR_UNSUPPORTED, "nheads %lld too large for the step's grid", (long long)H);

  ssd::StepArgs a{};
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.dt = static_cast<const __nv_bfloat16*>(dt_raw);
  a.A_log = A_log;
  a.B = static_cast<const __nv_bfloat16*>(B);
  a.C = static_cast<const __nv_bfloat16*>(C);
  a.D = D;
  a.dt_bias = dt_bias;
  a.z = static_cast<const __nv_bfloat16*>(z);
  a.h_in = h_in;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.h_out = h_out;
  a.H = int(H);
  a.G = int(G);
  (void)P;  // headdim is 64 (checked above)
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  constexpr int kS = ssd::kStepStates;
  if (N == 128) {
    const dim3 grid(unsigned(H * ssd::StepShape<128, kS>::kCtaPerHead), unsigned(Bt));
    z ? ssd::ssd_step_kernel<128, kS, true><<<grid, ssd::kStepThreads, 0, st>>>(a)
      : ssd::ssd_step_kernel<128, kS, false><<<grid, ssd::kStepThreads, 0, st>>>(a);
  } else {
    const dim3 grid(unsigned(H * ssd::StepShape<64, kS>::kCtaPerHead), unsigned(Bt));
    z ? ssd::ssd_step_kernel<64, kS, true><<<grid, ssd::kStepThreads, 0, st>>>(a)
      : ssd::ssd_step_kernel<64, kS, false><<<grid, ssd::kStepThreads, 0, st>>>(a);
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return ssd_fail(MAMBA_ERR_CUDA, "step launch failed: %s", cudaGetErrorString(e));
  return ssd_ok();
}

extern "C" MAMBA_API int mamba2_conv_silu(const mamba2_dims* dims, const void* xbc,
                                          const float* conv_w, const float* conv_b,
                                          const int32_t* seq_idx, const void* conv_state_in,
                                          void* x, void* B, void* C, void* conv_state_out,
                                          void* cuda_stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  const int64_t Bt = dims->batch, L = dims->seqlen, H = dims->nheads, P = dims->headdim,
                N = dims->d_state, G = dims->ngroups;
  const int64_t DI = H * P, GN = G * N, Cc = DI + 2 * GN;
  if (Cc > (int64_t(1) << 24)) return ssd_fail(MAMBA_ERR_UNSUPPORTED, "too many channels");
  const size_t act = size_t(Bt * L * Cc), cst = size_t(Bt * Cc * 3);
  const bool any = Bt > 0 && Cc > 0;
  const bool rows = any && L > 0;
  if ((rc = need(xbc, "xbc", rows, 16)) || (rc = need(conv_w, "conv_w", any, 16)) ||
      (rc = need(conv_b, "conv_b", false, 4)) || (rc = need(seq_idx, "seq_idx", false, 4)) ||
      (rc = need(conv_state_in, "conv_state_in", false, 2)) ||
      (rc = need(x, "x", rows, 16)) || (rc = need(B, "B", rows && GN > 0, 16)) ||
      (rc = need(C, "C", rows && GN > 0, 16)) ||
      (rc = need(conv_state_out, "conv_state_out", false, 2)))
    return rc;
  const Range ins[] = {{xbc, act * 2, "xbc"}, {conv_w, size_t(Cc) * 16, "conv_w"},
                       {conv_b, size_t(Cc) * 4, "conv_b"}, {seq_idx, size_t(Bt * L) * 4, "seq_idx"},
                       {conv_state_in, cst * 2, "conv_state_in"}};
  const Range outs[] = {{x, size_t(Bt * L * DI) * 2, "x"}, {B, size_t(Bt * L * GN) * 2, "B"},
                        {C, size_t(Bt * L * GN) * 2, "C"}, {conv_state_out, cst * 2, "conv_state_out"}};
  for (const Range& o : outs) {
    for (const Range& i : ins)
      if (overlap(o, i)) return ssd_fail(MAMBA_ERR_INVALID_ARGUMENT, "%s overlaps %s", o.name, i.name);
    for (const Range& o2 : outs)
      if (&o != &o2 && overlap(o, o2))
        return ssd_fail(MAMBA_ERR_INVALID_ARGUMENT, "%s overlaps %s", o.name, o2.name);
  }
  if (!any) return ssd_ok();
  ssd::ConvArgs a{};
  a.xbc = static_cast<const __nv_bfloat16*>(xbc);
  a.w = conv_w;
  a.bias = conv_b;
  a.seq_idx = seq_idx;
  a.cs_in = static_cast<const __nv_bfloat16*>(conv_state_in);
  a.x = static_cast<__nv_bfloat16*>(x);
  a.B = static_cast<__nv_bfloat16*>(B);
  a.C = static_cast<__nv_bfloat16*>(C);
  a.cs_out = static_cast<__nv_bfloat16*>(conv_state_out);
  a.L = L;
  a.Cc = int(Cc);
  a.DI = int(DI);
  a.GN = int(GN);
  if (L == 0 && !conv_state_out) return ssd_ok();
  const int64_t tiles = L > 0 ? (L + ssd::kConvSteps - 1) / ssd::kConvSteps : 1;  // L = 0: the state
  if (tiles > 65535) return ssd_fail(MAMBA_ERR_UNSUPPORTED, "seqlen too long for one launch");
  const dim3 grid(unsigned((Cc / 8 + ssd::kConvThreads - 1) / ssd::kConvThreads), unsigned(tiles),
                  unsigned(Bt));
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  if (seq_idx)
    ssd::conv_silu_kernel<true><<<grid, ssd::kConvThreads, 0, st>>>(a);
  else
    ssd::conv_silu_kernel<false><<<grid, ssd::kConvThreads, 0, st>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return ssd_fail(MAMBA_ERR_CUDA, "conv launch failed: %s", cudaGetErrorString(e));
  return ssd_ok();
}

extern "C" MAMBA_API int mamba2_gated_rmsnorm(const mamba2_dims* dims, const void* y, const void* z,
                                              const float* weight, float eps, void* out,
                                              void* cuda_stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  const int64_t Bt = dims->batch, L = dims->seqlen, H = dims->nheads, P = dims->headdim,
                G = dims->ngroups;
  const int64_t D = H * P, rows = Bt * L;
  if (!(eps >= 0.f)) return ssd_fail(MAMBA_ERR_INVALID_ARGUMENT, "eps must be >= 0");
  if (D > (int64_t(1) << 24)) return ssd_fail(MAMBA_ERR_UNSUPPORTED, "too many channels");
  const size_t act = size_t(rows * D);
  const bool any = act > 0;
  if ((rc = need(y, "y", any, 16)) || (rc = need(z, "z", any, 16)) ||
      (rc = need(weight, "weight", any, 16)) || (rc = need(out, "out", any, 16)))
    return rc;
  const Range out_r{out, act * 2, "out"};
  const Range ins[] = {{y, act * 2, "y"}, {z, act * 2, "z"}, {weight, size_t(D) * 4, "weight"}};
  for (const Range& i : ins)
    if (overlap(out_r, i)) return ssd_fail(MAMBA_ERR_INVALID_ARGUMENT, "out overlaps %s", i.name);
  if (!any) return ssd_ok();
  ssd::NormArgs a{};
  a.y = static_cast<const __nv_bfloat16*>(y);
  a.z = static_cast<const __nv_bfloat16*>(z);
  a.w = weight;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.rows = rows;
  a.D = int(D);
  a.gs = int(D / G);
  a.eps = eps;
  const int64_t items = rows * G;
  const int64_t grid = (items + ssd::kNormWarps - 1) / ssd::kNormWarps;
  if (grid > 0x7fffffff) return ssd_fail(MAMBA_ERR_UNSUPPORTED, "too many rows for one launch");
  if (a.gs <= 32 * 8 * ssd::kNormCachedUnits)
    ssd::gated_rmsnorm_kernel<true><<<unsigned(grid), ssd::kNormWarps * 32, 0,
                                      static_cast<cudaStream_t>(cuda_stream)>>>(a);
  else
    ssd::gated_rmsnorm_kernel<false><<<unsigned(grid), ssd::kNormWarps * 32, 0,
                                       static_cast<cudaStream_t>(cuda_stream)>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return ssd_fail(MAMBA_ERR_CUDA, "norm launch failed: %s", cudaGetErrorString(e));
  return ssd_ok();
}
