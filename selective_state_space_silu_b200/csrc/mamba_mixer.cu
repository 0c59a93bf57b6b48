// Host side of the C ABI declared in include/mamba_mixer.h: argument checks, the
// time-chunk plan, and kernel launches on the caller's stream.
//
// Every check happens before the first CUDA call; a failing call enqueues nothing.

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>

#include "context_symbol.h"
#include "mamba_mixer.h"
#include "fwd_kernel.cuh"
#include "fwd2_kernel.cuh"
#include "step.cuh"
#include "bwd_kernel.cuh"

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int ok() {
  g_last_error.clear();
  return MAMBA_OK;
}

// Test-only failure injection for the bounded-wait path (mamba_mixer_set_fault_injection):
// k >= 0 makes one CTA of the next forwards skip the copies of its tile k; -1 (the default)
// injects nothing.
std::atomic<int> g_inject_skip_tile{-1};
int inject_skip_tile() { return g_inject_skip_tile.load(std::memory_order_relaxed); }

// cudaFuncSetAttribute for a kernel's dynamic shared memory, once per kernel instantiation
// (each call site is its own template instance, so its static flag covers one kernel).
template <typename K>
cudaError_t set_smem_once(K kern, int bytes, bool& done) {
  if (done) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done = true;
  return e;
}

struct Span {
  const void* p;
  size_t bytes;
  const char* name;
};

bool overlaps(const Span& a, const Span& b) {
  if (!a.p || !b.p || a.bytes == 0 || b.bytes == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a.p), a1 = a0 + a.bytes;
  const uintptr_t b0 = reinterpret_cast<uintptr_t>(b.p), b1 = b0 + b.bytes;
  return a0 < b1 && b0 < a1;
}

bool mul_ok(int64_t a, int64_t b, int64_t* out) {
  if (a < 0 || b < 0) return false;
  if (a != 0 && b > INT64_MAX / a) return false;
  *out = a * b;
  return true;
}

// Validates sizes and support.  Fills element counts.
struct Sizes {
  int64_t act;     // batch*L*Di
  int64_t bc;      // batch*L*N
  int64_t state;   // batch*Di*N
  int64_t cstate;  // batch*Di*(K-1)
  int esize;       // bytes per io element
};

int check_dims(const mamba_dims* d, Sizes* s) {
  if (!d) return fail(MAMBA_ERR_INVALID_ARGUMENT, "dims is NULL");
  if (d->batch < 0 || d->seqlen < 0 || d->d_inner < 0 || d->d_state < 0 || d->d_conv < 0)
    return fail(MAMBA_ERR_INVALID_ARGUMENT, "negative size in dims");
  if (d->reserved != 0) return fail(MAMBA_ERR_INVALID_ARGUMENT, "dims.reserved must be 0");
  if (d->io_dtype != MAMBA_F32 && d->io_dtype != MAMBA_BF16)
    return fail(MAMBA_ERR_UNSUPPORTED, "io_dtype %d is not MAMBA_F32 or MAMBA_BF16",
                int(d->io_dtype));
  if (d->d_conv != 4) return fail(MAMBA_ERR_UNSUPPORTED, "d_conv %lld unsupported (only 4)",
                                  (long long)d->d_conv);
  if (d->d_state != 8 && d->d_state != 16)
    return fail(MAMBA_ERR_UNSUPPORTED, "d_state %lld unsupported (8 or 16)",
                (long long)d->d_state);
  if (d->d_inner % 8 != 0)
    return fail(MAMBA_ERR_UNSUPPORTED, "d_inner %lld is not a multiple of 8",
                (long long)d->d_inner);
  int64_t bl = 0;
  if (!mul_ok(d->batch, d->seqlen, &bl) || !mul_ok(bl, d->d_inner, &s->act) ||
      !mul_ok(bl, d->d_state, &s->bc) || !mul_ok(d->batch * d->d_inner, d->d_state, &s->state) ||
      !mul_ok(d->batch * d->d_inner, d->d_conv - 1, &s->cstate) || s->act > (INT64_MAX >> 3))
    return fail(MAMBA_ERR_INVALID_ARGUMENT, "sizes overflow");
  if (d->batch > 65535) return fail(MAMBA_ERR_UNSUPPORTED, "batch > 65535");
  if (d->d_inner > (int64_t(1) << 28))
    return fail(MAMBA_ERR_UNSUPPORTED, "d_inner > 2^28");
  if (d->seqlen > (int64_t(1) << 31) - 512)
    return fail(MAMBA_ERR_UNSUPPORTED, "seqlen >= 2^31 - 512");
  s->esize = d->io_dtype == MAMBA_F32 ? 4 : 2;
  return MAMBA_OK;
}

int check_ptr(const void* p, const char* name, bool required, size_t align) {
  if (!p) {
    if (required) return fail(MAMBA_ERR_INVALID_ARGUMENT, "%s is NULL", name);
    return MAMBA_OK;
  }
  if (reinterpret_cast<uintptr_t>(p) % align != 0)
    return fail(MAMBA_ERR_ALIGNMENT, "%s is not %zu-byte aligned", name, align);
  return MAMBA_OK;
}

// ---- time-chunk plan ---------------------------------------------------------------
// A CTA covers one batch row and 32 channels.  When there are too few such tiles to give
// every SM two resident CTAs (three fit: 68 KiB of shared memory each), the sequence is
// cut into time chunks (multiples of the tile length, at least 256 steps) that run in
// parallel with a carried state between them.  Every chunk past the first also costs a
// chunk-state pass over the chunk before it, yet the finer split keeps winning up to about
// thirteen chunk-CTAs per SM, because a lone CTA is latency-bound (about 100 clocks per
// step alone on an SM, 200 with three resident).  Measured on a 2 x 65536 x 2560 forward
// (160 tiles): 1, 2, 3, 4, 5, 7, 9, 12, 16, 24, 48 chunks take 4.69, 4.95, 4.65, 4.31,
// 4.11, 3.96, 3.86, 3.77, 3.92, 3.80, 3.86 ms.
constexpr int kChunkCtas = 148 * 13;
constexpr size_t kWsHeader = 256;  // status word + padding

struct Plan {
  int nchunks;
  int64_t chunk_len;
};

Plan make_plan(const mamba_dims* d) {
  Plan p{1, d->seqlen > 0 ? d->seqlen : 1};
  const int64_t tiles = d->batch * ((d->d_inner + mm::kCh - 1) / mm::kCh);
  if (tiles <= 0 || d->seqlen < 512 || tiles >= 2 * 148) return p;
  int64_t c = kChunkCtas / tiles;
  if (c < 2) c = 2;
  const int64_t cmax = d->seqlen / 256;
  if (c > cmax) c = cmax;
  if (c > 256) c = 256;
  if (c <= 1) return p;
  int64_t len = (d->seqlen + c - 1) / c;
  len = (len + mm::kTileT - 1) / mm::kTileT * mm::kTileT;
  p.nchunks = int((d->seqlen + len - 1) / len);
  p.chunk_len = len;
  return p;
}

// ---- forward plan --------------------------------------------------------------------
// Two 32-channel tiles per SM or more (the 130M-class layer: 384 tiles), and fp32 I/O: the
// warp-specialised kernel of fwd_kernel.cuh, with the parallel chunks of make_plan when
// there are few tiles.  bf16 I/O with fewer tiles (a long row over few channels: the long
// workload has 160): the fwd2 kernel, with four time groups per CTA (the two-level scan)
// for the parallelism one SM needs, and the sequence cut into chained chunks for the
// balance between SMs.  The CTA of chunk c starts from the end state that the CTA of chunk
// c-1 of the same tile left in the workspace, so nothing is recomputed; the units are
// claimed in order, so a unit's predecessor is always running or done.  Measured on the
// long workload (2 x 65536 x 2560): 3.45-3.48 ms with 8, 16 or 32 chunks per row, against
// 3.65 ms for the parallel chunks with their chunk-state pass.
constexpr int64_t kG4MinChunkLen = 1024;
constexpr int64_t kG4MaxChunks = 16;
constexpr size_t kUnitCounterOff = 64;                // in the header, after the status word

struct FwdPlan {
  Plan p;
  bool chained;
  bool v2;     // the fwd2 kernel
  int G;       // its time groups
};

// dtproj: the forward with the dt projection fused (always the fwd2 kernel, one time group
// when there are two tiles per SM or more); its chunking matches the plain forward's, so the
// two take the same workspace.
FwdPlan make_fwd_plan(const mamba_dims* d, bool dtproj = false) {
  FwdPlan f{make_plan(d), false, false, 1};
  const int64_t tiles = d->batch * ((d->d_inner + mm::kCh - 1) / mm::kCh);
  if (d->io_dtype != MAMBA_BF16) return f;
  const int64_t L = d->seqlen > 0 ? d->seqlen : 1;
  if (tiles >= 2 * 148) {
    if (dtproj) {
      f.v2 = true;
      f.p.nchunks = 1;
      f.p.chunk_len = L;
    }
    return f;
  }
  f.v2 = true;
  f.G = 4;
  int64_t c = 1;
  if (L >= 2 * kG4MinChunkLen) c = L / kG4MinChunkLen < kG4MaxChunks ? L / kG4MinChunkLen : kG4MaxChunks;
  f.p.nchunks = 1;
  f.p.chunk_len = L;
  if (c > 1) {
    int64_t len = (L + c - 1) / c;
    len = (len + mm::kTileT - 1) / mm::kTileT * mm::kTileT;
    f.p.nchunks = int((L + len - 1) / len);
    f.p.chunk_len = len;
  }
  f.chained = f.p.nchunks > 1;
  return f;
}

// Chained workspace: header (status word, unit counter), one flag per (tile, scan warp),
// then each tile's carried state [kCh][N] fp32.
struct ChainLayout {
  size_t flags, carry, total;
};
ChainLayout chain_layout(const mamba_dims* d) {
  const size_t tiles = size_t(d->batch) * size_t((d->d_inner + mm::kCh - 1) / mm::kCh);
  ChainLayout l;
  l.flags = kWsHeader;
  l.carry = l.flags + (tiles * mm::kScanWarps * sizeof(int) + 255) / 256 * 256;
  l.total = l.carry + tiles * size_t(mm::kCh) * size_t(d->d_state) * sizeof(float);
  return l;
}

size_t workspace_bytes_for(const mamba_dims* d, const Plan& p) {
  size_t agg = 0;
  if (p.nchunks > 1)
    agg = size_t(2) * size_t(d->batch) * size_t(p.nchunks - 1) * size_t(d->d_inner) *
          size_t(d->d_state) * sizeof(float);
  return kWsHeader + agg;
}

size_t fwd_workspace_for(const mamba_dims* d, const FwdPlan& f) {
  if (f.chained) return chain_layout(d).total;
  if (f.v2) return kWsHeader;
  return workspace_bytes_for(d, f.p);
}

// ---- TMA descriptors ---------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D map over a row-major [d2][d1][d0] tensor, box (b0, b1, 1).
bool make_map(CUtensorMap* m, const void* base, bool bf16, uint64_t d0, uint64_t d1,
              uint64_t d2, uint32_t b0, uint32_t b1, CUtensorMapSwizzle swz) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const uint64_t es = bf16 ? 2 : 4;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * es, d0 * d1 * es};
  const cuuint32_t box[3] = {b0, b1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
             const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over a row-major [d1][d0] bf16 tensor, box (b0, b1), 128-byte swizzle.
bool make_map2d_sw128(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint32_t b0,
                      uint32_t b1) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {d0, d1};
  const cuuint64_t strides[1] = {d0 * 2};
  const cuuint32_t box[2] = {b0, b1};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over a row-major [d2][d1][d0] bf16 tensor, box (b0, b1, 1), 128-byte swizzle.
bool make_map3d_sw128(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                      uint32_t b0, uint32_t b1) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  const cuuint32_t box[3] = {b0, b1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct FwdMaps {
  CUtensorMap x, z, dt, B, C;
  CUtensorMap w;    // the fused dt projection's W_dt (unused otherwise)
};

template <int N, bool kExt, int G, bool kChained, int KB, bool kCkpt = false>
cudaError_t launch_fwd2_kernel(const FwdMaps& m, const mm::f2::Params& a, dim3 grid,
                               cudaStream_t st) {
  using S = mm::f2::Smem<N, G, KB>;
  auto kern = mm::f2::fwd2_kernel<N, kExt, G, kChained, KB, kCkpt>;
  static bool attr_set = false;
  const cudaError_t e = set_smem_once(kern, S::kDynamic, attr_set);
  if (e != cudaSuccess) return e;
  kern<<<grid, mm::f2::threads<G, KB>(), S::kDynamic, st>>>(m.x, m.z, m.dt, m.B, m.C, m.w, a);
  return cudaGetLastError();
}

// KB = K blocks of 64 of the fused dt projection (0: dt_raw is an input).  One time group
// runs unchained only (the plan picks it for many channel tiles, one chunk per row).
template <int N, bool kExt, int KB = 0>
cudaError_t launch_fwd2(const FwdMaps& m, const mm::f2::Params& a, const FwdPlan& f,
                        cudaStream_t st) {
  const unsigned gx = unsigned(a.ntd);
  const dim3 units(gx * unsigned(a.batch) * unsigned(a.nchunks)), tiles(gx, unsigned(a.batch), 1);
  if constexpr (KB > 0) {
    if (f.G == 1) return launch_fwd2_kernel<N, false, 1, false, KB>(m, a, tiles, st);
    return f.chained ? launch_fwd2_kernel<N, false, 4, true, KB>(m, a, units, st)
                     : launch_fwd2_kernel<N, false, 4, false, KB>(m, a, tiles, st);
  } else if (!kExt && a.ckpt) {
    return f.chained ? launch_fwd2_kernel<N, false, 4, true, 0, true>(m, a, units, st)
                     : launch_fwd2_kernel<N, false, 4, false, 0, true>(m, a, tiles, st);
  } else {
    return f.chained ? launch_fwd2_kernel<N, kExt, 4, true, 0>(m, a, units, st)
                     : launch_fwd2_kernel<N, kExt, 4, false, 0>(m, a, tiles, st);
  }
}



template <int N, typename IO, bool P, bool kPre, bool kExt, bool kCkpt = false>
cudaError_t launch_fwd_kernel(const FwdMaps& m, const mm::FwdArgs<kExt>& a, dim3 grid,
                              cudaStream_t st) {
  using S = mm::FwdSmem<IO, N>;
  auto kern = mm::fwd_kernel<N, IO, P, kPre, kExt, kCkpt>;
  static bool attr_set = false;
  const cudaError_t e = set_smem_once(kern, S::kDynamic, attr_set);
  if (e != cudaSuccess) return e;
  kern<<<grid, mm::kFwdThreads, S::kDynamic, st>>>(m.x, m.z, m.dt, m.B, m.C, a);
  return cudaGetLastError();
}

template <int N, typename IO, bool P, bool kExt>
cudaError_t launch_fwd(const FwdMaps& m, const mm::FwdArgs<kExt>& a, int64_t batch,
                       cudaStream_t st) {
  const unsigned gx = unsigned((a.Di + mm::kCh - 1) / mm::kCh);
  if (a.nchunks > 1) {
    cudaError_t e = launch_fwd_kernel<N, IO, P, true, kExt>(
        m, a, dim3(gx, unsigned(batch), unsigned(a.nchunks - 1)), st);
    if (e != cudaSuccess) return e;
  }
  if (!kExt && a.ckpt)
    return launch_fwd_kernel<N, IO, P, false, false, true>(
        m, a, dim3(gx, unsigned(batch), unsigned(a.nchunks)), st);
  return launch_fwd_kernel<N, IO, P, false, kExt>(
      m, a, dim3(gx, unsigned(batch), unsigned(a.nchunks)), st);
}

template <bool kExt>
cudaError_t launch_fwd_any(const FwdMaps& m, const mm::FwdArgs<kExt>& a, const mamba_dims* d,
                           cudaStream_t st) {
  const bool f32 = d->io_dtype == MAMBA_F32;
  if (d->d_state == 16)
    return f32 ? launch_fwd<16, float, true, kExt>(m, a, d->batch, st)
               : launch_fwd<16, __nv_bfloat16, false, kExt>(m, a, d->batch, st);
  return f32 ? launch_fwd<8, float, true, kExt>(m, a, d->batch, st)
             : launch_fwd<8, __nv_bfloat16, false, kExt>(m, a, d->batch, st);
}

// The backward's kernels: with time chunks, the forward's chunk-state pass (P, H), the
// adjoint pass (Lambda), the zeroing of the rows two chunks add to, then the main pass.
template <int N, typename IO, bool P, bool kExt>
cudaError_t launch_bwd(const FwdMaps* m, const mm::FwdArgs<kExt>& pre,
                       const mm::BwdArgs<kExt>& a, int64_t batch, cudaStream_t st) {
  constexpr int smem = mm::BwdSmem<N, IO>::kTotal;
  const unsigned gx = unsigned((a.Di + mm::kBwdCh - 1) / mm::kBwdCh);
  cudaError_t e;
  if (a.nchunks > 1) {
    e = launch_fwd_kernel<N, IO, P, true, kExt>(
        *m, pre, dim3(gx, unsigned(batch), unsigned(a.nchunks - 1)), st);
    if (e != cudaSuccess) return e;
    auto adj = mm::bwd_kernel<N, IO, P, true, kExt>;
    static bool adj_attr_set = false;
    e = set_smem_once(adj, smem, adj_attr_set);
    if (e != cudaSuccess) return e;
    adj<<<dim3(gx, unsigned(batch), unsigned(a.nchunks - 1)), mm::kBwdThreads, smem, st>>>(a);
    mm::bwd_zero_bounds<<<dim3(unsigned(a.nchunks - 1), unsigned(batch)), 256, 0, st>>>(
        a.dxp, a.L, a.Di, a.chunk_len);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  auto kern = mm::bwd_kernel<N, IO, P, false, kExt>;
  static bool attr_set = false;
  e = set_smem_once(kern, smem, attr_set);
  if (e != cudaSuccess) return e;
  kern<<<dim3(gx, unsigned(batch), unsigned(a.nchunks)), mm::kBwdThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <bool kExt>
cudaError_t launch_bwd_any(const FwdMaps* m, const mm::FwdArgs<kExt>& pre,
                           const mm::BwdArgs<kExt>& a, const mamba_dims* d, cudaStream_t st) {
  const bool f32 = d->io_dtype == MAMBA_F32;
  if (d->d_state == 16)
    return f32 ? launch_bwd<16, float, true, kExt>(m, pre, a, d->batch, st)
               : launch_bwd<16, __nv_bfloat16, false, kExt>(m, pre, a, d->batch, st);
  return f32 ? launch_bwd<8, float, true, kExt>(m, pre, a, d->batch, st)
             : launch_bwd<8, __nv_bfloat16, false, kExt>(m, pre, a, d->batch, st);
}

// Backward workspace: header, tile start states, and with time chunks each chunk's
// (P, H) from the chunk-state pass and its adjoint Lambda.
struct BwdLayout {
  size_t states, P, H, Lam, total;   // byte offsets (total = size)
};
BwdLayout bwd_layout(const mamba_dims* d, const Plan& plan) {
  const size_t per = size_t(d->batch) * size_t(d->d_inner) * size_t(d->d_state) * sizeof(float);
  const size_t tiles = size_t((d->seqlen + mm::kBwdT - 1) / mm::kBwdT);
  BwdLayout l;
  l.states = kWsHeader;
  l.P = l.states + tiles * per;
  const size_t agg = plan.nchunks > 1 ? size_t(plan.nchunks - 1) * per : 0;
  l.H = l.P + agg;
  l.Lam = l.H + agg;
  l.total = l.Lam + (plan.nchunks > 1 ? size_t(plan.nchunks) * per : 0);
  return l;
}

size_t bwd_workspace_for(const mamba_dims* d) { return bwd_layout(d, make_plan(d)).total; }

// The decode step's status word: the step takes no workspace, so a bounded wait that runs
// out is recorded here (one word per context; mamba_mixer_step_check reads and clears it).
static __device__ int g_step_status;

// SMs of device `dev`, looked up once per device.
int sm_count(int dev) {
  static std::atomic<int> cache[64];
  if (dev < 0 || dev >= 64) return 148;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

template <int N, typename IO, bool P>
cudaError_t launch_step(mm::StepArgs& a, cudaStream_t st) {
  // About one wave: (channel block, row slice) CTAs of ceil(batch x blocks / resident CTAs)
  // rows each, walking their rows through the 2-deep ring.  Measured on 256 x 5120 (10
  // resident CTAs per SM, so 14 rows per CTA): 34.9 us, against 36.0 with 15 rows (a
  // strict single wave, whose last slice holds one row), 35.4 at 7 rows, 36.7 at 5 rows
  // (about 32 CTAs per SM, 2.8 waves), 41.4 at 12 rows (1.2 waves).
  auto kern = mm::step_kernel<N, IO, P>;
  constexpr int smem = mm::StepSmem<N, IO>::kTotal;
  static std::atomic<int> per_sm{0};   // resident CTAs per SM of this instantiation
  int occ = per_sm.load(std::memory_order_relaxed);
  if (occ == 0) {
    const cudaError_t e =
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, mm::kStepThreads, smem);
    if (e != cudaSuccess) return e;
    if (occ < 1) occ = 1;
    per_sm.store(occ, std::memory_order_relaxed);
  }
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const int64_t nblk = (a.Di + mm::kStepCh - 1) / mm::kStepCh;
  const int64_t slots = int64_t(occ) * sm_count(dev);
  int64_t rows = (a.batch * nblk + slots - 1) / slots;
  if (rows < 1) rows = 1;
  a.rows_per_cta = int(rows);
  const int64_t slices = (a.batch + rows - 1) / rows;
  kern<<<dim3(unsigned(nblk), unsigned(slices)), mm::kStepThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

namespace mm_internal {
// Lets the other translation units of the library report through mamba_last_error.
void set_last_error(const char* msg) { g_last_error = msg; }

// 4-D map over a row-major [d3][d2][d1][d0] bf16 tensor, box (b0, b1, b2, b3), 128-byte
// swizzle (b0 * 2 must be 128 bytes); for the other translation units' TMA copies.
bool make_map4d_sw128(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                      uint64_t d3, uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {d0, d1, d2, d3};
  const cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
  const cuuint32_t box[4] = {b0, b1, b2, b3};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace mm_internal

extern "C" {

const char* mamba_last_error(void) { return g_last_error.c_str(); }

const char* mamba_version(void) { return "mamba_mixer 0.1.0 (abi 1, sm_100a)"; }

size_t mamba_mixer_fwd_workspace_bytes(const mamba_dims* dims) {
  Sizes s;
  if (check_dims(dims, &s) != MAMBA_OK) return 0;
  return fwd_workspace_for(dims, make_fwd_plan(dims));
}

}  // extern "C"

namespace {

// Bytes of the state checkpoints: fp32 [batch, ceil(L/16), d_inner, d_state].
size_t ckpt_bytes_for(const mamba_dims* d) {
  return size_t(d->batch) * size_t((d->seqlen + 15) / 16) * size_t(d->d_inner) *
         size_t(d->d_state) * sizeof(float);
}

// The forward behind mamba_mixer_fwd and mamba_mixer_fwd_packed: seq_idx, h_in and
// conv_state_in are null for the former.
// dt_rank > 0: the dt projection is fused (dt_raw is NULL; dt_low [batch, L, dt_rank] and
// W_dt [d_inner, dt_rank], bf16, give dt_raw = dt_low W_dt^T inside the kernel).
int fwd_common(const mamba_dims* dims, const void* xp, const void* z, const void* dt_raw,
               const void* B, const void* C, const float* A_log, const float* D,
               const float* conv_w, const float* conv_b, const float* dt_bias,
               const int32_t* seq_idx, const float* h_in, const void* conv_state_in, void* y,
               float* h_out, void* conv_state_out, void* workspace, size_t workspace_bytes,
               void* cuda_stream, const void* dt_low = nullptr, const void* W_dt = nullptr,
               int64_t dt_rank = 0, float* ckpt = nullptr) {
  Sizes s;
  int rc = check_dims(dims, &s);
  if (rc) return rc;
  const bool act = s.act > 0, bc = s.bc > 0;
  const bool dtproj = dt_rank > 0;
  if ((rc = check_ptr(ckpt, "h_ckpt", false, 16))) return rc;
  if (dtproj) {
    if (dims->io_dtype != MAMBA_BF16)
      return fail(MAMBA_ERR_UNSUPPORTED, "the fused dt projection takes bf16 I/O only");
    if (dt_rank % 8 != 0 || dt_rank > 64 * mm::f2::kMaxDtBlocks)
      return fail(MAMBA_ERR_UNSUPPORTED, "dt_rank %lld unsupported (a multiple of 8 up to %d)",
                  (long long)dt_rank, 64 * mm::f2::kMaxDtBlocks);
    if ((rc = check_ptr(dt_low, "dt_low", act, 16)) ||
        (rc = check_ptr(W_dt, "W_dt", dims->d_inner > 0, 16)))
      return rc;
  }
  if ((rc = check_ptr(xp, "xp", act, 16)) || (rc = check_ptr(z, "z", act, 16)) ||
      (rc = check_ptr(dt_raw, "dt_raw", act && !dtproj, 16)) || (rc = check_ptr(B, "B", bc, 16)) ||
      (rc = check_ptr(C, "C", bc, 16)) || (rc = check_ptr(y, "y", act, 16)) ||
      (rc = check_ptr(A_log, "A_log", dims->d_inner > 0, 16)) ||
      (rc = check_ptr(D, "D", dims->d_inner > 0, 4)) ||
      (rc = check_ptr(conv_w, "conv_w", dims->d_inner > 0, 16)) ||
      (rc = check_ptr(conv_b, "conv_b", false, 4)) ||
      (rc = check_ptr(dt_bias, "dt_bias", dims->d_inner > 0, 4)) ||
      (rc = check_ptr(h_out, "h_out", false, 16)) ||
      (rc = check_ptr(conv_state_out, "conv_state_out", false, 2)) ||
      (rc = check_ptr(seq_idx, "seq_idx", false, 4)) ||
      (rc = check_ptr(h_in, "h_in", false, 16)) ||
      (rc = check_ptr(conv_state_in, "conv_state_in", false, 2)))
    return rc;
  const int64_t Di = dims->d_inner, N = dims->d_state;
  const Span ins[] = {{xp, size_t(s.act) * s.esize, "xp"},   {z, size_t(s.act) * s.esize, "z"},
                      {dt_raw, size_t(s.act) * s.esize, "dt_raw"},
                      {B, size_t(s.bc) * s.esize, "B"},     {C, size_t(s.bc) * s.esize, "C"},
                      {A_log, size_t(Di * N) * 4, "A_log"}, {D, size_t(Di) * 4, "D"},
                      {conv_w, size_t(Di) * 16, "conv_w"},  {conv_b, size_t(Di) * 4, "conv_b"},
                      {dt_bias, size_t(Di) * 4, "dt_bias"},
                      {seq_idx, size_t(dims->batch) * size_t(dims->seqlen) * 4, "seq_idx"},
                      {h_in, size_t(s.state) * 4, "h_in"},
                      {conv_state_in, size_t(s.cstate) * s.esize, "conv_state_in"},
                      {dt_low, dtproj ? size_t(dims->batch) * size_t(dims->seqlen) * size_t(dt_rank) * 2 : 0, "dt_low"},
                      {W_dt, dtproj ? size_t(Di) * size_t(dt_rank) * 2 : 0, "W_dt"}};
  const Span outs[] = {{y, size_t(s.act) * s.esize, "y"},
                       {h_out, size_t(s.state) * 4, "h_out"},
                       {conv_state_out, size_t(s.cstate) * s.esize, "conv_state_out"},
                       {ckpt, ckpt ? ckpt_bytes_for(dims) : 0, "h_ckpt"}};
  const FwdPlan fplan = make_fwd_plan(dims, dtproj);
  const Plan& plan = fplan.p;
  const size_t need = fwd_workspace_for(dims, fplan);
  const Span wsp{workspace, need, "workspace"};
  for (const Span& o : outs) {
    for (const Span& i : ins)
      if (overlaps(o, i)) return fail(MAMBA_ERR_INVALID_ARGUMENT, "%s overlaps %s", o.name, i.name);
    for (const Span& o2 : outs)
      if (&o2 != &o && overlaps(o, o2))
        return fail(MAMBA_ERR_INVALID_ARGUMENT, "%s overlaps %s", o.name, o2.name);
    if (overlaps(o, wsp)) return fail(MAMBA_ERR_INVALID_ARGUMENT, "%s overlaps workspace", o.name);
  }
  for (const Span& i : ins)
    if (overlaps(i, wsp)) return fail(MAMBA_ERR_INVALID_ARGUMENT, "workspace overlaps %s", i.name);
  if (!workspace || workspace_bytes < need)
    return fail(MAMBA_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed",
                workspace ? workspace_bytes : size_t(0), need);
  if (reinterpret_cast<uintptr_t>(workspace) % 16 != 0)
    return fail(MAMBA_ERR_WORKSPACE, "workspace is not 16-byte aligned");
  if (dims->batch == 0 || Di == 0) return ok();

  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  const bool f32 = dims->io_dtype == MAMBA_F32;
  if (dims->seqlen == 0) {
    // empty sequence: the states out are the initial ones (zero when absent)
    cudaError_t e = cudaSuccess;
    if (h_out)
      e = h_in ? cudaMemcpyAsync(h_out, h_in, size_t(s.state) * 4, cudaMemcpyDeviceToDevice, st)
               : cudaMemsetAsync(h_out, 0, size_t(s.state) * 4, st);
    if (e == cudaSuccess && conv_state_out)
      e = conv_state_in ? cudaMemcpyAsync(conv_state_out, conv_state_in, size_t(s.cstate) * s.esize,
                                          cudaMemcpyDeviceToDevice, st)
                        : cudaMemsetAsync(conv_state_out, 0, size_t(s.cstate) * s.esize, st);
    if (e != cudaSuccess)
      return fail(MAMBA_ERR_CUDA, "state reset failed: %s", cudaGetErrorString(e));
    return ok();
  }

  FwdMaps m;
  const uint64_t Bt = uint64_t(dims->batch), L = uint64_t(dims->seqlen);
  const CUtensorMapSwizzle swz = f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  const uint32_t nrow = uint32_t(mm::kTileT);
  const bool dt_ok = dtproj
      ? make_map3d_sw128(&m.dt, dt_low, uint64_t(dt_rank), L, Bt, 64, nrow) &&
        make_map2d_sw128(&m.w, W_dt, uint64_t(dt_rank), uint64_t(Di), 64, mm::kCh)
      : make_map(&m.dt, dt_raw, !f32, uint64_t(Di), L, Bt, mm::kCh, nrow, swz);
  if (!dtproj) m.w = m.dt;   // not read
  if (!make_map(&m.x, xp, !f32, uint64_t(Di), L, Bt, mm::kCh, nrow + mm::kHalo, swz) ||
      !make_map(&m.z, z, !f32, uint64_t(Di), L, Bt, mm::kCh, nrow, swz) || !dt_ok ||
      !make_map(&m.B, B, !f32, uint64_t(N), L, Bt, uint32_t(N), nrow, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map(&m.C, C, !f32, uint64_t(N), L, Bt, uint32_t(N), nrow, CU_TENSOR_MAP_SWIZZLE_NONE))
    return fail(MAMBA_ERR_CUDA, "cuTensorMapEncodeTiled failed or is unavailable");

  unsigned char* wsb = static_cast<unsigned char*>(workspace);
  if (fplan.v2) {
    mm::f2::Params a2{};
    a2.A_log = A_log; a2.D = D; a2.conv_w = conv_w; a2.conv_b = conv_b; a2.dt_bias = dt_bias;
    a2.y = static_cast<__nv_bfloat16*>(y);
    a2.h_out = h_out;
    a2.cs_out = static_cast<__nv_bfloat16*>(conv_state_out);
    a2.status = static_cast<int*>(workspace);
    a2.seq_idx = seq_idx;
    a2.ckpt = ckpt;
    a2.h_in = h_in;
    a2.cs_in = static_cast<const __nv_bfloat16*>(conv_state_in);
    a2.L = dims->seqlen; a2.Di = Di;
    a2.chunk_len = plan.chunk_len; a2.nchunks = plan.nchunks;
    a2.ntd = int((Di + mm::kCh - 1) / mm::kCh);
    a2.batch = int(dims->batch);
    a2.inject_skip_tile = inject_skip_tile();
    a2.dt_rank = int(dt_rank);
    cudaError_t e = cudaSuccess;
    if (fplan.chained) {
      const ChainLayout lay = chain_layout(dims);
      a2.unit_counter = reinterpret_cast<int*>(wsb + kUnitCounterOff);
      a2.carry_flag = reinterpret_cast<int*>(wsb + lay.flags);
      a2.carry = reinterpret_cast<float*>(wsb + lay.carry);
      // unit counter and carry flags start at zero (the status word at offset 0 is kept)
      e = cudaMemsetAsync(wsb + kUnitCounterOff, 0, lay.carry - kUnitCounterOff, st);
      if (e != cudaSuccess)
        return fail(MAMBA_ERR_CUDA, "workspace reset failed: %s", cudaGetErrorString(e));
    }
    const bool ext = seq_idx || h_in || conv_state_in;
    if (dtproj && dt_rank <= 64)
      e = N == 16 ? launch_fwd2<16, false, 1>(m, a2, fplan, st)
                  : launch_fwd2<8, false, 1>(m, a2, fplan, st);
    else if (dtproj)
      e = N == 16 ? launch_fwd2<16, false, 2>(m, a2, fplan, st)
                  : launch_fwd2<8, false, 2>(m, a2, fplan, st);
    else if (N == 16)
      e = ext ? launch_fwd2<16, true>(m, a2, fplan, st) : launch_fwd2<16, false>(m, a2, fplan, st);
    else
      e = ext ? launch_fwd2<8, true>(m, a2, fplan, st) : launch_fwd2<8, false>(m, a2, fplan, st);
    if (e != cudaSuccess)
      return fail(MAMBA_ERR_CUDA, "forward launch failed: %s", cudaGetErrorString(e));
    return ok();
  }

  mm::FwdParams a{};
  a.A_log = A_log; a.D = D; a.conv_w = conv_w; a.conv_b = conv_b; a.dt_bias = dt_bias;
  a.y = y; a.h_out = h_out; a.cs_out = conv_state_out;
  a.ckpt = ckpt;
  a.status = static_cast<int*>(workspace);
  a.L = dims->seqlen; a.Di = Di;
  a.nchunks = plan.nchunks; a.chunk_len = plan.chunk_len;
  // Test-only failure injection (bounded-wait path, mamba_mixer_set_fault_injection): k >= 0
  // makes one CTA skip the copies of its tile k; -1 (the default) injects nothing.
  a.inject_skip_tile = inject_skip_tile();
  cudaError_t e;
  if (plan.nchunks > 1) {
    const size_t agg = (need - kWsHeader) / sizeof(float) / 2;
    a.ws_P = reinterpret_cast<float*>(wsb + kWsHeader);
    a.ws_H = a.ws_P + agg;
  }
  if (seq_idx || h_in || conv_state_in) {
    mm::FwdArgs<true> ax;
    static_cast<mm::FwdParams&>(ax) = a;
    ax.ext = mm::FwdExt{seq_idx, h_in, conv_state_in};
    e = launch_fwd_any<true>(m, ax, dims, st);
  } else {
    mm::FwdArgs<false> ap;
    static_cast<mm::FwdParams&>(ap) = a;
    e = launch_fwd_any<false>(m, ap, dims, st);
  }
  if (e != cudaSuccess)
    return fail(MAMBA_ERR_CUDA, "forward launch failed: %s", cudaGetErrorString(e));
  return ok();
}

}  // namespace

extern "C" {

int mamba_mixer_fwd(const mamba_dims* dims, const void* xp, const void* z, const void* dt_raw,
                    const void* B, const void* C, const float* A_log, const float* D,
                    const float* conv_w, const float* conv_b, const float* dt_bias, void* y,
                    float* h_out, void* conv_state_out, void* workspace,
                    size_t workspace_bytes, void* cuda_stream) {
  return fwd_common(dims, xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, nullptr,
                    nullptr, nullptr, y, h_out, conv_state_out, workspace, workspace_bytes,
                    cuda_stream);
}

int mamba_mixer_fwd_packed(const mamba_dims* dims, const void* xp, const void* z,
                           const void* dt_raw, const void* B, const void* C, const float* A_log,
                           const float* D, const float* conv_w, const float* conv_b,
                           const float* dt_bias, const int32_t* seq_idx, const float* h_in,
                           const void* conv_state_in, void* y, float* h_out,
                           void* conv_state_out, void* workspace, size_t workspace_bytes,
                           void* cuda_stream) {
  return fwd_common(dims, xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, seq_idx, h_in,
                    conv_state_in, y, h_out, conv_state_out, workspace, workspace_bytes,
                    cuda_stream);
}

int mamba_mixer_fwd_dtproj(const mamba_dims* dims, int64_t dt_rank, const void* xp,
                           const void* z, const void* dt_low, const void* W_dt, const void* B,
                           const void* C, const float* A_log, const float* D,
                           const float* conv_w, const float* conv_b, const float* dt_bias,
                           void* y, float* h_out, void* conv_state_out, void* workspace,
                           size_t workspace_bytes, void* cuda_stream) {
  if (dt_rank <= 0) return fail(MAMBA_ERR_INVALID_ARGUMENT, "dt_rank must be positive");
  return fwd_common(dims, xp, z, nullptr, B, C, A_log, D, conv_w, conv_b, dt_bias, nullptr,
                    nullptr, nullptr, y, h_out, conv_state_out, workspace, workspace_bytes,
                    cuda_stream, dt_low, W_dt, dt_rank);
}

size_t mamba_mixer_ckpt_bytes(const mamba_dims* dims) {
  Sizes s;
  if (!dims || check_dims(dims, &s) != MAMBA_OK) return 0;
  return ckpt_bytes_for(dims);
}

int mamba_mixer_fwd_ckpt(const mamba_dims* dims, const void* xp, const void* z,
                         const void* dt_raw, const void* B, const void* C, const float* A_log,
                         const float* D, const float* conv_w, const float* conv_b,
                         const float* dt_bias, void* y, float* h_out, void* conv_state_out,
                         float* h_ckpt, void* workspace, size_t workspace_bytes,
                         void* cuda_stream) {
  if (!h_ckpt && dims && dims->batch > 0 && dims->seqlen > 0 && dims->d_inner > 0)
    return fail(MAMBA_ERR_INVALID_ARGUMENT, "h_ckpt is NULL");
  return fwd_common(dims, xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, nullptr,
                    nullptr, nullptr, y, h_out, conv_state_out, workspace, workspace_bytes,
                    cuda_stream, nullptr, nullptr, 0, h_ckpt);
}

int mamba_mixer_fwd_launches(const mamba_dims* dims) {
  Sizes s;
  if (check_dims(dims, &s) != MAMBA_OK) return -1;
  if (dims->batch == 0 || dims->d_inner == 0 || dims->seqlen == 0) return 0;
  const FwdPlan f = make_fwd_plan(dims);
  return (f.p.nchunks > 1 && !f.chained) ? 2 : 1;
}

int mamba_mixer_fwd_plan(const mamba_dims* dims, int* nchunks, int64_t* chunk_len,
                         int* time_groups, int* chained) {
  Sizes s;
  int rc = check_dims(dims, &s);
  if (rc) return rc;
  const FwdPlan f = make_fwd_plan(dims);
  if (nchunks) *nchunks = f.p.nchunks;
  if (chunk_len) *chunk_len = f.p.chunk_len;
  if (time_groups) *time_groups = f.G;
  if (chained) *chained = f.chained ? 1 : 0;
  return ok();
}

int mamba_mixer_step_check(void* cuda_stream) {
  void* sp = nullptr;
  char why[256];
  if (mm_host::symbol_in_context(reinterpret_cast<const void*>(&g_step_status), &sp,
                                 "mamba_mixer_step_check", why, sizeof(why)) != 0)
    return fail(MAMBA_ERR_CUDA, "%s", why);
  return mamba_mixer_check(sp, cuda_stream);
}

void mamba_mixer_set_fault_injection(int tile) {
  g_inject_skip_tile.store(tile < 0 ? -1 : tile, std::memory_order_relaxed);
}

int mamba_mixer_check(void* workspace, void* cuda_stream) {
  if (!workspace) return fail(MAMBA_ERR_INVALID_ARGUMENT, "workspace is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  int status = 0;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemcpy(&status, workspace, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(MAMBA_ERR_CUDA, "status read failed: %s", cudaGetErrorString(e));
  if (status != 0) {
    const int zero = 0;
    cudaMemcpy(workspace, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (status == mm::kStatusBadCopy)
      return fail(MAMBA_ERR_CUDA, "a forward kernel refused a TMA copy that failed its "
                  "alignment self-check (outputs incomplete)");
    return fail(MAMBA_ERR_TIMEOUT, "a forward kernel gave up on a bounded wait (status %d)", status);
  }
  return ok();
}

size_t mamba_mixer_bwd_workspace_bytes(const mamba_dims* dims) {
  Sizes s;
  if (check_dims(dims, &s) != MAMBA_OK) return 0;
  return bwd_workspace_for(dims);
}

}  // extern "C"

namespace {

// The backward behind mamba_mixer_bwd and mamba_mixer_bwd_packed (the latter's documents,
// cached start and state gradients are null for the former).
int bwd_common(const mamba_dims* dims, const void* xp, const void* z, const void* dt_raw,
               const void* B, const void* C, const float* A_log, const float* D,
               const float* conv_w, const float* conv_b, const float* dt_bias,
               const int32_t* seq_idx, const float* h_in, const void* conv_state_in,
               const void* dy, float* dxp, float* dz, float* ddt_raw, float* dB, float* dC,
               float* dA_log, float* dD, float* dconv_w, float* dconv_b, float* ddt_bias,
               float* dh_in, float* dconv_state_in, void* workspace, size_t workspace_bytes,
               void* cuda_stream, const float* ckpt = nullptr) {
  Sizes s;
  int rc = check_dims(dims, &s);
  if (rc) return rc;
  const bool act = s.act > 0, bc = s.bc > 0, par = dims->d_inner > 0;
  if ((rc = check_ptr(ckpt, "h_ckpt", false, 16))) return rc;
  if ((rc = check_ptr(xp, "xp", act, 16)) || (rc = check_ptr(z, "z", act, 16)) ||
      (rc = check_ptr(dt_raw, "dt_raw", act, 16)) || (rc = check_ptr(B, "B", bc, 16)) ||
      (rc = check_ptr(C, "C", bc, 16)) || (rc = check_ptr(dy, "dy", act, 16)) ||
      (rc = check_ptr(A_log, "A_log", par, 16)) || (rc = check_ptr(D, "D", par, 4)) ||
      (rc = check_ptr(conv_w, "conv_w", par, 16)) || (rc = check_ptr(conv_b, "conv_b", false, 4)) ||
      (rc = check_ptr(dt_bias, "dt_bias", par, 4)) ||
      (rc = check_ptr(dxp, "dxp", act, 16)) || (rc = check_ptr(dz, "dz", act, 16)) ||
      (rc = check_ptr(ddt_raw, "ddt_raw", act, 16)) || (rc = check_ptr(dB, "dB", bc, 16)) ||
      (rc = check_ptr(dC, "dC", bc, 16)) || (rc = check_ptr(dA_log, "dA_log", par, 16)) ||
      (rc = check_ptr(dD, "dD", par, 4)) || (rc = check_ptr(dconv_w, "dconv_w", par, 16)) ||
      (rc = check_ptr(dconv_b, "dconv_b", false, 4)) ||
      (rc = check_ptr(ddt_bias, "ddt_bias", par, 4)) ||
      (rc = check_ptr(seq_idx, "seq_idx", false, 4)) || (rc = check_ptr(h_in, "h_in", false, 16)) ||
      (rc = check_ptr(conv_state_in, "conv_state_in", false, 2)) ||
      (rc = check_ptr(dh_in, "dh_in", false, 16)) ||
      (rc = check_ptr(dconv_state_in, "dconv_state_in", false, 4)))
    return rc;
  const int64_t Di = dims->d_inner, N = dims->d_state;
  const Span ins[] = {{xp, size_t(s.act) * s.esize, "xp"},   {z, size_t(s.act) * s.esize, "z"},
                      {dt_raw, size_t(s.act) * s.esize, "dt_raw"},
                      {B, size_t(s.bc) * s.esize, "B"},     {C, size_t(s.bc) * s.esize, "C"},
                      {dy, size_t(s.act) * s.esize, "dy"},
                      {A_log, size_t(Di * N) * 4, "A_log"}, {D, size_t(Di) * 4, "D"},
                      {conv_w, size_t(Di) * 16, "conv_w"},  {conv_b, size_t(Di) * 4, "conv_b"},
                      {dt_bias, size_t(Di) * 4, "dt_bias"},
                      {seq_idx, size_t(dims->batch) * size_t(dims->seqlen) * 4, "seq_idx"},
                      {h_in, size_t(s.state) * 4, "h_in"},
                      {conv_state_in, size_t(s.cstate) * s.esize, "conv_state_in"},
                      {ckpt, ckpt ? ckpt_bytes_for(dims) : 0, "h_ckpt"}};
  const Span outs[] = {{dxp, size_t(s.act) * 4, "dxp"},      {dz, size_t(s.act) * 4, "dz"},
                       {ddt_raw, size_t(s.act) * 4, "ddt_raw"}, {dB, size_t(s.bc) * 4, "dB"},
                       {dC, size_t(s.bc) * 4, "dC"},          {dA_log, size_t(Di * N) * 4, "dA_log"},
                       {dD, size_t(Di) * 4, "dD"},            {dconv_w, size_t(Di) * 16, "dconv_w"},
                       {dconv_b, size_t(Di) * 4, "dconv_b"},  {ddt_bias, size_t(Di) * 4, "ddt_bias"},
                       {dh_in, size_t(s.state) * 4, "dh_in"},
                       {dconv_state_in, size_t(s.cstate) * 4, "dconv_state_in"}};
  const size_t need = bwd_workspace_for(dims);
  const Span wsp{workspace, need, "workspace"};
  for (const Span& o : outs) {
    for (const Span& i : ins)
      if (overlaps(o, i)) return fail(MAMBA_ERR_INVALID_ARGUMENT, "%s overlaps %s", o.name, i.name);
    for (const Span& o2 : outs)
      if (&o2 != &o && overlaps(o, o2))
        return fail(MAMBA_ERR_INVALID_ARGUMENT, "%s overlaps %s", o.name, o2.name);
    if (overlaps(o, wsp)) return fail(MAMBA_ERR_INVALID_ARGUMENT, "%s overlaps workspace", o.name);
  }
  for (const Span& i : ins)
    if (overlaps(i, wsp)) return fail(MAMBA_ERR_INVALID_ARGUMENT, "workspace overlaps %s", i.name);
  if (!workspace || workspace_bytes < need)
    return fail(MAMBA_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed",
                workspace ? workspace_bytes : size_t(0), need);
  if (reinterpret_cast<uintptr_t>(workspace) % 16 != 0)
    return fail(MAMBA_ERR_WORKSPACE, "workspace is not 16-byte aligned");
  if (dims->batch == 0 || Di == 0) return ok();

  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  // the sums over channels, batch and time accumulate into zeroed outputs
  cudaError_t e = cudaSuccess;
  const std::pair<void*, size_t> zero[] = {
      {dB, size_t(s.bc) * 4}, {dC, size_t(s.bc) * 4}, {dA_log, size_t(Di * N) * 4},
      {dD, size_t(Di) * 4}, {dconv_w, size_t(Di) * 16}, {dconv_b, size_t(Di) * 4},
      {ddt_bias, size_t(Di) * 4}};
  for (const auto& zr : zero)
    if (e == cudaSuccess && zr.first && zr.second) e = cudaMemsetAsync(zr.first, 0, zr.second, st);
  if (e != cudaSuccess) return fail(MAMBA_ERR_CUDA, "gradient reset failed: %s", cudaGetErrorString(e));
  if (dims->seqlen == 0) {
    // nothing flows back but into the initial state: the gradients of h_in and of the conv
    // window are zero (y is empty)
    if (dh_in && e == cudaSuccess) e = cudaMemsetAsync(dh_in, 0, size_t(s.state) * 4, st);
    if (dconv_state_in && e == cudaSuccess)
      e = cudaMemsetAsync(dconv_state_in, 0, size_t(s.cstate) * 4, st);
    if (e != cudaSuccess) return fail(MAMBA_ERR_CUDA, "gradient reset failed: %s", cudaGetErrorString(e));
    return ok();
  }

  const Plan plan = make_plan(dims);
  const BwdLayout lay = bwd_layout(dims, plan);
  unsigned char* wsb = static_cast<unsigned char*>(workspace);
  mm::BwdParams a{};
  a.xp = xp; a.z = z; a.dt = dt_raw; a.B = B; a.C = C; a.dy = dy;
  a.A_log = A_log; a.D = D; a.conv_w = conv_w; a.conv_b = conv_b; a.dt_bias = dt_bias;
  a.dxp = dxp; a.dz = dz; a.ddt = ddt_raw; a.dB = dB; a.dC = dC; a.dA_log = dA_log; a.dD = dD;
  a.dconv_w = dconv_w; a.dconv_b = dconv_b; a.ddt_bias = ddt_bias;
  a.ws_h = ckpt ? const_cast<float*>(ckpt) : reinterpret_cast<float*>(wsb + lay.states);
  a.states_given = ckpt ? 1 : 0;
  a.L = dims->seqlen; a.Di = Di;
  a.ntiles = int((dims->seqlen + mm::kBwdT - 1) / mm::kBwdT);
  a.chunk_len = plan.chunk_len;
  a.nchunks = plan.nchunks;
  a.ws_P = reinterpret_cast<const float*>(wsb + lay.P);
  a.ws_H = reinterpret_cast<const float*>(wsb + lay.H);
  a.ws_L = reinterpret_cast<float*>(wsb + lay.Lam);
  const bool f32 = dims->io_dtype == MAMBA_F32;
  FwdMaps m;
  mm::FwdParams fp{};
  if (plan.nchunks > 1) {
    // the forward's chunk-state pass over the same inputs gives each chunk's (P, H)
    const uint64_t Bt = uint64_t(dims->batch), L = uint64_t(dims->seqlen);
    const CUtensorMapSwizzle swz = f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    const uint32_t nrow = uint32_t(mm::kTileT);
    if (!make_map(&m.x, xp, !f32, uint64_t(Di), L, Bt, mm::kCh, nrow + mm::kHalo, swz) ||
        !make_map(&m.z, z, !f32, uint64_t(Di), L, Bt, mm::kCh, nrow, swz) ||
        !make_map(&m.dt, dt_raw, !f32, uint64_t(Di), L, Bt, mm::kCh, nrow, swz) ||
        !make_map(&m.B, B, !f32, uint64_t(N), L, Bt, uint32_t(N), nrow, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&m.C, C, !f32, uint64_t(N), L, Bt, uint32_t(N), nrow, CU_TENSOR_MAP_SWIZZLE_NONE))
      return fail(MAMBA_ERR_CUDA, "cuTensorMapEncodeTiled failed or is unavailable");
    fp.A_log = A_log; fp.D = D; fp.conv_w = conv_w; fp.conv_b = conv_b; fp.dt_bias = dt_bias;
    fp.ws_P = const_cast<float*>(a.ws_P);
    fp.ws_H = const_cast<float*>(a.ws_H);
    fp.status = static_cast<int*>(workspace);
    fp.L = dims->seqlen; fp.Di = Di;
    fp.chunk_len = plan.chunk_len; fp.nchunks = plan.nchunks;
    fp.inject_skip_tile = -1;
  }
  if (seq_idx || h_in || conv_state_in || dh_in || dconv_state_in) {
    mm::BwdParamsExt ax;
    static_cast<mm::BwdParams&>(ax) = a;
    ax.seq_idx = seq_idx; ax.h_in = h_in; ax.cs_in = conv_state_in;
    ax.dh_in = dh_in; ax.dcs_in = dconv_state_in;
    mm::FwdParamsExt px;
    static_cast<mm::FwdParams&>(px) = fp;
    px.ext = mm::FwdExt{seq_idx, nullptr, conv_state_in};   // chunk pairs start from zero
    e = launch_bwd_any<true>(&m, px, ax, dims, st);
  } else {
    e = launch_bwd_any<false>(&m, fp, a, dims, st);
  }
  if (e != cudaSuccess)
    return fail(MAMBA_ERR_CUDA, "backward launch failed: %s", cudaGetErrorString(e));
  return ok();
}

}  // namespace

extern "C" {

int mamba_mixer_bwd(const mamba_dims* dims, const void* xp, const void* z, const void* dt_raw,
                    const void* B, const void* C, const float* A_log, const float* D,
                    const float* conv_w, const float* conv_b, const float* dt_bias,
                    const void* dy, float* dxp, float* dz, float* ddt_raw, float* dB, float* dC,
                    float* dA_log, float* dD, float* dconv_w, float* dconv_b, float* ddt_bias,
                    void* workspace, size_t workspace_bytes, void* cuda_stream) {
  return bwd_common(dims, xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, nullptr,
                    nullptr, nullptr, dy, dxp, dz, ddt_raw, dB, dC, dA_log, dD, dconv_w, dconv_b,
                    ddt_bias, nullptr, nullptr, workspace, workspace_bytes, cuda_stream);
}

int mamba_mixer_bwd_ckpt(const mamba_dims* dims, const void* xp, const void* z,
                         const void* dt_raw, const void* B, const void* C, const float* A_log,
                         const float* D, const float* conv_w, const float* conv_b,
                         const float* dt_bias, const float* h_ckpt, const void* dy, float* dxp,
                         float* dz, float* ddt_raw, float* dB, float* dC, float* dA_log,
                         float* dD, float* dconv_w, float* dconv_b, float* ddt_bias,
                         void* workspace, size_t workspace_bytes, void* cuda_stream) {
  if (!h_ckpt && dims && dims->batch > 0 && dims->seqlen > 0 && dims->d_inner > 0)
    return fail(MAMBA_ERR_INVALID_ARGUMENT, "h_ckpt is NULL");
  return bwd_common(dims, xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, nullptr,
                    nullptr, nullptr, dy, dxp, dz, ddt_raw, dB, dC, dA_log, dD, dconv_w, dconv_b,
                    ddt_bias, nullptr, nullptr, workspace, workspace_bytes, cuda_stream, h_ckpt);
}

int mamba_mixer_bwd_packed(const mamba_dims* dims, const void* xp, const void* z,
                           const void* dt_raw, const void* B, const void* C, const float* A_log,
                           const float* D, const float* conv_w, const float* conv_b,
                           const float* dt_bias, const int32_t* seq_idx, const float* h_in,
                           const void* conv_state_in, const void* dy, float* dxp, float* dz,
                           float* ddt_raw, float* dB, float* dC, float* dA_log, float* dD,
                           float* dconv_w, float* dconv_b, float* ddt_bias, float* dh_in,
                           float* dconv_state_in, void* workspace, size_t workspace_bytes,
                           void* cuda_stream) {
  return bwd_common(dims, xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, seq_idx, h_in,
                    conv_state_in, dy, dxp, dz, ddt_raw, dB, dC, dA_log, dD, dconv_w, dconv_b,
                    ddt_bias, dh_in, dconv_state_in, workspace, workspace_bytes, cuda_stream);
}

int mamba_mixer_step(const mamba_dims* dims, const void* xp, const void* z, const void* dt_raw,
                     const void* B, const void* C, const float* A_log, const float* D,
                     const float* conv_w, const float* conv_b, const float* dt_bias,
                     const float* h_in, const void* conv_state_in, void* y, float* h_out,
                     void* conv_state_out, void* cuda_stream) {
  Sizes s;
  int rc = check_dims(dims, &s);
  if (rc) return rc;
  if (dims->seqlen != 1)
    return fail(MAMBA_ERR_INVALID_ARGUMENT, "step needs seqlen == 1 (got %lld)",
                (long long)dims->seqlen);
  const bool act = s.act > 0;
  const bool st_ = s.state > 0;
  if ((rc = check_ptr(xp, "xp", act, 16)) || (rc = check_ptr(z, "z", act, 16)) ||
      (rc = check_ptr(dt_raw, "dt_raw", act, 16)) || (rc = check_ptr(B, "B", act, 16)) ||
      (rc = check_ptr(C, "C", act, 16)) || (rc = check_ptr(y, "y", act, 16)) ||
      (rc = check_ptr(A_log, "A_log", dims->d_inner > 0, 16)) ||
      (rc = check_ptr(D, "D", dims->d_inner > 0, 4)) ||
      (rc = check_ptr(conv_w, "conv_w", dims->d_inner > 0, 16)) ||
      (rc = check_ptr(conv_b, "conv_b", false, 4)) ||
      (rc = check_ptr(dt_bias, "dt_bias", dims->d_inner > 0, 4)) ||
      (rc = check_ptr(h_in, "h_in", st_, 16)) || (rc = check_ptr(h_out, "h_out", st_, 16)) ||
      (rc = check_ptr(conv_state_in, "conv_state_in", st_, 2)) ||
      (rc = check_ptr(conv_state_out, "conv_state_out", st_, 2)))
    return rc;
  const int64_t Di = dims->d_inner, N = dims->d_state;
  const Span ins[] = {{xp, size_t(s.act) * s.esize, "xp"},   {z, size_t(s.act) * s.esize, "z"},
                      {dt_raw, size_t(s.act) * s.esize, "dt_raw"},
                      {B, size_t(s.bc) * s.esize, "B"},     {C, size_t(s.bc) * s.esize, "C"},
                      {A_log, size_t(Di * N) * 4, "A_log"}, {D, size_t(Di) * 4, "D"},
                      {conv_w, size_t(Di) * 16, "conv_w"},  {conv_b, size_t(Di) * 4, "conv_b"},
                      {dt_bias, size_t(Di) * 4, "dt_bias"}};
  const Span h_in_s{h_in, size_t(s.state) * 4, "h_in"};
  const Span cs_in_s{conv_state_in, size_t(s.cstate) * s.esize, "conv_state_in"};
  const Span y_s{y, size_t(s.act) * s.esize, "y"};
  const Span h_out_s{h_out, size_t(s.state) * 4, "h_out"};
  const Span cs_out_s{conv_state_out, size_t(s.cstate) * s.esize, "conv_state_out"};
  const Span outs[] = {y_s, h_out_s, cs_out_s};
  for (const Span& o : outs)
    for (const Span& i : ins)
      if (overlaps(o, i)) return fail(MAMBA_ERR_INVALID_ARGUMENT, "%s overlaps %s", o.name, i.name);
  if (overlaps(y_s, h_out_s) || overlaps(y_s, cs_out_s) || overlaps(h_out_s, cs_out_s) ||
      overlaps(y_s, h_in_s) || overlaps(y_s, cs_in_s))
    return fail(MAMBA_ERR_INVALID_ARGUMENT, "output buffers overlap");
  // in place is allowed only as exact aliasing
  if (overlaps(h_out_s, h_in_s) && h_out != h_in)
    return fail(MAMBA_ERR_INVALID_ARGUMENT, "h_out partially overlaps h_in");
  if (overlaps(cs_out_s, cs_in_s) && conv_state_out != conv_state_in)
    return fail(MAMBA_ERR_INVALID_ARGUMENT, "conv_state_out partially overlaps conv_state_in");
  if (overlaps(h_out_s, cs_in_s) || overlaps(cs_out_s, h_in_s))
    return fail(MAMBA_ERR_INVALID_ARGUMENT, "state outputs overlap the other state input");
  if (dims->batch == 0 || Di == 0) return ok();

  mm::StepArgs a{};
  a.xp = xp; a.z = z; a.dt = dt_raw; a.B = B; a.C = C;
  a.A_log = A_log; a.D = D; a.conv_w = conv_w; a.conv_b = conv_b; a.dt_bias = dt_bias;
  a.h_in = h_in; a.cs_in = conv_state_in; a.y = y; a.h_out = h_out; a.cs_out = conv_state_out;
  a.batch = dims->batch; a.Di = Di;
  {
    void* sp = nullptr;
    char why[256];
    if (mm_host::symbol_in_context(reinterpret_cast<const void*>(&g_step_status), &sp,
                                   "mamba_mixer_step", why, sizeof(why)) != 0)
      return fail(MAMBA_ERR_CUDA, "%s", why);
    a.status = static_cast<int*>(sp);
  }
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t e;
  const bool f32 = dims->io_dtype == MAMBA_F32;
  if (N == 16)
    e = f32 ? launch_step<16, float, true>(a, st) : launch_step<16, __nv_bfloat16, false>(a, st);
  else
    e = f32 ? launch_step<8, float, true>(a, st) : launch_step<8, __nv_bfloat16, false>(a, st);
  if (e != cudaSuccess)
    return fail(MAMBA_ERR_CUDA, "step launch failed: %s", cudaGetErrorString(e));
  return ok();
}

}  // extern "C"
