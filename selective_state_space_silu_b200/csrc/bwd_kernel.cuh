// Backward of the fused mixer core, by forward recompute (calm-mamba 0.1.4, section "GPU
// acceleration (Triton kernels)": the scan's backward recomputes the forward).
//
// Gradients of sum(dy * y) for a forward from zero state, in fp32 (the openfluke stress
// test keeps boundary gradients in Float32):
//   per (b, t, d): dxp, dz, ddt_raw;  per (b, t, n): dB, dC (summed over the channels);
//   per d: dA_log, dD, dconv_w, dconv_b, ddt_bias (summed over batch and time).
//
// CTA = one batch row x 32 channels, 128 threads = 4 warps of 8 channels x 4 lanes; lane
// (chl = lane & 7, j = lane >> 3) owns states [j*kS, (j+1)*kS) of channel chl, as in the
// forward's scan warps.  Two sweeps over time:
//   forward  -- the recurrence from zero, storing the state at the start of every 16-step
//               tile (workspace, fp32 [batch, tiles, d_inner, d_state]);
//   reverse  -- tiles last to first: reload the tile's start state, recompute its 16
//               states h_t and per-(t, d) scalars (pre-activations and their sigmoids)
//               into shared memory, then walk the tile
//               backwards with the adjoint state lam (lam += dyc*C; gradients; lam *= a).
// Each tile's inputs are staged in shared memory one tile ahead (16-byte cp.async by all
// threads, two slots).  The conv's input gradient needs dpre of the 3 following steps,
// which the reverse walk has just produced: a 3-value window per channel carries it across
// tiles.  dB and dC are
// summed over the 8 channels of a warp by butterflies, over the 4 warps in shared memory,
// and over CTAs (channel tiles) with global atomics; the per-d gradients are summed over
// batch rows with global atomics.  The gradient outputs must be zero on entry.
//
// Time chunks (long rows with few channel tiles): chunk c starts its forward sweep from the
// state carried through chunks 0..c-1 (the forward's chunk-state pass gives each chunk's
// decay product P and end state H from zero: h = P*h + H) and its reverse walk from the
// adjoint carried back from chunks c+1..C-1, composed the same way from each chunk's P and
// its adjoint carried out from zero (Lambda, written by this kernel's kAdj instance).  The
// input gradient of a chunk's last 3 steps also takes dpre of the next chunk's first 3: both
// chunks add their parts atomically into those (zeroed) rows.
//
// Documents and a cached start (kExt instances, mamba_mixer_bwd_packed): where seq_idx
// changes at step t, the conv taps before t carry no gradient and the state entering t is
// zero, so the adjoint is cut there (lam = 0 after step t); the adjoint left after step 0 is
// the gradient of h_in, and the conv input gradient of the 3 positions before 0 is that of
// conv_state_in.
#pragma once

#include <float.h>

#include <type_traits>

#include "device_math.cuh"
#include "sm100_primitives.cuh"

namespace mm {

struct BwdParams {
  const void* xp;
  const void* z;
  const void* dt;
  const void* B;
  const void* C;
  const void* dy;
  const float* A_log;
  const float* D;
  const float* conv_w;
  const float* conv_b;   // may be null
  const float* dt_bias;
  float* dxp;
  float* dz;
  float* ddt;
  float* dB;
  float* dC;
  float* dA_log;
  float* dD;
  float* dconv_w;
  float* dconv_b;        // may be null
  float* ddt_bias;
  float* ws_h;           // [batch, tiles, d_inner, N] tile start states
  int states_given;      // 1: ws_h already holds them (the forward's checkpoints), no forward sweep
  int64_t L, Di;
  int ntiles;            // 16-step tiles over the whole sequence
  // time chunks (as the forward's plan; chunk_len a multiple of the tile length)
  int64_t chunk_len;
  int nchunks;
  const float* ws_P;     // [batch, nchunks-1, d_inner, N] decay product of each chunk
  const float* ws_H;     // [batch, nchunks-1, d_inner, N] end state of each chunk from zero
  float* ws_L;           // [batch, nchunks, d_inner, N] adjoint carried out of each chunk from zero
};

// Extra arguments of the kExt instances (documents and a cached start; each may be null).
// Only those instances take them, so the plain kernels' argument block stays as it is.
struct BwdParamsExt : BwdParams {
  const int32_t* seq_idx;  // [batch, L] document ids
  const float* h_in;       // [batch, d_inner, N] state before token 0
  const void* cs_in;       // [batch, d_inner, 3] conv window before token 0
  float* dh_in;            // [batch, d_inner, N] gradient of h_in
  float* dcs_in;           // [batch, d_inner, 3] gradient of conv_state_in (fp32)
};
template <bool kExt>
using BwdArgs = typename std::conditional<kExt, BwdParamsExt, BwdParams>::type;

constexpr int kBwdThreads = 128;
constexpr int kBwdCh = 32;
constexpr int kBwdT = 16;       // steps per tile
constexpr int kBwdHalo = 4;     // x' rows staged before a tile (3 needed)

template <int N, typename IO>
struct BwdSmem {
  static constexpr int kS = N / 4;
  static constexpr int kEs = int(sizeof(IO));
  static constexpr int kRow = kBwdCh * kEs;                  // one step of 32 channels
  static constexpr int kBCRow = N * kEs;                     // one step of B (or C)
  // one staging slot: x' (with halo), dt_raw, z, dy, B, C of one tile
  static constexpr int kXOff = 0;
  static constexpr int kDtOff = kXOff + (kBwdT + kBwdHalo) * kRow;
  static constexpr int kZOff = kDtOff + kBwdT * kRow;
  static constexpr int kDyOff = kZOff + kBwdT * kRow;
  static constexpr int kBOff = kDyOff + kBwdT * kRow;
  static constexpr int kCOff = kBOff + kBwdT * kBCRow;
  static constexpr int kSlot = kCOff + kBwdT * kBCRow;
  static constexpr int kHs = kBwdT * kBwdThreads * kS * 4;   // h_t per (step, lane)
  static constexpr int kSc = kBwdT * kBwdCh * 16;            // {Delta, u, dyc, 0} per (step, ch)
  static constexpr int kSc2 = kBwdT * kBwdCh * 16;           // {SiLU'(pre), s(v), gate', 0}
  static constexpr int kE = kBwdT * kBwdCh * 16;             // {C.h, lam.B, sum ah A, dpre}
  static constexpr int kDn = 4 * kBwdCh * 4;                 // dpre of the later tile's steps 0..2
  static constexpr int kAcc = 2 * kBwdT * N * 4;              // dB, dC partial sums per tile
  static constexpr int kHsOff = 2 * kSlot;
  static constexpr int kScOff = kHsOff + kHs;
  static constexpr int kSc2Off = kScOff + kSc;
  static constexpr int kEOff = kSc2Off + kSc2;
  static constexpr int kDnOff = kEOff + kE;
  static constexpr int kAccOff = kDnOff + kDn;
  static constexpr int kTotal = kAccOff + kAcc;
  static_assert(kSlot % 16 == 0 && kRow % 16 == 0 && kBCRow % 16 == 0, "16-byte staging units");
};

// kS consecutive I/O elements as fp32 from shared memory (kS = 4 or 2).
template <int kS, typename IO>
__device__ __forceinline__ void lds_io_row(uint32_t a, float* out) {
  if constexpr (sizeof(IO) == 4) {
    if constexpr (kS == 4) {
      const float4 v = lds_f32x4(a);
      out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    } else {
      out[0] = lds_f32(a); out[1] = lds_f32(a + 4);
    }
  } else {
    if constexpr (kS == 4) {
      uint32_t w0, w1;
      asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w0), "=r"(w1) : "r"(a));
      out[0] = __uint_as_float(w0 << 16); out[1] = __uint_as_float(w0 & 0xffff0000u);
      out[2] = __uint_as_float(w1 << 16); out[3] = __uint_as_float(w1 & 0xffff0000u);
    } else {
      uint32_t w0;
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w0) : "r"(a));
      out[0] = __uint_as_float(w0 << 16); out[1] = __uint_as_float(w0 & 0xffff0000u);
    }
  }
}

// A lane's kS fp32 states at shared address a (16- or 8-byte aligned): one vector access.
template <int kS>
__device__ __forceinline__ void sts_states(uint32_t a, const float* v) {
  if constexpr (kS == 4)
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(v[0]), "f"(v[1]),
                 "f"(v[2]), "f"(v[3]) : "memory");
  else
    asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(a), "f"(v[0]), "f"(v[1]) : "memory");
}
template <int kS>
__device__ __forceinline__ void lds_states(uint32_t a, float* v) {
  if constexpr (kS == 4) {
    const float4 x = lds_f32x4(a);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  } else {
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v[0]), "=f"(v[1]) : "r"(a));
  }
}

template <typename IO>
__device__ __forceinline__ float lds_one(uint32_t a) {
  if constexpr (sizeof(IO) == 4) return lds_f32(a);
  else return __uint_as_float(lds_u16(a) << 16);
}

// 16 bytes global -> shared (L2 only), or 16 zero bytes when !valid (src-size 0: the source
// is not read; a valid address is passed all the same).
__device__ __forceinline__ void cp_async16_zfill(uint32_t sdst, const void* gsrc, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sdst), "l"(gsrc),
               "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit_() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int kPending>
__device__ __forceinline__ void cp_async_wait_() {
  asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory");
}

template <bool kPrecise>
__device__ __forceinline__ float sigmoid_(float v) {
  if constexpr (kPrecise) return 1.0f / (1.0f + expf(-v));
  else return rcp_approx(1.0f + ex2_approx(-v * kLog2e));
}

template <int N, typename IO, bool kPrecise, bool kAdj, bool kExt>
__global__ void __launch_bounds__(kBwdThreads, 3)   // 3 CTAs per SM: 70 KB of shared memory each
bwd_kernel(const BwdArgs<kExt> p) {
  using M = Math<kPrecise>;
  using Sm = BwdSmem<N, IO>;
  constexpr int kS = N / 4;
  constexpr int kEs = Sm::kEs;
  extern __shared__ __align__(16) unsigned char smem[];
  const uint32_t sb = smem_addr(smem);
  const uint32_t hsa = sb + uint32_t(Sm::kHsOff) + uint32_t(threadIdx.x * (N / 4) * 4);  // this lane's h_t slots
  float4* sc = reinterpret_cast<float4*>(smem + Sm::kScOff);
  float4* sc2 = reinterpret_cast<float4*>(smem + Sm::kSc2Off);
  float4* E = reinterpret_cast<float4*>(smem + Sm::kEOff);
  float* dnext = reinterpret_cast<float*>(smem + Sm::kDnOff);   // [3][kBwdCh]
  float* acc = reinterpret_cast<float*>(smem + Sm::kAccOff);   // [2][T][N]

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int chl = lane & 7;
  const int j = lane >> 3;
  const int cl = warp * 8 + chl;
  const int64_t d0 = int64_t(blockIdx.x) * kBwdCh;
  const int64_t b = blockIdx.y;
  // d_inner % 8 == 0: a warp's 8 channels are all in range or all out; an out-of-range warp
  // takes part in the barriers and shuffles on zero-filled data and stores nothing
  const bool active = d0 + cl < p.Di;
  const int64_t d = active ? d0 + cl : 0;
  const int64_t L = p.L, Di = p.Di;
  // this CTA's time chunk (the kAdj instance runs chunks 1..C-1)
  const int c = kAdj ? int(blockIdx.z) + 1 : int(blockIdx.z);
  const int64_t t_begin = int64_t(c) * p.chunk_len;
  const int64_t t_end = t_begin + p.chunk_len < L ? t_begin + p.chunk_len : L;
  const int kb = int(t_begin / kBwdT);                        // first and one-past-last tile
  const int ke = int((t_end + kBwdT - 1) / kBwdT);

  // Stage tile k into slot `slot`: x' rows t0-4 .. t0+T-1, dt_raw and B rows t0 .. t0+T-1,
  // and with `all` also z, dy and C; 16-byte units copied by all threads; rows outside
  // [0, L) and channels past d_inner read as zeros.
  auto stage = [&](int k, int slot, bool all) {
    const int64_t t0 = int64_t(k) * kBwdT;
    const uint32_t base = sb + uint32_t(slot * Sm::kSlot);
    constexpr int kU = Sm::kRow / 16;                 // units per staged row of 32 channels
    constexpr int kUbc = Sm::kBCRow / 16;             // units per row of B or C
    constexpr int nx = (kBwdT + kBwdHalo) * kU;
    constexpr int nr = kBwdT * kU;
    constexpr int nbc = kBwdT * kUbc;
    const int nrows = all ? 3 : 1;                    // dt (, z, dy)
    const int nbcs = all ? 2 : 1;                     // B (, C)
    const int total = nx + nr * nrows + nbc * nbcs;
    for (int e = tid; e < total; e += kBwdThreads) {
      const unsigned char* src;
      uint32_t dst;
      bool ok;
      if (e < nx + nr * nrows) {
        int arr = 0, r = e;                            // arr: 0 x', 1 dt, 2 z, 3 dy
        if (r >= nx) { r -= nx; arr = 1 + r / nr; r %= nr; }
        const int row = r / kU, u = r % kU;
        const int64_t t = t0 + row - (arr == 0 ? kBwdHalo : 0);
        const int64_t ch = d0 + int64_t(u) * (16 / kEs);
        ok = t >= 0 && t < L && ch < Di;
        const void* g = arr == 0 ? p.xp : arr == 1 ? p.dt : arr == 2 ? p.z : p.dy;
        src = static_cast<const unsigned char*>(g) + (ok ? ((b * L + t) * Di + ch) * kEs : 0);
        const int off = arr == 0 ? Sm::kXOff : arr == 1 ? Sm::kDtOff : arr == 2 ? Sm::kZOff
                                                                               : Sm::kDyOff;
        dst = base + uint32_t(off + r * 16);
      } else {
        int r = e - nx - nr * nrows;
        const int arr = r / nbc;                       // 0 B, 1 C
        r %= nbc;
        const int row = r / kUbc, u = r % kUbc;
        const int64_t t = t0 + row;
        ok = t < L;
        const void* g = arr == 0 ? p.B : p.C;
        src = static_cast<const unsigned char*>(g) + (ok ? (b * L + t) * N * kEs + u * 16 : 0);
        dst = base + uint32_t((arr == 0 ? Sm::kBOff : Sm::kCOff) + r * 16);
      }
      cp_async16_zfill(dst, src, ok);
    }
    cp_async_commit_();
  };

  // Document ids of steps t0-4 .. t0+15 of tile k, one per lane (lanes 0..19), and the reset
  // bits they give: bit i + 4 set when step t0 + i starts a document (i >= -3).
  [[maybe_unused]] auto ids_for = [&](int k) -> int32_t {
    if constexpr (kExt) {
      const int64_t T = int64_t(k) * kBwdT - 4 + lane;
      if (p.seq_idx && lane < kBwdT + 4 && T >= 0 && T < L) return __ldg(p.seq_idx + b * L + T);
    }
    return 0;
  };
  [[maybe_unused]] auto reset_bits = [&](int k, int32_t id) -> uint32_t {
    if constexpr (kExt) {
      if (!p.seq_idx) return 0u;
      const int64_t T = int64_t(k) * kBwdT - 4 + lane;
      const int32_t prv = __shfl_up_sync(0xffffffffu, id, 1);
      return __ballot_sync(0xffffffffu, lane >= 1 && lane < kBwdT + 4 && T >= 1 && T < L &&
                                            id != prv);
    }
    return 0u;
  };
  // x' of step t < 0 from the cached conv window (zero without one)
  [[maybe_unused]] auto x_before = [&](int64_t t) -> float {
    if constexpr (kExt) {
      if (p.cs_in) return IOT<IO>::to_f(static_cast<const IO*>(p.cs_in)[(b * Di + d) * 3 + (3 + t)]);
    }
    return 0.0f;
  };

  float A[kS], A2[kS];
#pragma unroll
  for (int s = 0; s < kS; ++s) {
    const float al = __ldg(p.A_log + d * N + j * kS + s);
    A[s] = fmaxf(-expf(al), -FLT_MAX);              // A = -exp(A_log), for the gradients
    A2[s] = fmaxf(M::neg_exp(al) * M::a_scale(), -FLT_MAX);   // as the forward holds it
  }
  // one step of the forward recurrence; with a reset at this step the entering state is zero
  auto step_state = [&](float* h, float del, float du, const float* Bv, bool reset) {
#pragma unroll
    for (int s = 0; s < kS; ++s) {
      const float a = M::decay(del, A2[s]);
      h[s] = (reset ? 0.0f : a * h[s]) + du * Bv[s];
    }
  };
  const float w0 = __ldg(p.conv_w + d * 4 + 0), w1 = __ldg(p.conv_w + d * 4 + 1);
  const float w2 = __ldg(p.conv_w + d * 4 + 2), w3 = __ldg(p.conv_w + d * 4 + 3);
  const float cb = p.conv_b ? __ldg(p.conv_b + d) : 0.0f;
  const float dtb = __ldg(p.dt_bias + d);
  const float Dd = __ldg(p.D + d);
  // the conv pre-activation of step t0 + i from x' of steps t-3..t (taps before a document
  // start dropped): bits are the tile's reset bits
  auto conv_pre = [&](float xa, float xb, float xc, float xt, uint32_t bits, int i) {
    const bool m1 = !((bits >> (i + 4)) & 1u);
    const bool m2 = m1 && !((bits >> (i + 3)) & 1u);
    const bool m3 = m2 && !((bits >> (i + 2)) & 1u);
    return cb + w0 * (m3 ? xa : 0.0f) + w1 * (m2 ? xb : 0.0f) + w2 * (m1 ? xc : 0.0f) + w3 * xt;
  };
  float* ck = p.ws_h + ((b * p.ntiles) * Di + d) * N + j * kS;   // + k * Di * N per tile
  const uint32_t colx = uint32_t(cl * kEs);
  const uint32_t colbc = uint32_t(j * kS * kEs);
  // The per-(t, d) scalars of a tile, computed once per (t, d): the 4 lanes of a channel take
  // steps j, j+4, j+8, j+12.  sc gets {Delta, u, dyc, 0}; with kFull (the reverse sweep,
  // whose tiles also hold z and dy) dyc = dy*z*s(z) is the gated output's gradient and sc2
  // gets {SiLU'(pre), s(v), dy*SiLU'(z), 0}, s the logistic function.  xr(i) is x' of step
  // t0 + i (i >= -3).
  auto tile_scalars = [&](auto full_tag, uint32_t sl, int cnt, uint32_t bits, auto xr) {
    constexpr bool kFull = decltype(full_tag)::value;
#pragma unroll
    for (int m = 0; m < kBwdT / 4; ++m) {
      const int i = j + 4 * m;
      if (i < cnt) {
        const float pre = conv_pre(xr(i - 3), xr(i - 2), xr(i - 1), xr(i), bits, i);
        const float v = lds_one<IO>(sl + Sm::kDtOff + i * Sm::kRow + colx) + dtb;
        const float sp = sigmoid_<kPrecise>(pre);
        const float u = pre * sp;
        float dyc = 0.0f;
        if constexpr (kFull) {
          const float zt = lds_one<IO>(sl + Sm::kZOff + i * Sm::kRow + colx);
          const float dyt = lds_one<IO>(sl + Sm::kDyOff + i * Sm::kRow + colx);
          const float sz = sigmoid_<kPrecise>(zt);
          dyc = dyt * zt * sz;
          sc2[i * kBwdCh + cl] = make_float4(sp * (1.0f + pre * (1.0f - sp)), sigmoid_<kPrecise>(v),
                                             dyt * (sz * (1.0f + zt * (1.0f - sz))), 0.0f);
        }
        sc[i * kBwdCh + cl] = make_float4(M::softplus(v), u, dyc, 0.0f);
      }
    }
    __syncwarp();
  };

  if constexpr (kAdj) {
    // ---- adjoint carried out of chunk c from zero, last step first:
    //      lam += dyc*C; lam = reset ? 0 : a*lam
    float lam[kS];
#pragma unroll
    for (int s = 0; s < kS; ++s) lam[s] = 0.0f;
    stage(ke - 1, 0, true);
    int32_t id = ids_for(ke - 1);
    for (int k = ke - 1, it = 0; k >= kb; --k, ++it) {
      if (k - 1 >= kb) stage(k - 1, (it + 1) & 1, true);
      else cp_async_commit_();
      const uint32_t bits = reset_bits(k, id);
      if (k - 1 >= kb) id = ids_for(k - 1);
      cp_async_wait_<1>();
      __syncthreads();
      const uint32_t sl = sb + uint32_t((it & 1) * Sm::kSlot);
      const int64_t t0 = int64_t(k) * kBwdT;
      const int cnt = int(t0 + kBwdT < t_end ? kBwdT : t_end - t0);
#pragma unroll 2
      for (int i = cnt - 1; i >= 0; --i) {
        const float del = M::softplus(lds_one<IO>(sl + Sm::kDtOff + i * Sm::kRow + colx) + dtb);
        const float zt = lds_one<IO>(sl + Sm::kZOff + i * Sm::kRow + colx);
        const float dyc = lds_one<IO>(sl + Sm::kDyOff + i * Sm::kRow + colx) * zt * sigmoid_<kPrecise>(zt);
        const bool reset = (bits >> (i + 4)) & 1u;
        float Cv[kS];
        lds_io_row<kS, IO>(sl + Sm::kCOff + i * Sm::kBCRow + colbc, Cv);
#pragma unroll
        for (int s = 0; s < kS; ++s)
          lam[s] = reset ? 0.0f : (lam[s] + dyc * Cv[s]) * M::decay(del, A2[s]);
      }
      __syncthreads();
    }
    cp_async_wait_<0>();
    if (active) {
      float* o = p.ws_L + ((b * p.nchunks + c) * Di + d) * N + j * kS;
#pragma unroll
      for (int s = 0; s < kS; ++s) o[s] = lam[s];
    }
  } else {
    // ---- forward sweep: tile start states, from the state carried into this chunk (not
    // needed when the forward left them: mamba_mixer_fwd_ckpt)
    if (!p.states_given) {
      float h[kS];
#pragma unroll
      for (int s = 0; s < kS; ++s) h[s] = 0.0f;
      if constexpr (kExt) {
        if (p.h_in) {
#pragma unroll
          for (int s = 0; s < kS; ++s) h[s] = __ldg(p.h_in + (b * Di + d) * N + j * kS + s);
        }
      }
      for (int cc = 0; cc < c; ++cc) {
        const int64_t o = ((b * (p.nchunks - 1) + cc) * Di + d) * N + j * kS;
#pragma unroll
        for (int s = 0; s < kS; ++s) h[s] = p.ws_P[o + s] * h[s] + p.ws_H[o + s];
      }
      stage(kb, 0, false);
      int32_t id = ids_for(kb);
      for (int k = kb, it = 0; k < ke; ++k, ++it) {
        if (k + 1 < ke) stage(k + 1, (it + 1) & 1, false);
        else cp_async_commit_();
        const uint32_t bits = reset_bits(k, id);
        if (k + 1 < ke) id = ids_for(k + 1);
        if (active) {
#pragma unroll
          for (int s = 0; s < kS; ++s) ck[int64_t(k) * Di * N + s] = h[s];
        }
        cp_async_wait_<1>();
        __syncthreads();
        const uint32_t sl = sb + uint32_t((it & 1) * Sm::kSlot);
        const int64_t t0 = int64_t(k) * kBwdT;
        const int cnt = int(t0 + kBwdT < t_end ? kBwdT : t_end - t0);
        tile_scalars(std::false_type{}, sl, cnt, bits, [&](int i) {
          if (kExt && t0 + i < 0) return x_before(t0 + i);
          return lds_one<IO>(sl + Sm::kXOff + uint32_t((i + kBwdHalo) * Sm::kRow) + colx);
        });
#pragma unroll 2
        for (int i = 0; i < cnt; ++i) {
          const float4 q = sc[i * kBwdCh + cl];
          float Bv[kS];
          lds_io_row<kS, IO>(sl + Sm::kBOff + i * Sm::kBCRow + colbc, Bv);
          step_state(h, q.x, q.x * q.y, Bv, (bits >> (i + 4)) & 1u);
        }
        __syncthreads();   // the slot (and sc) are refilled by the next iteration
      }
    }

    // ---- reverse sweep
    float lam[kS], dA[kS];
#pragma unroll
    for (int s = 0; s < kS; ++s) { lam[s] = 0.0f; dA[s] = 0.0f; }
    // the adjoint carried back into this chunk: lam = P_c' * lam + Lambda_c', c' = C-1 .. c+1
    for (int cc = p.nchunks - 1; cc > c; --cc) {
      const int64_t oL = ((b * p.nchunks + cc) * Di + d) * N + j * kS;
      const int64_t oP = ((b * (p.nchunks - 1) + cc) * Di + d) * N + j * kS;
#pragma unroll
      for (int s = 0; s < kS; ++s)
        lam[s] = (cc < p.nchunks - 1 ? p.ws_P[oP + s] * lam[s] : 0.0f) + p.ws_L[oL + s];
    }
    // per-d gradient sums of this lane's steps (reduced over the channel's 4 lanes at the end)
    float aD = 0.0f, aDtb = 0.0f, aCb = 0.0f, aW0 = 0.0f, aW1 = 0.0f, aW2 = 0.0f, aW3 = 0.0f;
    for (int i = tid; i < 2 * kBwdT * N; i += kBwdThreads) acc[i] = 0.0f;
    // no tile after the chunk's last: the dpre of the steps after it count as zero here (the
    // next chunk adds its own part of those input gradients)
    if (j < 3) dnext[j * kBwdCh + cl] = 0.0f;
    uint32_t bits_later = 0u;   // reset bits of the tile after the current one
    __syncthreads();   // also orders this thread's checkpoint stores before its reloads

    float hn[kS];   // start state of the tile processed next (loaded one tile ahead)
#pragma unroll
    for (int s = 0; s < kS; ++s) hn[s] = ck[int64_t(ke - 1) * Di * N + s];
    stage(ke - 1, 0, true);
    int32_t id = ids_for(ke - 1);
    // no reset at s, s-1, .., s-r+1 (step s of a tile with reset bits `bt`): the conv tap r
    // of step s (x' of step s - r) reaches its pre-activation
    auto tap_live = [](uint32_t bt, int s, int r) -> bool {
      return ((bt >> (s + 5 - r)) & ((1u << r) - 1u)) == 0u;
    };
    for (int k = ke - 1, it = 0; k >= kb; --k, ++it) {
      if (k - 1 >= kb) stage(k - 1, (it + 1) & 1, true);
      else cp_async_commit_();
      const uint32_t bits = reset_bits(k, id);
      if (k - 1 >= kb) id = ids_for(k - 1);
      float h0[kS], h[kS];
#pragma unroll
      for (int s = 0; s < kS; ++s) h0[s] = h[s] = hn[s];
      if (k - 1 >= kb) {
#pragma unroll
        for (int s = 0; s < kS; ++s) hn[s] = ck[int64_t(k - 1) * Di * N + s];
      }
      cp_async_wait_<1>();
      __syncthreads();
      const uint32_t sl = sb + uint32_t((it & 1) * Sm::kSlot);
      const int64_t t0 = int64_t(k) * kBwdT;
      const int cnt = int(t0 + kBwdT < t_end ? kBwdT : t_end - t0);
      auto xrow = [&](int i) {   // x' of step t0 + i, i >= -4 (the halo rows)
        if (kExt && t0 + i < 0) return x_before(t0 + i);
        return lds_one<IO>(sl + Sm::kXOff + uint32_t((i + kBwdHalo) * Sm::kRow) + colx);
      };

      // recompute the tile: the per-(t, d) scalars, then the states h_t
      tile_scalars(std::true_type{}, sl, cnt, bits, xrow);
#pragma unroll 2
      for (int i = 0; i < cnt; ++i) {
        const float4 q = sc[i * kBwdCh + cl];
        float Bv[kS];
        lds_io_row<kS, IO>(sl + Sm::kBOff + i * Sm::kBCRow + colbc, Bv);
        step_state(h, q.x, q.x * q.y, Bv, (bits >> (i + 4)) & 1u);
        sts_states<kS>(hsa + uint32_t(i * kBwdThreads * kS * 4), h);
      }
      __syncwarp();

      // walk the tile backwards with the adjoint state; per step, this lane's partial sums
      // of C.h, lam.B and sum_n lam h_{t-1} a A go to the step's record (one per lane after a
      // reduce-scatter over the channel's 4 lanes), dB and dC to the tile's sums
      float ht[kS];
      lds_states<kS>(hsa + uint32_t((cnt - 1) * kBwdThreads * kS * 4), ht);
#pragma unroll 4
      for (int i = cnt - 1; i >= 0; --i) {
        const bool m1 = !((bits >> (i + 4)) & 1u);           // no reset at t
        const float4 q = sc[i * kBwdCh + cl];
        const float del = q.x, u = q.y, dyc = q.z;
        const float delu = del * u;
        float Bv[kS], Cv[kS], hp[kS];
        lds_io_row<kS, IO>(sl + Sm::kBOff + i * Sm::kBCRow + colbc, Bv);
        lds_io_row<kS, IO>(sl + Sm::kCOff + i * Sm::kBCRow + colbc, Cv);
        if (i > 0) {
          lds_states<kS>(hsa + uint32_t((i - 1) * kBwdThreads * kS * 4), hp);
        } else {
#pragma unroll
          for (int s = 0; s < kS; ++s) hp[s] = h0[s];
        }
        float ycp = 0.0f, lamB = 0.0f, ahA = 0.0f, cB[kS], cC[kS];
#pragma unroll
        for (int s = 0; s < kS; ++s) {
          const float hin = m1 ? hp[s] : 0.0f;                 // the state entering step t
          ycp += Cv[s] * ht[s];
          const float a = M::decay(del, A2[s]);
          lam[s] += dyc * Cv[s];
          cB[s] = lam[s] * delu;
          cC[s] = dyc * ht[s];
          lamB += lam[s] * Bv[s];
          const float ah = lam[s] * hin * a;
          ahA += ah * A[s];
          dA[s] += ah * del;
          lam[s] = m1 ? lam[s] * a : 0.0f;
          ht[s] = hp[s];                                       // h_t of step t - 1
        }
        // reduce-scatter of {C.h, lam.B, sum ah A} over the channel's 4 lanes (lane bits 4,
        // 3): lane j ends with the channel's sum of value j (lane 3 with nothing)
        {
          const bool hi = (j & 2) != 0;
          float k0 = hi ? ahA : ycp, k1 = hi ? 0.0f : lamB;
          const float s0 = hi ? ycp : ahA, s1 = hi ? lamB : 0.0f;
          k0 += __shfl_xor_sync(0xffffffffu, s0, 16);
          k1 += __shfl_xor_sync(0xffffffffu, s1, 16);
          const bool odd = (j & 1) != 0;
          float kp = odd ? k1 : k0;
          kp += __shfl_xor_sync(0xffffffffu, odd ? k0 : k1, 8);
          if (j < 3) reinterpret_cast<float*>(E + i * kBwdCh + cl)[j] = kp;
        }
        // dB, dC summed over the warp's 8 channels (lane bits 0..2) by a reduce-scatter:
        // the 2*kS values {cB, cC} are halved at each round, so lane chl ends with value chl
        // (kS = 4) or, after a last all-reduce round, value chl >> 1 (kS = 2)
        {
          float vv[2 * kS];
#pragma unroll
          for (int s = 0; s < kS; ++s) { vv[s] = cB[s]; vv[kS + s] = cC[s]; }
          int m = 4;
#pragma unroll
          for (int half = kS; half >= 1; half >>= 1, m >>= 1) {
            const bool hi = (chl & m) != 0;
#pragma unroll
            for (int e = 0; e < half; ++e) {
              const float keep = hi ? vv[half + e] : vv[e];
              const float send = hi ? vv[e] : vv[half + e];
              vv[e] = keep + __shfl_xor_sync(0xffffffffu, send, m);
            }
          }
          int idx = chl;                                   // kS = 4: 3 rounds, one value each
          if constexpr (kS == 2) {
            vv[0] += __shfl_xor_sync(0xffffffffu, vv[0], 1);
            idx = chl >> 1;
          }
          if (active && (kS == 4 || (chl & 1) == 0)) {
            const int which = idx / kS, s = idx % kS;     // 0: dB, 1: dC
            atomicAdd(&acc[(which * kBwdT + i) * N + j * kS + s], vv[0]);
          }
        }
      }
      __syncwarp();

      // per (t, d), once (lane j takes steps j, j+4, j+8, j+12): the gate, Delta and conv
      // pre-activation gradients
      float dp[kBwdT / 4];
#pragma unroll
      for (int m = 0; m < kBwdT / 4; ++m) {
        const int i = j + 4 * m;
        dp[m] = 0.0f;
        if (i < cnt) {
          const float4 e = E[i * kBwdCh + cl];             // {C.h, lam.B, sum ah A, -}
          const float4 q = sc[i * kBwdCh + cl];            // {Delta, u, dyc, -}
          const float4 g = sc2[i * kBwdCh + cl];           // {SiLU'(pre), s(v), gate', -}
          const float yc = e.x + Dd * q.y;
          const float du = q.x * e.y + q.z * Dd;
          const float dv = (q.y * e.y + e.z) * g.y;        // softplus' = s
          dp[m] = du * g.x;
          reinterpret_cast<float*>(E + i * kBwdCh + cl)[3] = dp[m];
          aD += q.z * q.y;
          aDtb += dv;
          aCb += dp[m];
          if (active) {
            const int64_t o = (b * L + t0 + i) * Di + d;
            p.dz[o] = yc * g.z;
            p.ddt[o] = dv;
          }
        }
      }
      __syncwarp();
      // the conv: x' of step t feeds the pre-activations of steps t .. t+3 (taps 0..3 back);
      // its input gradient takes their dpre, the later tile's first 3 from dnext
#pragma unroll
      for (int m = 0; m < kBwdT / 4; ++m) {
        const int i = j + 4 * m;
        if (i < cnt) {
          const float d0v = dp[m];
          aW3 += d0v * xrow(i);
          if (tap_live(bits, i, 1)) aW2 += d0v * xrow(i - 1);
          if (tap_live(bits, i, 2)) aW1 += d0v * xrow(i - 2);
          if (tap_live(bits, i, 3)) aW0 += d0v * xrow(i - 3);
          float dx = w3 * d0v;
#pragma unroll
          for (int r = 1; r <= 3; ++r) {
            const int sidx = i + r;
            const float wr = r == 1 ? w2 : r == 2 ? w1 : w0;
            if (sidx < cnt) {
              if (tap_live(bits, sidx, r)) dx += wr * reinterpret_cast<const float*>(E + sidx * kBwdCh + cl)[3];
            } else if (sidx >= kBwdT) {
              if (tap_live(bits_later, sidx - kBwdT, r)) dx += wr * dnext[(sidx - kBwdT) * kBwdCh + cl];
            }
          }
          if (active) {
            const int64_t t = t0 + i;
            const int64_t o = (b * L + t) * Di + d;
            if (c < p.nchunks - 1 && t >= t_end - 3) atomicAdd(p.dxp + o, dx);  // + next chunk's part
            else p.dxp[o] = dx;
          }
        }
      }
      __syncwarp();
      if (j < 3) dnext[j * kBwdCh + cl] = dp[0];           // steps 0..2 of this tile, for the next
      bits_later = bits;
      __syncthreads();
      // this tile's dB, dC of the CTA's 32 channels into the global sums
      for (int e = tid; e < 2 * kBwdT * N; e += kBwdThreads) {
        const int which = e / (kBwdT * N), r = e % (kBwdT * N), i = r / N, n = r % N;
        if (i < cnt) {
          float* dst = which ? p.dC : p.dB;
          atomicAdd(dst + (b * L + t0 + i) * N + n, acc[e]);
        }
        acc[e] = 0.0f;
      }
      __syncthreads();
    }
    cp_async_wait_<0>();

    // sums over the channel's 4 lanes (lane bits 3 and 4)
#pragma unroll
    for (int m = 8; m <= 16; m <<= 1) {
      aD += __shfl_xor_sync(0xffffffffu, aD, m);
      aDtb += __shfl_xor_sync(0xffffffffu, aDtb, m);
      aCb += __shfl_xor_sync(0xffffffffu, aCb, m);
      aW0 += __shfl_xor_sync(0xffffffffu, aW0, m);
      aW1 += __shfl_xor_sync(0xffffffffu, aW1, m);
      aW2 += __shfl_xor_sync(0xffffffffu, aW2, m);
      aW3 += __shfl_xor_sync(0xffffffffu, aW3, m);
    }
    if (!active) return;
    // the input gradient of the 3 positions before the chunk from its first 3 steps' dpre
    // (dnext now holds them; bits_later the reset bits of the chunk's first tile)
    if (j == 0) {
      float qv[3];
#pragma unroll
      for (int qq = 1; qq <= 3; ++qq) {
        float v = 0.0f;
#pragma unroll
        for (int r = qq; r <= 3; ++r) {
          const int sidx = r - qq;                           // step of the chunk's first tile
          const float wr = r == 1 ? w2 : r == 2 ? w1 : w0;
          if (sidx < int(t_end - t_begin) && tap_live(bits_later, sidx, r))
            v += wr * dnext[sidx * kBwdCh + cl];
        }
        qv[qq - 1] = v;
      }
      if (c > 0) {
        // this chunk's part of the input gradient of the previous chunk's last 3 steps
        float* o = p.dxp + (b * L + t_begin) * Di + d;
        atomicAdd(o - Di, qv[0]);
        atomicAdd(o - 2 * Di, qv[1]);
        atomicAdd(o - 3 * Di, qv[2]);
      } else if constexpr (kExt) {
        // the conv input gradient of the 3 positions before 0 is that of the initial window
        if (p.dcs_in) {
          float* o = p.dcs_in + (b * Di + d) * 3;
          o[2] = qv[0]; o[1] = qv[1]; o[0] = qv[2];
        }
      }
    }
    if constexpr (kExt) {
      // the adjoint after step 0 is the gradient of the initial state
      if (c == 0 && p.dh_in) {
#pragma unroll
        for (int s = 0; s < kS; ++s) p.dh_in[(b * Di + d) * N + j * kS + s] = lam[s];
      }
    }
#pragma unroll
    for (int s = 0; s < kS; ++s) atomicAdd(p.dA_log + d * N + j * kS + s, dA[s] * A[s]);
    if (j == 0) {
      atomicAdd(p.dD + d, aD);
      atomicAdd(p.ddt_bias + d, aDtb);
      if (p.dconv_b) atomicAdd(p.dconv_b + d, aCb);
      atomicAdd(p.dconv_w + d * 4 + 0, aW0);
      atomicAdd(p.dconv_w + d * 4 + 1, aW1);
      atomicAdd(p.dconv_w + d * 4 + 2, aW2);
      atomicAdd(p.dconv_w + d * 4 + 3, aW3);
    }
  }
}

// Zeroes the 3 rows of dxp before every chunk start (c >= 1), which two chunks then add to.
__global__ void bwd_zero_bounds(float* dxp, int64_t L, int64_t Di, int64_t chunk_len) {
  const int64_t b = blockIdx.y;
  const int64_t t0 = int64_t(blockIdx.x + 1) * chunk_len - 3;
  float* row = dxp + (b * L + t0) * Di;
  for (int64_t e = threadIdx.x; e < 3 * Di; e += blockDim.x) row[e] = 0.0f;
}

}  // namespace mm
