// Single-token decode step on a cached (h, conv state) pair.
//
// kLanes lanes share one channel (b, d) -- 2 by default (measured on 256 x 5120: 43 us
// against 51 us with 4) -- and each owns N/kLanes consecutive states, so the state of a
// warp's channels (32/kLanes x 64 B for N = 16) moves with 16-byte loads and stores,
// fully coalesced: the state is ~86 % of this HBM-bound kernel's bytes.  The per-channel
// scalar work (conv, softplus, SiLU) is repeated by the lanes of a channel -- a few
// instructions -- and the readout C.h is reduced with butterfly shuffles.
//
// Each lane starts its own state's copy into shared memory (cp.async, 16-byte units)
// before the other loads and waits for it just before the recurrence, so the registers
// the state will occupy are free while the loads are in flight; with the launch bound
// of 6 CTAs per SM this measured 42.0 us against 42.6-43.1 us for plain register loads
// (256 x 5120; 8 CTAs per SM spills and takes 48.7 us).  No barrier is needed: every
// lane reads back only what it copied itself.
//
// In-place update (h_out == h_in, conv_state_out == conv_state_in) is safe.  The state:
// every element is read and then written by the same lane, the write after the lane's
// cp.async has completed.  The conv state: both lanes of a channel read cs_in but only
// lane j == 0 writes cs_out; the ordering point is the __shfl_xor_sync of the readout,
// whose operands depend on both lanes' cs_in loads, so neither lane passes it before its
// loads have returned, and lane 0's stores come after it.  An edit that moves those stores
// above the shuffle (or the shuffle above the loads' use) breaks in-place decode.
#pragma once

#include "device_math.cuh"
#include "sm100_primitives.cuh"

namespace mm {

struct StepArgs {
  const void* xp;
  const void* z;
  const void* dt;
  const void* B;
  const void* C;
  const float* A_log;
  const float* D;
  const float* conv_w;
  const float* conv_b;  // may be null
  const float* dt_bias;
  const float* h_in;
  const void* cs_in;
  void* y;
  float* h_out;
  void* cs_out;
  int64_t batch, Di;
};

constexpr int kStepThreads = 256;
#ifndef MM_STEP_LANES
#define MM_STEP_LANES 2
#endif
constexpr int kStepLanes = MM_STEP_LANES;   // lanes per channel

// kS consecutive I/O elements (kS = 8, 4 or 2) as fp32 through vector loads.
template <int kS, typename IO>
__device__ __forceinline__ void ld_small(const IO* p, float* out) {
  if constexpr (sizeof(IO) == 2) {
    if constexpr (kS == 8) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        out[2 * k] = __uint_as_float(wv[k] << 16);
        out[2 * k + 1] = __uint_as_float(wv[k] & 0xffff0000u);
      }
    } else if constexpr (kS == 4) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
      out[0] = __uint_as_float(v.x << 16); out[1] = __uint_as_float(v.x & 0xffff0000u);
      out[2] = __uint_as_float(v.y << 16); out[3] = __uint_as_float(v.y & 0xffff0000u);
    } else {
      const uint32_t v = __ldg(reinterpret_cast<const unsigned int*>(p));
      out[0] = __uint_as_float(v << 16); out[1] = __uint_as_float(v & 0xffff0000u);
    }
  } else {
    if constexpr (kS == 8) {
      const float4 v0 = __ldg(reinterpret_cast<const float4*>(p));
      const float4 v1 = __ldg(reinterpret_cast<const float4*>(p + 4));
      out[0] = v0.x; out[1] = v0.y; out[2] = v0.z; out[3] = v0.w;
      out[4] = v1.x; out[5] = v1.y; out[6] = v1.z; out[7] = v1.w;
    } else if constexpr (kS == 4) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(p));
      out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    } else {
      const float2 v = __ldg(reinterpret_cast<const float2*>(p));
      out[0] = v.x; out[1] = v.y;
    }
  }
}

// kS consecutive fp32 values (kS multiple of 2) through 16- or 8-byte loads.
template <int kS, bool kStream>
__device__ __forceinline__ void ld_f32s(const float* p, float* out) {
#pragma unroll
  for (int i = 0; i < kS; i += 4) {
    if constexpr (kS - 0 >= 4) {
      const float4 v = kStream ? __ldcs(reinterpret_cast<const float4*>(p + i))
                               : __ldg(reinterpret_cast<const float4*>(p + i));
      out[i] = v.x; out[i + 1] = v.y; out[i + 2] = v.z; out[i + 3] = v.w;
    } else {
      const float2 v = kStream ? __ldcs(reinterpret_cast<const float2*>(p + i))
                               : __ldg(reinterpret_cast<const float2*>(p + i));
      out[i] = v.x; out[i + 1] = v.y;
    }
  }
}

template <int N, typename IO, bool kPrecise, int kLanes>
__global__ void __launch_bounds__(kStepThreads, 6)
step_kernel(StepArgs a) {
  using M = Math<kPrecise>;
  constexpr int S = N / kLanes;  // states per lane
  static_assert(kLanes == 2 || kLanes == 4, "2 or 4 lanes per channel");
  // grid: (ceil(kLanes*Di / kStepThreads), batch); no integer division on the device
  const int t = blockIdx.x * kStepThreads + threadIdx.x;
  const int64_t b = blockIdx.y;
  const int64_t d = t / kLanes;            // power of two: a shift
  const int j = t % kLanes;
  // kLanes*Di is a multiple of 16 (Di % 8 == 0) and of 32 for 4 lanes; for 2 lanes the
  // half-warp tails of a partial warp are still whole channels, and the shuffles below
  // only pair lanes of the same channel.
  if (d >= a.Di) return;
  const int64_t ch = b * a.Di + d;         // flat (b, d)

  // --- loads: the state first (the bulk of the bytes; global -> shared), then the rest
  float h[S], A2[S], Bv[S], Cv[S];
  __shared__ __align__(16) float hsm[kStepThreads * S];
  static_assert(S % 4 == 0, "the state moves in 16-byte units");
  {
    const uint32_t dst = smem_addr(&hsm[threadIdx.x * S]);
    const float* src = a.h_in + ch * N + j * S;
#pragma unroll
    for (int i = 0; i < S; i += 4)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + i * 4), "l"(src + i) : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  ld_f32s<S, false>(a.A_log + d * N + j * S, A2);
  ld_small<S>(static_cast<const IO*>(a.B) + b * N + j * S, Bv);
  ld_small<S>(static_cast<const IO*>(a.C) + b * N + j * S, Cv);
  const IO* cs_in = static_cast<const IO*>(a.cs_in) + ch * 3;
  const float s0 = IOT<IO>::to_f(cs_in[0]);
  const float s1 = IOT<IO>::to_f(cs_in[1]);
  const float s2 = IOT<IO>::to_f(cs_in[2]);
  const float xt = IOT<IO>::ld(static_cast<const IO*>(a.xp) + ch);
  const float zt = IOT<IO>::ld(static_cast<const IO*>(a.z) + ch);
  const float dtr = IOT<IO>::ld(static_cast<const IO*>(a.dt) + ch);
  const float4 w = __ldg(reinterpret_cast<const float4*>(a.conv_w + d * 4));
  const float cb = a.conv_b ? __ldg(a.conv_b + d) : 0.0f;
  const float dtb = __ldg(a.dt_bias + d);
  const float Dd = __ldg(a.D + d);

  asm volatile("cp.async.wait_group 0;" ::: "memory");
#pragma unroll
  for (int i = 0; i < S; i += 4) {
    const float4 v = *reinterpret_cast<const float4*>(&hsm[threadIdx.x * S + i]);
    h[i] = v.x; h[i + 1] = v.y; h[i + 2] = v.z; h[i + 3] = v.w;
  }
  // --- conv + SiLU, softplus (same on the lanes of the channel)
  const float pre = cb + w.x * s0 + w.y * s1 + w.z * s2 + w.w * xt;
  const float u = M::silu(pre);
  const float delta = M::softplus(dtr + dtb);
  const float du = delta * u;

  // --- one recurrence step on this lane's states
  float part = 0.0f;
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const float Ak = M::neg_exp(A2[s]) * M::a_scale();
    h[s] = M::decay(delta, Ak) * h[s] + du * Bv[s];
    part += Cv[s] * h[s];
  }
  const unsigned mask = __activemask();
  part += __shfl_xor_sync(mask, part, 1);
  if constexpr (kLanes == 4) part += __shfl_xor_sync(mask, part, 2);

  // --- stores
  float* ho = a.h_out + ch * N + j * S;
#pragma unroll
  for (int i = 0; i < S; i += 4) {
    if constexpr (S >= 4) {
      __stcs(reinterpret_cast<float4*>(ho + i), make_float4(h[i], h[i + 1], h[i + 2], h[i + 3]));
    } else {
      __stcs(reinterpret_cast<float2*>(ho + i), make_float2(h[i], h[i + 1]));
    }
  }
  if (j == 0) {
    const float out = (part + Dd * u) * M::silu(zt);
    static_cast<IO*>(a.y)[ch] = IOT<IO>::from_f(out);
    IO* cso = static_cast<IO*>(a.cs_out) + ch * 3;
    cso[0] = IOT<IO>::from_f(s1);
    cso[1] = IOT<IO>::from_f(s2);
    cso[2] = IOT<IO>::from_f(xt);
  }
}

}  // namespace mm
