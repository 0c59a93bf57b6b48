// Single-token decode step on a cached (h, conv state) pair.
//
// Four lanes share one channel (b, d); each lane owns N/4 consecutive states, so a warp
// moves 8 channels' fp32 state (8 x 64 B for N = 16) with one 16-byte load per lane:
// fully coalesced, which is what matters for this HBM-bound kernel (the state is ~86%
// of its bytes).  The per-channel scalar work (conv, softplus, SiLU) is repeated by the
// four lanes -- it is a few instructions -- and the readout C.h is reduced with two
// butterfly shuffles.
//
// In-place update (h_out == h_in, conv_state_out == conv_state_in) is safe: every
// element is read and then written by the same warp, with the writes ordered after all
// of the warp's reads by the shuffle reduction they depend on.
#pragma once

#include "device_math.cuh"

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
constexpr int kStepLanes = 4;

template <int N, typename IO, bool kPrecise>
__global__ void __launch_bounds__(kStepThreads)
step_kernel(StepArgs a) {
  using M = Math<kPrecise>;
  constexpr int S = N / kStepLanes;  // states per lane
  const int64_t gt = int64_t(blockIdx.x) * kStepThreads + threadIdx.x;
  const int64_t ch = gt / kStepLanes;      // flat (b, d)
  const int j = int(gt % kStepLanes);
  // batch*Di*4 is a multiple of 32 (Di % 8 == 0): a warp is all in range or all out.
  if (ch >= a.batch * a.Di) return;
  const int64_t b = ch / a.Di;
  const int64_t d = ch - b * a.Di;

  const IO* cs_in = static_cast<const IO*>(a.cs_in);
  // --- loads
  float h[S], Ak[S], Bv[S], Cv[S];
  const float* hp = a.h_in + ch * N + j * S;
  if constexpr (S == 4) {
    const float4 v = *reinterpret_cast<const float4*>(hp);
    h[0] = v.x; h[1] = v.y; h[2] = v.z; h[3] = v.w;
  } else {
    const float2 v = *reinterpret_cast<const float2*>(hp);
    h[0] = v.x; h[1] = v.y;
  }
  const IO* Bm = static_cast<const IO*>(a.B) + b * N + j * S;
  const IO* Cm = static_cast<const IO*>(a.C) + b * N + j * S;
#pragma unroll
  for (int s = 0; s < S; ++s) {
    Ak[s] = M::neg_exp(__ldg(a.A_log + d * N + j * S + s)) * M::a_scale();
    Bv[s] = IOT<IO>::ld(Bm + s);
    Cv[s] = IOT<IO>::ld(Cm + s);
  }
  const float s0 = IOT<IO>::to_f(cs_in[ch * 3 + 0]);
  const float s1 = IOT<IO>::to_f(cs_in[ch * 3 + 1]);
  const float s2 = IOT<IO>::to_f(cs_in[ch * 3 + 2]);
  const float xt = IOT<IO>::ld(static_cast<const IO*>(a.xp) + ch);
  const float zt = IOT<IO>::ld(static_cast<const IO*>(a.z) + ch);
  const float dtr = IOT<IO>::ld(static_cast<const IO*>(a.dt) + ch);

  // --- conv + SiLU, softplus (same on the four lanes)
  const float cb = a.conv_b ? __ldg(a.conv_b + d) : 0.0f;
  const float* w = a.conv_w + d * 4;
  const float pre = cb + __ldg(w) * s0 + __ldg(w + 1) * s1 + __ldg(w + 2) * s2 + __ldg(w + 3) * xt;
  const float u = M::silu(pre);
  const float delta = M::softplus(dtr + __ldg(a.dt_bias + d));
  const float du = delta * u;

  // --- one recurrence step on this lane's states
  float part = 0.0f;
#pragma unroll
  for (int s = 0; s < S; ++s) {
    h[s] = M::decay(delta, Ak[s]) * h[s] + du * Bv[s];
    part += Cv[s] * h[s];
  }
  part += __shfl_xor_sync(0xffffffffu, part, 1);
  part += __shfl_xor_sync(0xffffffffu, part, 2);

  // --- stores
  float* ho = a.h_out + ch * N + j * S;
  if constexpr (S == 4) {
    *reinterpret_cast<float4*>(ho) = make_float4(h[0], h[1], h[2], h[3]);
  } else {
    *reinterpret_cast<float2*>(ho) = make_float2(h[0], h[1]);
  }
  if (j == 0) {
    const float out = (part + __ldg(a.D + d) * u) * M::silu(zt);
    static_cast<IO*>(a.y)[ch] = IOT<IO>::from_f(out);
    IO* cso = static_cast<IO*>(a.cs_out) + ch * 3;
    cso[0] = IOT<IO>::from_f(s1);
    cso[1] = IOT<IO>::from_f(s2);
    cso[2] = IOT<IO>::from_f(xt);
  }
}

}  // namespace mm
