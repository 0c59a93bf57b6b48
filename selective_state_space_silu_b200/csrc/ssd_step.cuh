// Mamba2 single-token decode step on a cached state.
//
// niverel-mamba 0.1.0, section "Autoregressive decoding": step(x_t, state) returns the
// output and a new state, and concatenated steps equal the forward over the sequence.  One
// step of the Mamba2 recurrence (see ssd_kernel.cuh) for every (batch row b, head h,
// channel p):
//
//   Delta = softplus(dt_raw[b,h] + dt_bias[h]),  A = -exp(A_log[h])
//   h[p, n] <- exp(Delta A) h[p, n] + Delta x[b,h,p] B[b,g,n]
//   y[b,h,p] = C[b,g,:] . h[p, :] + D[h] x[b,h,p]     (times SiLU(z[b,h,p]) when z is given)
//
// The state (headdim x d_state fp32 per head) is nearly all of the bytes, so the kernel is
// an HBM stream: each thread owns kStepStates consecutive states of one row (b, h, p) and
// moves them with 16-byte streaming loads and stores; the row's readout C . h is reduced
// with xor shuffles over its d_state / kStepStates lanes.  In-place update (h_out == h_in) is safe: every
// element is read and then written by the same thread.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "device_math.cuh"

namespace ssd {

struct StepArgs {
  const __nv_bfloat16* x;   // [Bt, H, P]
  const __nv_bfloat16* dt;  // [Bt, H]
  const float* A_log;       // [H]
  const __nv_bfloat16* B;   // [Bt, G, N]
  const __nv_bfloat16* C;   // [Bt, G, N]
  const float* D;           // [H]
  const float* dt_bias;     // [H]
  const __nv_bfloat16* z;   // [Bt, H, P] or null
  const float* h_in;        // [Bt, H, P, N]
  __nv_bfloat16* y;         // [Bt, H, P]
  float* h_out;             // [Bt, H, P, N]
  int H, G;
};

constexpr int kStepThreads = 256;
#ifndef MM_SSD_STEP_STATES
#define MM_SSD_STEP_STATES 8
#endif
// consecutive states per thread: 8 (two 16-byte loads of the state in flight per thread)
// measured 69.8 us on 256 sequences x 24 heads x 64 x d_state 128 (0.89 of the measured
// copy bandwidth), against 108.9 us with 4 and 90.6 us with 16
constexpr int kStepStates = MM_SSD_STEP_STATES;

// kS bf16 values as fp32 (kS = 4, 8 or 16), from 8- or 16-byte loads.
template <int kS>
__device__ __forceinline__ void ld_bf16s(const __nv_bfloat16* p, float* out) {
  if constexpr (kS == 4) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    out[0] = __uint_as_float(v.x << 16); out[1] = __uint_as_float(v.x & 0xffff0000u);
    out[2] = __uint_as_float(v.y << 16); out[3] = __uint_as_float(v.y & 0xffff0000u);
  } else {
#pragma unroll
    for (int i = 0; i < kS / 8; ++i) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(p) + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        out[8 * i + 2 * k] = __uint_as_float(w[k] << 16);
        out[8 * i + 2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
      }
    }
  }
}

// Rows (b, h, p) per CTA and CTAs per (b, h): headdim is 64.
template <int N, int kS>
struct StepShape {
  static constexpr int kLpr = N / kS;                    // lanes per row
  static constexpr int kRowsPerCta = kStepThreads / kLpr;
  static constexpr int kCtaPerHead = 64 / kRowsPerCta;
};

// Grid: (H * kCtaPerHead, Bt) CTAs of kStepThreads threads; every index is a shift.
template <int N, int kS, bool kGate>
__global__ void __launch_bounds__(kStepThreads) ssd_step_kernel(const StepArgs a) {
  using Sh = StepShape<N, kS>;
  constexpr int LPR = Sh::kLpr;  // lanes per row: a row never straddles warps
  static_assert(kS % 4 == 0 && LPR >= 4 && LPR <= 32 && 32 % LPR == 0, "states per thread");
  static_assert(64 % Sh::kRowsPerCta == 0, "a CTA's rows must belong to one (b, h)");
  const int h = blockIdx.x / Sh::kCtaPerHead;
  const int64_t b = blockIdx.y;
  const int p = (blockIdx.x % Sh::kCtaPerHead) * Sh::kRowsPerCta + threadIdx.x / LPR;
  const int q = threadIdx.x % LPR;  // this thread's states kS q .. kS q + kS - 1
  const int64_t bh = b * a.H + h;
  const int64_t row = bh * 64 + p;
  const int lane = threadIdx.x & 31;
  // Delta, the decay and the group depend on (b, h) only, shared by the whole CTA: lane 0
  // of each warp computes them and broadcasts them
  float delta = 0.f, dec = 0.f;
  int g = 0;
  if (lane == 0) {
    const float dtr = __bfloat162float(a.dt[bh]);
    const float A2 = -mm::ex2_approx(__ldg(a.A_log + h) * mm::kLog2e) * mm::kLog2e;  // A log2 e
    delta = mm::Math<false>::softplus(dtr + __ldg(a.dt_bias + h));
    dec = mm::ex2_approx(delta * A2);
    g = h / (a.H / a.G);
  }
  delta = __shfl_sync(0xffffffffu, delta, 0);
  dec = __shfl_sync(0xffffffffu, dec, 0);
  g = __shfl_sync(0xffffffffu, g, 0);

  float hv[kS], bv[kS], cv[kS];
  const float4* hin = reinterpret_cast<const float4*>(a.h_in + row * N + kS * q);
#pragma unroll
  for (int i = 0; i < kS / 4; ++i) {
    const float4 v = __ldcs(hin + i);
    hv[4 * i] = v.x; hv[4 * i + 1] = v.y; hv[4 * i + 2] = v.z; hv[4 * i + 3] = v.w;
  }
  ld_bf16s<kS>(a.B + (b * a.G + g) * N + kS * q, bv);
  ld_bf16s<kS>(a.C + (b * a.G + g) * N + kS * q, cv);
  const float xv = __bfloat162float(a.x[row]);
  const float dx = delta * xv;

  float part = 0.f;
#pragma unroll
  for (int i = 0; i < kS; ++i) {
    hv[i] = fmaf(dec, hv[i], dx * bv[i]);
    part = fmaf(cv[i], hv[i], part);
  }
#pragma unroll
  for (int o = 1; o < LPR; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  float4* hout = reinterpret_cast<float4*>(a.h_out + row * N + kS * q);
#pragma unroll
  for (int i = 0; i < kS / 4; ++i)
    __stcs(hout + i, make_float4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]));
  if (q == 0) {
    float out = part + __ldg(a.D + h) * xv;
    if constexpr (kGate) out *= mm::Math<false>::silu(__bfloat162float(a.z[row]));
    a.y[row] = __float2bfloat16_rn(out);
  }
}

}  // namespace ssd
