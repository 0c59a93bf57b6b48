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
// an HBM stream: each thread owns 4 consecutive states of one row (b, h, p) and moves
// them with one 16-byte streaming load and store; the row's readout C . h is reduced with
// xor shuffles over its d_state / 4 lanes.  In-place update (h_out == h_in) is safe: every
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
  int64_t rows;             // Bt * H * P
  int H, G, P;
};

constexpr int kStepThreads = 256;

// Grid: ceil(rows * N / 4 / kStepThreads) CTAs of kStepThreads threads.
template <int N, bool kGate>
__global__ void __launch_bounds__(kStepThreads) ssd_step_kernel(const StepArgs a) {
  constexpr int LPR = N / 4;  // lanes per row (32 or 16): a row never straddles warps
  static_assert(LPR == 32 || LPR == 16, "d_state 128 or 64");
  const int64_t gt = int64_t(blockIdx.x) * kStepThreads + threadIdx.x;
  const int64_t row = gt / LPR;  // (b, h, p) flattened
  const int q = int(gt % LPR);   // this thread's states 4q .. 4q + 3
  if (row >= a.rows) return;     // whole rows drop out together (LPR divides 32)
  const int64_t bh = row / a.P;
  const int h = int(bh % a.H);
  const int64_t b = bh / a.H;
  const int g = h / (a.H / a.G);

  const float4 hv = __ldcs(reinterpret_cast<const float4*>(a.h_in + row * N) + q);
  const uint2 bb = __ldg(reinterpret_cast<const uint2*>(a.B + (b * a.G + g) * N) + q);
  const uint2 cc = __ldg(reinterpret_cast<const uint2*>(a.C + (b * a.G + g) * N) + q);
  const float xv = __bfloat162float(a.x[row]);
  const float dtr = __bfloat162float(a.dt[bh]);
  const float A2 = -mm::ex2_approx(__ldg(a.A_log + h) * mm::kLog2e) * mm::kLog2e;  // A log2 e
  const float delta = mm::Math<false>::softplus(dtr + __ldg(a.dt_bias + h));
  const float dec = mm::ex2_approx(delta * A2);
  const float dx = delta * xv;

  const float b0 = __uint_as_float(bb.x << 16), b1 = __uint_as_float(bb.x & 0xffff0000u);
  const float b2 = __uint_as_float(bb.y << 16), b3 = __uint_as_float(bb.y & 0xffff0000u);
  const float c0 = __uint_as_float(cc.x << 16), c1 = __uint_as_float(cc.x & 0xffff0000u);
  const float c2 = __uint_as_float(cc.y << 16), c3 = __uint_as_float(cc.y & 0xffff0000u);
  float4 ho;
  ho.x = fmaf(dec, hv.x, dx * b0);
  ho.y = fmaf(dec, hv.y, dx * b1);
  ho.z = fmaf(dec, hv.z, dx * b2);
  ho.w = fmaf(dec, hv.w, dx * b3);
  float part = c0 * ho.x + c1 * ho.y + c2 * ho.z + c3 * ho.w;
  // only this row's lanes: with 16 lanes per row the other half-warp may have exited
  const unsigned mask = LPR == 32 ? 0xffffffffu : (0xffffu << (threadIdx.x & 16));
#pragma unroll
  for (int o = 1; o < LPR; o <<= 1) part += __shfl_xor_sync(mask, part, o);
  __stcs(reinterpret_cast<float4*>(a.h_out + row * N) + q, ho);
  if (q == 0) {
    float out = part + __ldg(a.D + h) * xv;
    if constexpr (kGate) out *= mm::Math<false>::silu(__bfloat162float(a.z[row]));
    a.y[row] = __float2bfloat16_rn(out);
  }
}

}  // namespace ssd
