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
//   forward  -- the recurrence from zero, storing the state at the start of every 32-step
//               tile (workspace, fp32 [batch, tiles, d_inner, d_state]);
//   reverse  -- tiles last to first: reload the tile's start state, recompute its 32
//               states h_t and per-(t, d) scalars into shared memory, then walk the tile
//               backwards with the adjoint state lam (lam += dyc*C; gradients; lam *= a).
// The conv's input gradient needs dpre of the 3 following steps, which the reverse walk has
// just produced: a 3-value window per channel carries it across tiles.  dB and dC are
// summed over the 8 channels of a warp by butterflies, over the 4 warps in shared memory,
// and over CTAs (channel tiles) with global atomics; the per-d gradients are summed over
// batch rows with global atomics.  The gradient outputs must be zero on entry.
#pragma once

#include <float.h>

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
  int64_t L, Di;
  int ntiles;
};

constexpr int kBwdThreads = 128;
constexpr int kBwdCh = 32;
constexpr int kBwdT = 32;

template <int N>
struct BwdSmem {
  static constexpr int kS = N / 4;
  static constexpr int kHs = kBwdT * kBwdThreads * kS * 4;   // h_t per (step, lane)
  static constexpr int kSc = kBwdT * kBwdCh * 16;            // {pre, u, Delta, v} per (step, ch)
  static constexpr int kX = kBwdT * kBwdCh * 4;              // x'_t per (step, ch)
  static constexpr int kAcc = 2 * kBwdT * N * 4;              // dB, dC partial sums per tile
  static constexpr int kTotal = kHs + kSc + kX + kAcc;
};

// kS consecutive I/O elements as fp32 (kS = 4 or 2).
template <int kS, typename IO>
__device__ __forceinline__ void ld_io_row(const IO* p, float* out) {
  if constexpr (sizeof(IO) == 4) {
    if constexpr (kS == 4) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(p));
      out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    } else {
      const float2 v = __ldg(reinterpret_cast<const float2*>(p));
      out[0] = v.x; out[1] = v.y;
    }
  } else {
    if constexpr (kS == 4) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
      out[0] = __uint_as_float(v.x << 16); out[1] = __uint_as_float(v.x & 0xffff0000u);
      out[2] = __uint_as_float(v.y << 16); out[3] = __uint_as_float(v.y & 0xffff0000u);
    } else {
      const uint32_t v = __ldg(reinterpret_cast<const unsigned int*>(p));
      out[0] = __uint_as_float(v << 16); out[1] = __uint_as_float(v & 0xffff0000u);
    }
  }
}

template <bool kPrecise>
__device__ __forceinline__ float sigmoid_(float v) {
  if constexpr (kPrecise) return 1.0f / (1.0f + expf(-v));
  else return rcp_approx(1.0f + ex2_approx(-v * kLog2e));
}

// SiLU'(v) = s (1 + v (1 - s)), s = sigmoid(v)
template <bool kPrecise>
__device__ __forceinline__ float silu_grad(float v) {
  const float s = sigmoid_<kPrecise>(v);
  return s * (1.0f + v * (1.0f - s));
}

template <int N, typename IO, bool kPrecise>
__global__ void __launch_bounds__(kBwdThreads)
bwd_kernel(const BwdParams p) {
  using M = Math<kPrecise>;
  using Sm = BwdSmem<N>;
  constexpr int kS = N / 4;
  extern __shared__ __align__(16) unsigned char smem[];
  float* hs = reinterpret_cast<float*>(smem);
  float4* sc = reinterpret_cast<float4*>(smem + Sm::kHs);
  float* xs = reinterpret_cast<float*>(smem + Sm::kHs + Sm::kSc);
  float* acc = reinterpret_cast<float*>(smem + Sm::kHs + Sm::kSc + Sm::kX);  // [2][T][N]

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int chl = lane & 7;
  const int j = lane >> 3;
  const int cl = warp * 8 + chl;
  const int64_t d0 = int64_t(blockIdx.x) * kBwdCh;
  const int64_t b = blockIdx.y;
  // d_inner % 8 == 0: a warp's 8 channels are all in range or all out; an out-of-range warp
  // takes part in the barriers and shuffles on channel 0's data and stores nothing
  const bool active = d0 + cl < p.Di;
  const int64_t d = active ? d0 + cl : 0;
  const int64_t L = p.L, Di = p.Di;
  const IO* xp = static_cast<const IO*>(p.xp);
  const IO* zz = static_cast<const IO*>(p.z);
  const IO* dt = static_cast<const IO*>(p.dt);
  const IO* dyp = static_cast<const IO*>(p.dy);
  const IO* Bp = static_cast<const IO*>(p.B) + b * L * N + j * kS;
  const IO* Cp = static_cast<const IO*>(p.C) + b * L * N + j * kS;

  float A[kS], A2[kS];
#pragma unroll
  for (int s = 0; s < kS; ++s) {
    const float al = __ldg(p.A_log + d * N + j * kS + s);
    A[s] = fmaxf(-expf(al), -FLT_MAX);              // A = -exp(A_log), for the gradients
    A2[s] = fmaxf(M::neg_exp(al) * M::a_scale(), -FLT_MAX);   // as the forward holds it
  }
  const float w0 = __ldg(p.conv_w + d * 4 + 0), w1 = __ldg(p.conv_w + d * 4 + 1);
  const float w2 = __ldg(p.conv_w + d * 4 + 2), w3 = __ldg(p.conv_w + d * 4 + 3);
  const float cb = p.conv_b ? __ldg(p.conv_b + d) : 0.0f;
  const float dtb = __ldg(p.dt_bias + d);
  const float Dd = __ldg(p.D + d);
  auto X = [&](int64_t t) -> float {   // x'[b, t, d], zero before the sequence
    return t >= 0 ? IOT<IO>::to_f(xp[(b * L + t) * Di + d]) : 0.0f;
  };
  float* ck = p.ws_h + ((b * p.ntiles) * Di + d) * N + j * kS;   // + k * Di * N per tile

  // ---- forward sweep: tile start states
  {
    float h[kS];
#pragma unroll
    for (int s = 0; s < kS; ++s) h[s] = 0.0f;
    float xa = 0.0f, xb = 0.0f, xc = 0.0f;
    for (int k = 0; k < p.ntiles; ++k) {
      if (active) {
#pragma unroll
        for (int s = 0; s < kS; ++s) ck[int64_t(k) * Di * N + s] = h[s];
      }
      const int64_t t0 = int64_t(k) * kBwdT;
      const int64_t t1 = t0 + kBwdT < L ? t0 + kBwdT : L;
      for (int64_t t = t0; t < t1; ++t) {
        const float xt = X(t);
        const float pre = cb + w0 * xa + w1 * xb + w2 * xc + w3 * xt;
        xa = xb; xb = xc; xc = xt;
        const float u = M::silu(pre);
        const float del = M::softplus(IOT<IO>::to_f(dt[(b * L + t) * Di + d]) + dtb);
        float Bv[kS];
        ld_io_row<kS>(Bp + t * N, Bv);
#pragma unroll
        for (int s = 0; s < kS; ++s) h[s] = M::decay(del, A2[s]) * h[s] + del * u * Bv[s];
      }
    }
  }

  // ---- reverse sweep
  float lam[kS], dA[kS];
#pragma unroll
  for (int s = 0; s < kS; ++s) { lam[s] = 0.0f; dA[s] = 0.0f; }
  float dp1 = 0.0f, dp2 = 0.0f, dp3 = 0.0f;          // dpre of steps t+1, t+2, t+3
  float aD = 0.0f, aDtb = 0.0f, aCb = 0.0f, aW0 = 0.0f, aW1 = 0.0f, aW2 = 0.0f, aW3 = 0.0f;
  for (int i = tid; i < 2 * kBwdT * N; i += kBwdThreads) acc[i] = 0.0f;
  __syncthreads();

  for (int k = p.ntiles - 1; k >= 0; --k) {
    const int64_t t0 = int64_t(k) * kBwdT;
    const int cnt = int(t0 + kBwdT < L ? kBwdT : L - t0);
    // recompute the tile: h_t, {pre, u, Delta, v}, x'_t
    float h0[kS], h[kS];
#pragma unroll
    for (int s = 0; s < kS; ++s) h0[s] = h[s] = ck[int64_t(k) * Di * N + s];
    float xa = X(t0 - 3), xb = X(t0 - 2), xc = X(t0 - 1);
    const float xm3 = xa, xm2 = xb, xm1 = xc;        // x' before the tile, for dconv_w
    for (int i = 0; i < cnt; ++i) {
      const int64_t t = t0 + i;
      const float xt = X(t);
      const float pre = cb + w0 * xa + w1 * xb + w2 * xc + w3 * xt;
      xa = xb; xb = xc; xc = xt;
      const float u = M::silu(pre);
      const float v = IOT<IO>::to_f(dt[(b * L + t) * Di + d]) + dtb;
      const float del = M::softplus(v);
      float Bv[kS];
      ld_io_row<kS>(Bp + t * N, Bv);
#pragma unroll
      for (int s = 0; s < kS; ++s) {
        h[s] = M::decay(del, A2[s]) * h[s] + del * u * Bv[s];
        hs[(i * kBwdThreads + tid) * kS + s] = h[s];
      }
      if (j == 0) {
        sc[i * kBwdCh + cl] = make_float4(pre, u, del, v);
        xs[i * kBwdCh + cl] = xt;
      }
    }
    __syncwarp();

    for (int i = cnt - 1; i >= 0; --i) {
      const int64_t t = t0 + i;
      const float4 q = sc[i * kBwdCh + cl];
      const float pre = q.x, u = q.y, del = q.z, v = q.w;
      const int64_t o = (b * L + t) * Di + d;
      const float zt = IOT<IO>::to_f(zz[o]);
      const float dyt = IOT<IO>::to_f(dyp[o]);
      const float sz = sigmoid_<kPrecise>(zt);
      const float dyc = dyt * zt * sz;
      float Bv[kS], Cv[kS], hp[kS], ht[kS];
      ld_io_row<kS>(Bp + t * N, Bv);
      ld_io_row<kS>(Cp + t * N, Cv);
      float ycp = 0.0f, duP = 0.0f, ddP = 0.0f, cB[kS], cC[kS];
#pragma unroll
      for (int s = 0; s < kS; ++s) {
        ht[s] = hs[(i * kBwdThreads + tid) * kS + s];
        hp[s] = i > 0 ? hs[((i - 1) * kBwdThreads + tid) * kS + s] : h0[s];
        ycp += Cv[s] * ht[s];
        const float a = M::decay(del, A2[s]);
        lam[s] += dyc * Cv[s];
        cB[s] = lam[s] * del * u;
        cC[s] = dyc * ht[s];
        duP += lam[s] * del * Bv[s];
        const float ah = lam[s] * hp[s] * a;
        ddP += lam[s] * Bv[s] * u + ah * A[s];
        dA[s] += ah * del;
        lam[s] *= a;
      }
      // channel sums over the 4 lanes of a channel (lane bits 3 and 4)
#pragma unroll
      for (int m = 8; m <= 16; m <<= 1) {
        ycp += __shfl_xor_sync(0xffffffffu, ycp, m);
        duP += __shfl_xor_sync(0xffffffffu, duP, m);
        ddP += __shfl_xor_sync(0xffffffffu, ddP, m);
      }
      // dB, dC summed over the warp's 8 channels (lane bits 0..2)
#pragma unroll
      for (int m = 1; m <= 4; m <<= 1) {
#pragma unroll
        for (int s = 0; s < kS; ++s) {
          cB[s] += __shfl_xor_sync(0xffffffffu, cB[s], m);
          cC[s] += __shfl_xor_sync(0xffffffffu, cC[s], m);
        }
      }
      if (chl == 0 && active) {
#pragma unroll
        for (int s = 0; s < kS; ++s) {
          atomicAdd(&acc[i * N + j * kS + s], cB[s]);
          atomicAdd(&acc[(kBwdT + i) * N + j * kS + s], cC[s]);
        }
      }
      const float yc = ycp + Dd * u;
      const float du = duP + dyc * Dd;
      const float dv = ddP * sigmoid_<kPrecise>(v);
      const float dpre = du * silu_grad<kPrecise>(pre);
      // x' of steps t-3..t for the weight gradient
      const float x0 = xs[i * kBwdCh + cl];
      const float x1 = i >= 1 ? xs[(i - 1) * kBwdCh + cl] : xm1;
      const float x2 = i >= 2 ? xs[(i - 2) * kBwdCh + cl] : (i == 1 ? xm1 : xm2);
      const float x3 = i >= 3 ? xs[(i - 3) * kBwdCh + cl] : (i == 2 ? xm1 : (i == 1 ? xm2 : xm3));
      aW3 += dpre * x0; aW2 += dpre * x1; aW1 += dpre * x2; aW0 += dpre * x3;
      aCb += dpre;
      aDtb += dv;
      aD += dyc * u;
      const float dx = w3 * dpre + w2 * dp1 + w1 * dp2 + w0 * dp3;
      dp3 = dp2; dp2 = dp1; dp1 = dpre;
      if (j == 0 && active) {
        p.dz[o] = dyt * yc * silu_grad<kPrecise>(zt);
        p.ddt[o] = dv;
        p.dxp[o] = dx;
      }
    }
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

  if (!active) return;
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

}  // namespace mm
