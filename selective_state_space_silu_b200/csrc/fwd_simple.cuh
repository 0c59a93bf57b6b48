// First fused forward: one thread per channel (b, d) holding all d_state states in
// registers, sequential in time inside a time chunk.
//
// Long sequences are cut into `nchunks` time chunks so that more threads run at once.
// The carry between chunks uses the scan's pair form: over a chunk c the state map is
//   h_end = P_c * h_start + H_c,   P_c[n] = prod_t exp(Delta_t A_n),  H_c = local end
// state from zero.  Kernel 1 (fwd_chunk_state) computes (P_c, H_c) for chunks
// 0..nchunks-2 into the workspace; kernel 2 (fwd_chunk_main) starts chunk c from
// h_start = fold of (P, H) over chunks 0..c-1 and produces y, h_out and the conv state.
#pragma once

#include "device_math.cuh"

namespace mm {

struct FwdArgs {
  const void* xp;
  const void* z;
  const void* dt;
  const void* B;
  const void* C;
  const float* A_log;
  const float* D;
  const float* conv_w;
  const float* conv_b;   // may be null
  const float* dt_bias;
  void* y;
  float* h_out;          // may be null
  void* cs_out;          // may be null
  float* ws_P;           // [batch, nchunks-1, d_inner, N]
  float* ws_H;           // [batch, nchunks-1, d_inner, N]
  int64_t batch, L, Di;
  int64_t chunk_len;
  int nchunks;
};

constexpr int kSimpleThreads = 128;

// Loads conv weights, bias and the K-1 = 3 inputs that precede t0 (zeros before t = 0).
template <typename IO>
__device__ __forceinline__ void conv_prologue(const FwdArgs& a, int64_t b, int64_t d,
                                              int64_t t0, float w[4], float& cb,
                                              float hist[3]) {
  const IO* xp = static_cast<const IO*>(a.xp);
#pragma unroll
  for (int k = 0; k < 4; ++k) w[k] = __ldg(a.conv_w + d * 4 + k);
  cb = a.conv_b ? __ldg(a.conv_b + d) : 0.0f;
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const int64_t t = t0 - 3 + k;
    hist[k] = t >= 0 ? IOT<IO>::ld(xp + (b * a.L + t) * a.Di + d) : 0.0f;
  }
}

template <int N, typename IO, bool kPrecise>
__global__ void __launch_bounds__(kSimpleThreads)
fwd_chunk_state(FwdArgs a) {
  using M = Math<kPrecise>;
  const int64_t d = int64_t(blockIdx.x) * kSimpleThreads + threadIdx.x;
  const int64_t b = blockIdx.y;
  const int c = blockIdx.z;  // 0 .. nchunks-2
  if (d >= a.Di) return;
  const int64_t t0 = int64_t(c) * a.chunk_len;
  const int64_t t1 = t0 + a.chunk_len;  // never the last chunk, so t1 <= L

  const IO* xp = static_cast<const IO*>(a.xp);
  const IO* dt = static_cast<const IO*>(a.dt);
  const IO* Bm = static_cast<const IO*>(a.B);

  float w[4], cb, hist[3];
  conv_prologue<IO>(a, b, d, t0, w, cb, hist);
  const float dtb = __ldg(a.dt_bias + d);
  float Ak[N], h[N], P[N];
#pragma unroll
  for (int n = 0; n < N; ++n) {
    Ak[n] = M::neg_exp(__ldg(a.A_log + d * N + n)) * M::a_scale();
    h[n] = 0.0f;
    P[n] = 1.0f;
  }
  for (int64_t t = t0; t < t1; ++t) {
    const int64_t row = b * a.L + t;
    const float xt = IOT<IO>::ld(xp + row * a.Di + d);
    const float pre = cb + w[0] * hist[0] + w[1] * hist[1] + w[2] * hist[2] + w[3] * xt;
    hist[0] = hist[1]; hist[1] = hist[2]; hist[2] = xt;
    const float u = M::silu(pre);
    const float delta = M::softplus(IOT<IO>::ld(dt + row * a.Di + d) + dtb);
    const float du = delta * u;
    float Bv[N];
    load_row<N>(Bm + row * N, Bv);
#pragma unroll
    for (int n = 0; n < N; ++n) {
      const float dA = M::decay(delta, Ak[n]);
      h[n] = dA * h[n] + du * Bv[n];
      P[n] *= dA;
    }
  }
  const int64_t o = ((b * (a.nchunks - 1) + c) * a.Di + d) * N;
#pragma unroll
  for (int n = 0; n < N; n += 4) {
    *reinterpret_cast<float4*>(a.ws_P + o + n) = make_float4(P[n], P[n + 1], P[n + 2], P[n + 3]);
    *reinterpret_cast<float4*>(a.ws_H + o + n) = make_float4(h[n], h[n + 1], h[n + 2], h[n + 3]);
  }
}

template <int N, typename IO, bool kPrecise>
__global__ void __launch_bounds__(kSimpleThreads)
fwd_chunk_main(FwdArgs a) {
  using M = Math<kPrecise>;
  const int64_t d = int64_t(blockIdx.x) * kSimpleThreads + threadIdx.x;
  const int64_t b = blockIdx.y;
  const int c = blockIdx.z;
  if (d >= a.Di) return;
  const int64_t t0 = int64_t(c) * a.chunk_len;
  const int64_t t1 = t0 + a.chunk_len < a.L ? t0 + a.chunk_len : a.L;

  const IO* xp = static_cast<const IO*>(a.xp);
  const IO* zz = static_cast<const IO*>(a.z);
  const IO* dt = static_cast<const IO*>(a.dt);
  const IO* Bm = static_cast<const IO*>(a.B);
  const IO* Cm = static_cast<const IO*>(a.C);
  IO* y = static_cast<IO*>(a.y);

  float w[4], cb, hist[3];
  conv_prologue<IO>(a, b, d, t0, w, cb, hist);
  const float dtb = __ldg(a.dt_bias + d);
  const float Dd = __ldg(a.D + d);
  float Ak[N], h[N];
#pragma unroll
  for (int n = 0; n < N; ++n) {
    Ak[n] = M::neg_exp(__ldg(a.A_log + d * N + n)) * M::a_scale();
    h[n] = 0.0f;
  }
  // carried prefix: fold the (P, H) pairs of the chunks before this one
  for (int cc = 0; cc < c; ++cc) {
    const int64_t o = ((b * (a.nchunks - 1) + cc) * a.Di + d) * N;
#pragma unroll
    for (int n = 0; n < N; ++n) h[n] = a.ws_P[o + n] * h[n] + a.ws_H[o + n];
  }

  for (int64_t t = t0; t < t1; ++t) {
    const int64_t row = b * a.L + t;
    const float xt = IOT<IO>::ld(xp + row * a.Di + d);
    const float pre = cb + w[0] * hist[0] + w[1] * hist[1] + w[2] * hist[2] + w[3] * xt;
    hist[0] = hist[1]; hist[1] = hist[2]; hist[2] = xt;
    const float u = M::silu(pre);
    const float delta = M::softplus(IOT<IO>::ld(dt + row * a.Di + d) + dtb);
    const float du = delta * u;
    float Bv[N], Cv[N];
    load_row<N>(Bm + row * N, Bv);
    load_row<N>(Cm + row * N, Cv);
    float acc = 0.0f;
#pragma unroll
    for (int n = 0; n < N; ++n) {
      h[n] = M::decay(delta, Ak[n]) * h[n] + du * Bv[n];
      acc += Cv[n] * h[n];
    }
    acc += Dd * u;
    const float g = acc * M::silu(IOT<IO>::ld(zz + row * a.Di + d));
    y[row * a.Di + d] = IOT<IO>::from_f(g);
  }
  if (c == a.nchunks - 1) {
    if (a.h_out) {
      float* ho = a.h_out + (b * a.Di + d) * N;
#pragma unroll
      for (int n = 0; n < N; n += 4)
        *reinterpret_cast<float4*>(ho + n) = make_float4(h[n], h[n + 1], h[n + 2], h[n + 3]);
    }
    if (a.cs_out) {
      IO* cs = static_cast<IO*>(a.cs_out) + (b * a.Di + d) * 3;
#pragma unroll
      for (int k = 0; k < 3; ++k) cs[k] = IOT<IO>::from_f(hist[k]);
    }
  }
}

}  // namespace mm
