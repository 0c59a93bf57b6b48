// The Mamba2 layer's two neighbours of the scan: the causal depthwise conv + SiLU over the
// concatenated x, B, C channels, and the gated RMSNorm of the scan's output
// (niverel-mamba 0.1.0, section "The weight contract": conv1d over d_inner + 2 ngroups
// d_state channels with 4 taps, norm.weight over d_inner with eps 1e-5).  Both are HBM
// streams of bf16 activations.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "device_math.cuh"

namespace ssd {

// ---------------------------------------------------------------- conv + SiLU
struct ConvArgs {
  const __nv_bfloat16* xbc;   // [Bt, L, Cc], Cc = DI + 2 GN
  const float* w;             // [Cc, 4]
  const float* bias;          // [Cc] or null
  const int32_t* seq_idx;     // [Bt, L] or null
  const __nv_bfloat16* cs_in; // [Bt, Cc, 3] or null (zeros)
  __nv_bfloat16* x;           // [Bt, L, DI]
  __nv_bfloat16* B;           // [Bt, L, GN]
  __nv_bfloat16* C;           // [Bt, L, GN]
  __nv_bfloat16* cs_out;      // [Bt, Cc, 3] or null
  int64_t L;
  int Cc, DI, GN;
};

constexpr int kConvThreads = 128;
constexpr int kConvSteps = 16;  // time steps per thread

__device__ __forceinline__ void bf16x8_to_f32(uint4 v, float* o) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    o[2 * k] = __uint_as_float(w[k] << 16);
    o[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
  }
}

// Grid (ceil(Cc / 8 / kConvThreads), ceil(L / kConvSteps), Bt).  Thread: 8 consecutive
// channels (one 16-byte unit; units never straddle the x / B / C boundaries, all multiples
// of 8) of one row over kConvSteps steps, with the 3 previous inputs in registers.  A tap
// reads zero when an id change lies between its input's step and t: `lr` is the last
// change position seen (INT64_MIN before any), and a tap from step src is live iff
// src >= lr (the state before step 0 counts as the first document's).
template <bool kSeq>
__global__ void __launch_bounds__(kConvThreads) conv_silu_kernel(const ConvArgs a) {
  const int unit = blockIdx.x * kConvThreads + threadIdx.x;
  const int c0 = unit * 8;
  if (c0 >= a.Cc) return;
  const int64_t b = blockIdx.z;
  const int64_t t0 = int64_t(blockIdx.y) * kConvSteps;
  const int64_t t1 = t0 + kConvSteps < a.L ? t0 + kConvSteps : a.L;
  const __nv_bfloat16* xr = a.xbc + b * a.L * a.Cc + c0;
  const int32_t* ids = kSeq ? a.seq_idx + b * a.L : nullptr;

  float w[8][4], bs[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(a.w) + (c0 + i));
    w[i][0] = v.x; w[i][1] = v.y; w[i][2] = v.z; w[i][3] = v.w;
    bs[i] = a.bias ? __ldg(a.bias + c0 + i) : 0.f;
  }
  // the 3 inputs before t0 (p[0] oldest): from the row, or the conv state (zeros when absent)
  float p[3][8];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const int64_t src = t0 - 3 + j;
    if (src >= 0) {
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(xr + src * a.Cc)), p[j]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        p[j][i] = a.cs_in ? __bfloat162float(a.cs_in[(b * a.Cc + c0 + i) * 3 + (3 + src)]) : 0.f;
    }
  }
  int64_t lr = INT64_MIN;
  if constexpr (kSeq) {
    for (int64_t u = t0 - 2 > 1 ? t0 - 2 : 1; u < t0; ++u)
      if (ids[u] != ids[u - 1]) lr = u;
  }
  __nv_bfloat16* dst;
  int64_t dstride;
  int dc;
  if (c0 < a.DI) { dst = a.x; dstride = a.DI; dc = c0; }
  else if (c0 < a.DI + a.GN) { dst = a.B; dstride = a.GN; dc = c0 - a.DI; }
  else { dst = a.C; dstride = a.GN; dc = c0 - a.DI - a.GN; }
  dst += b * a.L * dstride + dc;

  // step t + 1's input is requested before step t's math (one more load in flight per
  // thread; two ahead cost registers and measured slower: 61.8 against 49.6 us)
  uint4 nxt = t0 < t1 ? __ldg(reinterpret_cast<const uint4*>(xr + t0 * a.Cc)) : make_uint4(0, 0, 0, 0);
  for (int64_t t = t0; t < t1; ++t) {
    float cur[8];
    const uint4 raw = nxt;
    if (t + 1 < t1) nxt = __ldg(reinterpret_cast<const uint4*>(xr + (t + 1) * a.Cc));
    bf16x8_to_f32(raw, cur);
    float m0 = 1.f, m1 = 1.f, m2 = 1.f;  // live taps t-3, t-2, t-1
    if constexpr (kSeq) {
      if (t >= 1 && ids[t] != ids[t - 1]) lr = t;
      m0 = t - 3 >= lr ? 1.f : 0.f;
      m1 = t - 2 >= lr ? 1.f : 0.f;
      m2 = t - 1 >= lr ? 1.f : 0.f;
    }
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float v[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = 2 * k + e;
        float pre = bs[i] + w[i][3] * cur[i];
        pre = fmaf(w[i][2] * m2, p[2][i], pre);
        pre = fmaf(w[i][1] * m1, p[1][i], pre);
        pre = fmaf(w[i][0] * m0, p[0][i], pre);
        v[e] = pre * mm::rcp_approx(1.0f + mm::ex2_approx(-pre * mm::kLog2e));  // SiLU
      }
      const __nv_bfloat162 pk = __floats2bfloat162_rn(v[0], v[1]);
      o[k] = *reinterpret_cast<const uint32_t*>(&pk);
    }
    *reinterpret_cast<uint4*>(dst + t * dstride) = make_uint4(o[0], o[1], o[2], o[3]);
#pragma unroll
    for (int i = 0; i < 8; ++i) { p[0][i] = p[1][i]; p[1][i] = p[2][i]; p[2][i] = cur[i]; }
  }

  // the conv state out: the last 3 entries of [state ; row], zero where an id change lies
  // between the entry's step and L - 1 (written by the last tile)
  if (a.cs_out && t1 == a.L) {
    const int64_t L = a.L;
    for (int j = 0; j < 3; ++j) {
      const int64_t src = L - 3 + j;
      bool live = true;
      if constexpr (kSeq) {
        for (int64_t u = src + 1 > 1 ? src + 1 : 1; u < L; ++u)
          if (ids[u] != ids[u - 1]) live = false;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        __nv_bfloat16 v = __float2bfloat16_rn(0.f);
        if (live) {
          if (src >= 0) v = xr[src * a.Cc + i];
          else if (a.cs_in) v = a.cs_in[(b * a.Cc + c0 + i) * 3 + (3 + src)];
        }
        a.cs_out[(b * a.Cc + c0 + i) * 3 + j] = v;
      }
    }
  }
}

// ---------------------------------------------------------------- gated RMSNorm
struct NormArgs {
  const __nv_bfloat16* y;  // [rows, D]
  const __nv_bfloat16* z;  // [rows, D]
  const float* w;          // [D]
  __nv_bfloat16* out;      // [rows, D]
  int64_t rows;
  int D, gs;               // channels per row, channels per group (multiple of 8)
  float eps;
};

constexpr int kNormWarps = 8;
constexpr int kNormCachedUnits = 8;   // 16-byte units per lane kept in registers (gs <= 2048)

// Grid ceil(rows * (D / gs) / kNormWarps) CTAs of kNormWarps warps; one warp per (row,
// group): sum of (y SiLU(z))^2 over the group, then the scaled output.  kCached (groups of
// at most 32 kNormCachedUnits 8-channel units): every load of the group is issued up front
// and y SiLU(z) stays in registers for the output; otherwise the second pass re-reads the
// group's 4 gs bytes from cache.
template <bool kCached>
__global__ void __launch_bounds__(kNormWarps * 32) gated_rmsnorm_kernel(const NormArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t item = int64_t(blockIdx.x) * kNormWarps + (threadIdx.x >> 5);
  const int groups = a.D / a.gs;
  if (item >= a.rows * groups) return;  // whole warps
  const int64_t row = item / groups;
  const int c0 = int(item % groups) * a.gs;
  const __nv_bfloat16* yr = a.y + row * a.D + c0;
  const __nv_bfloat16* zr = a.z + row * a.D + c0;
  const int units = a.gs / 8;
  float ss = 0.f;
  if constexpr (kCached) {
    uint4 yc[kNormCachedUnits], zc[kNormCachedUnits];
#pragma unroll
    for (int i = 0; i < kNormCachedUnits; ++i) {
      const int u = lane + 32 * i;
      if (u < units) {
        yc[i] = __ldg(reinterpret_cast<const uint4*>(yr) + u);
        zc[i] = __ldg(reinterpret_cast<const uint4*>(zr) + u);
      }
    }
    float g[kNormCachedUnits][8];
#pragma unroll
    for (int i = 0; i < kNormCachedUnits; ++i) {
      const int u = lane + 32 * i;
      if (u < units) {
        float yv[8], zv[8];
        bf16x8_to_f32(yc[i], yv);
        bf16x8_to_f32(zc[i], zv);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          g[i][e] = yv[e] * mm::Math<false>::silu(zv[e]);
          ss = fmaf(g[i][e], g[i][e], ss);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = rsqrtf(ss / float(a.gs) + a.eps);
#pragma unroll
    for (int i = 0; i < kNormCachedUnits; ++i) {
      const int u = lane + 32 * i;
      if (u < units) {
        const float4 w0 = __ldg(reinterpret_cast<const float4*>(a.w + c0) + 2 * u);
        const float4 w1 = __ldg(reinterpret_cast<const float4*>(a.w + c0) + 2 * u + 1);
        const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const __nv_bfloat162 pk = __floats2bfloat162_rn(g[i][2 * k] * r * wv[2 * k],
                                                          g[i][2 * k + 1] * r * wv[2 * k + 1]);
          o[k] = *reinterpret_cast<const uint32_t*>(&pk);
        }
        reinterpret_cast<uint4*>(a.out + row * a.D + c0)[u] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  } else {
  for (int u = lane; u < units; u += 32) {
    float yv[8], zv[8];
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(yr) + u), yv);
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(zr) + u), zv);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float g = yv[i] * mm::Math<false>::silu(zv[i]);
      ss = fmaf(g, g, ss);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = rsqrtf(ss / float(a.gs) + a.eps);
  for (int u = lane; u < units; u += 32) {
    float yv[8], zv[8];
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(yr) + u), yv);
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(zr) + u), zv);
    const float4 w0 = __ldg(reinterpret_cast<const float4*>(a.w + c0) + 2 * u);
    const float4 w1 = __ldg(reinterpret_cast<const float4*>(a.w + c0) + 2 * u + 1);
    const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float g0 = yv[2 * k] * mm::Math<false>::silu(zv[2 * k]) * r * wv[2 * k];
      const float g1 = yv[2 * k + 1] * mm::Math<false>::silu(zv[2 * k + 1]) * r * wv[2 * k + 1];
      const __nv_bfloat162 pk = __floats2bfloat162_rn(g0, g1);
      o[k] = *reinterpret_cast<const uint32_t*>(&pk);
    }
    reinterpret_cast<uint4*>(a.out + row * a.D + c0)[u] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  }
}

}  // namespace ssd
