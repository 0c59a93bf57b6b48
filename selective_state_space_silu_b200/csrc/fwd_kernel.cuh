// Fused forward of the selective-SSM mixer core for sm_100a.
//
// Work decomposition
//   CTA   = one batch row b, a tile of kCh = 32 channels, one time chunk.
//   warp  = 8 channels x 4 lanes.  Lane (chl = lane & 7, j = lane >> 3) owns states
//           n in [j*kS, (j+1)*kS), kS = d_state / 4, of channel chl.  Keeping j uniform
//           within each 8-lane phase makes the B/C shared-memory reads phase broadcasts.
//   quad  = 4 consecutive time steps.  Lane j computes the per-(t, d) scalar work of step
//           t0 + j (conv + SiLU, softplus, SiLU(z)); the step sizes are exchanged with
//           shuffles, every lane advances its states through the 4 steps, and the partial
//           readouts C.h are reduce-scattered so that lane j finishes step t0 + j.
//
// Data movement
//   A producer warp streams 32-step tiles of x' (with a 4-row halo for the causal conv),
//   z, dt_raw, B and C into a ring of shared-memory stages with TMA (3-D tensor maps,
//   no multicast); x'/z/dt tiles use the 64/128-byte swizzle so that the lanes of a warp
//   (4 rows x 8 channels) read without bank conflicts.  Negative or past-the-end time
//   coordinates read zeros, which is the causal left padding at t < 0.  The consumer
//   warps widen each B/C tile to fp32 once (shared by the 32 channels), then run the
//   scan from registers.  y is stored directly (8 channels x 2 bytes per lane phase).
//
// Time chunks (long sequences)
//   A chunk c > 0 starts from the state carried out of chunks 0..c-1.  The chunk-state
//   pass (kPrepass = true) runs the same recurrence over chunks 0..nchunks-2 and writes
//   each chunk's pair (P, H): decay product prod_t exp(Delta_t A) and end state from zero.
//   The main pass folds h = P*h + H over the earlier chunks to get its initial state.
//
// Every mbarrier wait is bounded (see sm100_primitives.cuh); on a timeout the CTA stops
// issuing work, waits (bounded) for the copies it started, records MAMBA_ERR_TIMEOUT in
// the status word and returns.
#pragma once

#include <cuda.h>

#include "device_math.cuh"
#include "sm100_primitives.cuh"

namespace mm {

struct FwdParams {
  const float* A_log;
  const float* D;
  const float* conv_w;
  const float* conv_b;  // may be null
  const float* dt_bias;
  void* y;
  float* h_out;         // may be null
  void* cs_out;         // may be null
  float* ws_P;          // [batch, nchunks-1, d_inner, N]
  float* ws_H;          // [batch, nchunks-1, d_inner, N]
  int* status;          // device status word
  int64_t L, Di;
  int64_t chunk_len;    // multiple of kTileT
  int nchunks;
};

constexpr int kCh = 32;          // channels per CTA
constexpr int kTileT = 32;       // time steps per tile
constexpr int kHalo = 4;         // x' rows loaded before each tile (3 needed)
constexpr int kStages = 3;       // shared-memory ring depth
constexpr int kConsumers = 128;  // 4 warps
constexpr int kFwdThreads = kConsumers + 32;

template <typename IO, int N>
struct FwdSmem {
  static constexpr int kRow = kCh * int(sizeof(IO));            // 64 or 128 bytes
  static constexpr int kXBytes = (kTileT + kHalo) * kRow;
  static constexpr int kZBytes = kTileT * kRow;
  static constexpr int kBBytes = kTileT * N * int(sizeof(IO));
  static constexpr int kBCfBytes = kTileT * 2 * N * 4;
  static constexpr int align1k(int v) { return (v + 1023) / 1024 * 1024; }
  static constexpr int kXOff = 0;
  static constexpr int kZOff = align1k(kXBytes);
  static constexpr int kDtOff = kZOff + align1k(kZBytes);
  static constexpr int kBOff = kDtOff + align1k(kZBytes);
  static constexpr int kCOff = kBOff + align1k(kBBytes);
  static constexpr int kBCfOff = kCOff + align1k(kBBytes);
  static constexpr int kStageBytes = align1k(kBCfOff + kBCfBytes);
  static constexpr int kBarOff = kStages * kStageBytes;
  static constexpr int kTotal = kBarOff + 3 * kStages * 8 + 16;
  static constexpr int kDynamic = kTotal + 1024;  // slack to align the base to 1 KiB
};

// Byte offset of (row, col) in a swizzled tile with kRow-byte rows (64B or 128B swizzle:
// the 16-byte unit index is XORed with address bits 7.. of the row start).
template <int kRow>
__device__ __forceinline__ uint32_t swz(int row, int col_bytes) {
  const uint32_t a = uint32_t(row) * kRow + uint32_t(col_bytes);
  return a ^ (((a >> 7) & uint32_t(kRow / 16 - 1)) << 4);
}

template <typename IO>
__device__ __forceinline__ float lds_io(uint32_t a);
template <>
__device__ __forceinline__ float lds_io<float>(uint32_t a) {
  return lds_f32(a);
}
template <>
__device__ __forceinline__ float lds_io<__nv_bfloat16>(uint32_t a) {
  return __uint_as_float(lds_u16(a) << 16);
}

template <int N, typename IO, bool kPrecise, bool kPrepass>
__global__ void __launch_bounds__(kFwdThreads)
fwd_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_z,
           const __grid_constant__ CUtensorMap tm_dt, const __grid_constant__ CUtensorMap tm_B,
           const __grid_constant__ CUtensorMap tm_C, const FwdParams p) {
  using M = Math<kPrecise>;
  using S = FwdSmem<IO, N>;
  constexpr int kS = N / 4;
  constexpr int kRow = S::kRow;
  constexpr int kEs = int(sizeof(IO));

  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  unsigned char* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sb = smem_addr(smem);                 // 1 KiB-aligned shared address
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOff);   // TMA landed
  uint64_t* ready = full + kStages;                                  // B/C widened
  uint64_t* empty = ready + kStages;                                 // consumers done
  int* prod_abort = reinterpret_cast<int*>(empty + kStages);

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int d0 = blockIdx.x * kCh;
  const int b = blockIdx.y;
  const int c = blockIdx.z;
  const int64_t t_begin = int64_t(c) * p.chunk_len;
  const int64_t t_end = t_begin + p.chunk_len < p.L ? t_begin + p.chunk_len : p.L;
  const int ntiles = int((t_end - t_begin + kTileT - 1) / kTileT);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&ready[s], 1);
      mbar_init(&empty[s], kConsumers / 32);
    }
    *prod_abort = 0;
  }
  __syncthreads();

  constexpr uint32_t kTxBytes =
      uint32_t(S::kXBytes + (kPrepass ? 1 : 2) * S::kZBytes + (kPrepass ? 1 : 2) * S::kBBytes);

  if (tid >= kConsumers) {
    // ------------------------------------------------------------ producer warp
    // The warp walks the tiles together: lane 0 issues the copies, all lanes widen B/C.
    const bool leader = lane == 0;
    int issued = 0;
    auto issue = [&](int k) {
      const int s = k % kStages;
      if (leader) {
        const uint32_t st = sb + uint32_t(s * S::kStageBytes);
        const int tt = int(t_begin) + k * kTileT;
        constexpr uint32_t kSwzAlign = 1024, kPlainAlign = 128;
        mbar_arrive_expect_tx(&full[s], kTxBytes);
        tma_load_3d(st + S::kXOff, &tm_x, &full[s], d0, tt - kHalo, b, kSwzAlign, kEs, p.status);
        tma_load_3d(st + S::kDtOff, &tm_dt, &full[s], d0, tt, b, kSwzAlign, kEs, p.status);
        tma_load_3d(st + S::kBOff, &tm_B, &full[s], 0, tt, b, kPlainAlign, kEs, p.status);
        if constexpr (!kPrepass) {
          tma_load_3d(st + S::kZOff, &tm_z, &full[s], d0, tt, b, kSwzAlign, kEs, p.status);
          tma_load_3d(st + S::kCOff, &tm_C, &full[s], 0, tt, b, kPlainAlign, kEs, p.status);
        }
      }
      __syncwarp();
      issued = k + 1;
    };
    for (int k = 0; k < ntiles && k < kStages; ++k) issue(k);
    bool good = true;
    for (int k = 0; k < ntiles && good; ++k) {
      const int s = k % kStages;
      good = __all_sync(0xffffffffu, mbar_wait(&full[s], uint32_t(k / kStages) & 1u, p.status));
      if (!good) break;
      // widen this tile's B (and C) to fp32, interleaved as [t][j]{B[kS], C[kS]}
      const uint32_t st = sb + uint32_t(s * S::kStageBytes);
      for (int idx = lane; idx < kTileT * N; idx += 32) {
        const int t = idx / N, n = idx - t * N;
        const int jj = n / kS, ss = n - jj * kS;
        const uint32_t dst = st + S::kBCfOff + uint32_t(((t * 4 + jj) * (2 * kS) + ss) * 4);
        sts_f32(dst, lds_io<IO>(st + S::kBOff + idx * kEs));
        if constexpr (!kPrepass) sts_f32(dst + kS * 4, lds_io<IO>(st + S::kCOff + idx * kEs));
      }
      __syncwarp();
      if (leader) mbar_arrive(&ready[s]);
      // refill the stage of tile k-1 once the consumers have released it
      const int kn = k - 1 + kStages;
      if (k >= 1 && kn < ntiles) {
        const int sp = (k - 1) % kStages;
        good = __all_sync(0xffffffffu,
                          mbar_wait(&empty[sp], uint32_t((k - 1) / kStages) & 1u, p.status));
        if (good) issue(kn);
      }
    }
    if (!good) *reinterpret_cast<volatile int*>(prod_abort) = 1;
    named_bar_sync(0, kFwdThreads);
    // drain: every copy this CTA started must land before the CTA exits
    if (leader && *reinterpret_cast<volatile int*>(prod_abort)) {
      for (int k = issued - kStages < 0 ? 0 : issued - kStages; k < issued; ++k)
        mbar_wait(&full[k % kStages], uint32_t(k / kStages) & 1u, nullptr);
    }
    return;
  }

  // -------------------------------------------------------------- consumer warps
  const int warp = tid >> 5;
  const int chl = lane & 7;
  const int j = lane >> 3;
  const int cl = warp * 8 + chl;  // channel within the CTA tile
  // d_inner % 8 == 0, so a warp's 8 channels are all in range or all out of range; an
  // out-of-range warp still walks the tiles (it releases every stage) but reads channel
  // 0's parameters and stores nothing.
  const bool active = d0 + cl < p.Di;
  const int64_t d = active ? d0 + cl : 0;

  const float w0 = __ldg(p.conv_w + d * 4 + 0), w1 = __ldg(p.conv_w + d * 4 + 1);
  const float w2 = __ldg(p.conv_w + d * 4 + 2), w3 = __ldg(p.conv_w + d * 4 + 3);
  const float cb = p.conv_b ? __ldg(p.conv_b + d) : 0.0f;
  const float dtb = __ldg(p.dt_bias + d);
  const float Dd = kPrepass ? 0.0f : __ldg(p.D + d);
  float A2[kS], h[kS], P[kS];
#pragma unroll
  for (int s = 0; s < kS; ++s) {
    A2[s] = M::neg_exp(__ldg(p.A_log + d * N + j * kS + s)) * M::a_scale();
    h[s] = 0.0f;
    P[s] = 1.0f;
  }
  if constexpr (!kPrepass) {
    // carried prefix: fold the (P, H) pairs of chunks 0..c-1
    for (int cc = 0; cc < c; ++cc) {
      const int64_t o = ((int64_t(b) * (p.nchunks - 1) + cc) * p.Di + d) * N + j * kS;
#pragma unroll
      for (int s = 0; s < kS; ++s) h[s] = p.ws_P[o + s] * h[s] + p.ws_H[o + s];
    }
  }

  IO* y = static_cast<IO*>(p.y);
  const int col_bytes = cl * kEs;
  bool ok = true;
  for (int k = 0; k < ntiles; ++k) {
    const int s = k % kStages;
    const uint32_t st = sb + uint32_t(s * S::kStageBytes);
    const int64_t tt = t_begin + int64_t(k) * kTileT;
    ok = __all_sync(0xffffffffu, mbar_wait(&ready[s], uint32_t(k / kStages) & 1u, p.status) &&
                                     mbar_wait(&full[s], uint32_t(k / kStages) & 1u, p.status));
    if (!ok) break;

    const uint32_t X = st + S::kXOff, Z = st + S::kZOff, DT = st + S::kDtOff;
    const uint32_t BCF = st + S::kBCfOff + uint32_t(j * 2 * kS * 4);

    // scalar work of step (4q + j) of this tile
    auto scalar = [&](int q, float& dl, float& dul, float& skip, float& szl) {
      const int r = 4 * q + j;                        // tile row of this lane's step
      const float x0 = lds_io<IO>(X + swz<kRow>(r + 1, col_bytes));
      const float x1 = lds_io<IO>(X + swz<kRow>(r + 2, col_bytes));
      const float x2 = lds_io<IO>(X + swz<kRow>(r + 3, col_bytes));
      const float x3 = lds_io<IO>(X + swz<kRow>(r + 4, col_bytes));
      const float pre = cb + w0 * x0 + w1 * x1 + w2 * x2 + w3 * x3;
      const float u = M::silu(pre);
      dl = M::softplus(lds_io<IO>(DT + swz<kRow>(r, col_bytes)) + dtb);
      dul = dl * u;
      if constexpr (!kPrepass) {
        skip = Dd * u;
        szl = M::silu(lds_io<IO>(Z + swz<kRow>(r, col_bytes)));
      } else {
        skip = 0.0f;
        szl = 0.0f;
      }
    };

    float dl, dul, dsk, sz;
    scalar(0, dl, dul, dsk, sz);
#pragma unroll 1
    for (int q = 0; q < kTileT / 4; ++q) {
      float di[4], dui[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        di[i] = __shfl_sync(0xffffffffu, dl, (i << 3) | chl);
        dui[i] = __shfl_sync(0xffffffffu, dul, (i << 3) | chl);
      }
      const float cur_skip = dsk, cur_sz = sz;
      if (q + 1 < kTileT / 4) scalar(q + 1, dl, dul, dsk, sz);

      // steps past the chunk end (ragged last tile) leave the state untouched
      const int64_t left = t_end - (tt + 4 * q);
      const int nvalid = left >= 4 ? 4 : int(left);
      float yp[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        yp[i] = 0.0f;
        if (i >= nvalid) continue;
        const uint32_t row = BCF + uint32_t((4 * q + i) * 4 * 2 * kS * 4);
        float Bv[kS], Cv[kS];
        if constexpr (kS == 4) {
          const float4 bv = lds_f32x4(row);
          Bv[0] = bv.x; Bv[1] = bv.y; Bv[2] = bv.z; Bv[3] = bv.w;
          if constexpr (!kPrepass) {
            const float4 cv = lds_f32x4(row + 16);
            Cv[0] = cv.x; Cv[1] = cv.y; Cv[2] = cv.z; Cv[3] = cv.w;
          }
        } else {
          const float4 v = lds_f32x4(row);
          Bv[0] = v.x; Bv[1] = v.y; Cv[0] = v.z; Cv[1] = v.w;
        }
        float acc = 0.0f;
#pragma unroll
        for (int s2 = 0; s2 < kS; ++s2) {
          const float a = M::decay(di[i], A2[s2]);
          h[s2] = a * h[s2] + dui[i] * Bv[s2];
          if constexpr (kPrepass) P[s2] *= a;
          else acc += Cv[s2] * h[s2];
        }
        yp[i] = acc;
      }
      if constexpr (!kPrepass) {
        // reduce-scatter over j (lane bits 4 then 3): lane j ends with step j's sum
        const bool hi = (j & 2) != 0;
        float k0 = hi ? yp[2] : yp[0], k1 = hi ? yp[3] : yp[1];
        const float s0 = hi ? yp[0] : yp[2], s1 = hi ? yp[1] : yp[3];
        k0 += __shfl_xor_sync(0xffffffffu, s0, 16);
        k1 += __shfl_xor_sync(0xffffffffu, s1, 16);
        const bool odd = (j & 1) != 0;
        float kp = odd ? k1 : k0;
        const float sp = odd ? k0 : k1;
        kp += __shfl_xor_sync(0xffffffffu, sp, 8);
        if (j < nvalid && active) {
          const float out = (kp + cur_skip) * cur_sz;
          y[(int64_t(b) * p.L + tt + 4 * q + j) * p.Di + d] = IOT<IO>::from_f(out);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  named_bar_sync(0, kFwdThreads);  // pairs with the producer warp's barrier
  if (!ok || !active) return;

  if constexpr (kPrepass) {
    const int64_t o = ((int64_t(b) * (p.nchunks - 1) + c) * p.Di + d) * N + j * kS;
#pragma unroll
    for (int s = 0; s < kS; ++s) {
      p.ws_P[o + s] = P[s];
      p.ws_H[o + s] = h[s];
    }
  } else if (c == p.nchunks - 1) {
    if (p.h_out) {
      float* ho = p.h_out + (int64_t(b) * p.Di + d) * N + j * kS;
      if constexpr (kS == 4) {
        *reinterpret_cast<float4*>(ho) = make_float4(h[0], h[1], h[2], h[3]);
      } else {
        *reinterpret_cast<float2*>(ho) = make_float2(h[0], h[1]);
      }
    }
    if (p.cs_out && j < 3) {
      // last 3 entries of xpad: x'[L-3+j] (zeros for negative t) from the last x tile
      const int kl = ntiles - 1;
      const uint32_t X = sb + uint32_t((kl % kStages) * S::kStageBytes) + S::kXOff;
      const int64_t tt = t_begin + int64_t(kl) * kTileT;
      const int r = int(p.L - 3 + j - (tt - kHalo));
      IO* cs = static_cast<IO*>(p.cs_out) + (int64_t(b) * p.Di + d) * 3;
      cs[j] = IOT<IO>::from_f(lds_io<IO>(X + swz<kRow>(r, col_bytes)));
    }
  }
}

}  // namespace mm
