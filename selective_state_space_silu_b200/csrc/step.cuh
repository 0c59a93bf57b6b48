// Single-token decode step on a cached (h, conv state) pair (calm-mamba 0.1.4, introduction:
// O(1) per token with a cached state; niverel-mamba 0.1.0, section "Autoregressive
// decoding": y_t, state_t = step(x_t, state_{t-1})).
//
// The state is ~86 % of the bytes (h in and out: 128 of 148 bytes per (row, channel) at
// d_state 16, bf16 I/O), so the kernel is an HBM stream.  A CTA owns a block of 64 channels
// for a slice of batch rows and walks the rows in order:
//   * per CTA, once: the per-channel parameters -- A = -exp(A_log) (times log2 e), conv
//     weights and bias, D, dt_bias -- into registers, so no (row, channel) repeats them;
//   * per row, by TMA bulk copies (cp.async.bulk, one lane) into a ring of kStepStages: the
//     row's state slab h[b, d0:d0+64, :] (contiguous, 4 KB at d_state 16), its x', z and
//     dt_raw (64 contiguous elements each) and its B and C;
//   * 2 lanes per channel (N/2 states each): conv + SiLU, softplus, the recurrence step,
//     the readout reduced by one shuffle, the gate; the new state goes to a staging buffer
//     in shared memory and leaves by a bulk store (kStepOut staging buffers, so a row's store
//     may still be reading while the next rows compute);
//   * the conv state (3 elements per channel, only 2-byte aligned by contract) moves with
//     plain loads (one row ahead) and stores, by lane 0 of each channel.
// In-place update (h_out == h_in, conv_state_out == conv_state_in) is safe: a row's slab has
// landed in shared memory before the same row's store is issued, rows are disjoint, and each
// channel's conv state is read and then written by its lane 0 alone.
// Every wait is bounded: on a timeout the CTA records MAMBA_ERR_TIMEOUT in the step's status
// word, waits (bounded) for the copies it started, and returns.
#pragma once

#include <cuda_bf16.h>

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
  int* status;          // the step's status word (device)
  int64_t batch, Di;
  int rows_per_cta;
};

constexpr int kStepCh = 64;                   // channels per CTA
constexpr int kStepThreads = 2 * kStepCh;     // 2 lanes per channel
constexpr int kStepStages = 2;                // input ring (2 measured faster than 3, 4 or 6)
constexpr int kStepOut = 3;                   // output staging buffers

template <int N, typename IO>
struct StepSmem {
  static constexpr int kES = int(sizeof(IO));
  static constexpr int kH = kStepCh * N * 4;                 // state slab
  static constexpr int kRow = kStepCh * kES;                 // x', z or dt_raw of the block
  static constexpr int kBC = ((N * kES) + 15) / 16 * 16;     // B or C of the row
  static constexpr int kHOff = 0;
  static constexpr int kXOff = kH;
  static constexpr int kZOff = kXOff + kRow;
  static constexpr int kDtOff = kZOff + kRow;
  static constexpr int kBOff = kDtOff + kRow;
  static constexpr int kCOff = kBOff + kBC;
  static constexpr int kStage = (kCOff + kBC + 127) / 128 * 128;
  static constexpr int kOutOff = kStepStages * kStage;      // [kStepOut] {h slab, y row}
  static constexpr int kOutH = kH;
  static constexpr int kOutY = (kRow + 127) / 128 * 128;
  static constexpr int kOut = kOutH + kOutY;
  static constexpr int kBarOff = kOutOff + kStepOut * kOut;
  static constexpr int kTotal = kBarOff + 8 * kStepStages;
};

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(dst), "l"(src), "r"(bytes), "r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void bulk_s2g(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
               ::"l"(dst), "r"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int kPending>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(kPending) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// kS consecutive I/O elements at a 16-byte (bf16: 8-byte for kS = 4) aligned shared address
template <typename IO, int kS>
__device__ __forceinline__ void lds_io_n(uint32_t a, float* out) {
  if constexpr (sizeof(IO) == 2) {
    if constexpr (kS % 8 == 0) {
#pragma unroll
      for (int i = 0; i < kS; i += 8) {
        uint32_t w[4];
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(a + 2 * i));
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          out[i + 2 * k] = __uint_as_float(w[k] << 16);
          out[i + 2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
        }
      }
    } else {
      static_assert(kS == 4, "4 or a multiple of 8 bf16 values");
      uint32_t w0, w1;
      asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w0), "=r"(w1) : "r"(a));
      out[0] = __uint_as_float(w0 << 16); out[1] = __uint_as_float(w0 & 0xffff0000u);
      out[2] = __uint_as_float(w1 << 16); out[3] = __uint_as_float(w1 & 0xffff0000u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < kS; i += 4) {
      const float4 v = lds_f32x4(a + 4 * i);
      out[i] = v.x; out[i + 1] = v.y; out[i + 2] = v.z; out[i + 3] = v.w;
    }
  }
}
template <typename IO>
__device__ __forceinline__ float lds_io1(uint32_t a) {
  if constexpr (sizeof(IO) == 2) return __uint_as_float(lds_u16(a) << 16);
  else return lds_f32(a);
}

template <int N, typename IO, bool kPrecise>
__global__ void __launch_bounds__(kStepThreads)
step_kernel(const StepArgs a) {
  using M = Math<kPrecise>;
  using S = StepSmem<N, IO>;
  constexpr int kS = N / 2;                  // states per lane
  extern __shared__ __align__(16) unsigned char step_smem[];
  unsigned char* smem = step_smem;
  const uint32_t sb = smem_addr(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOff);

  const int tid = threadIdx.x;
  const int chl = tid >> 1, j = tid & 1;
  const int64_t d0 = int64_t(blockIdx.x) * kStepCh;
  const int nch = a.Di - d0 < kStepCh ? int(a.Di - d0) : kStepCh;   // a multiple of 8
  const bool active = chl < nch;
  const int64_t d = active ? d0 + chl : d0;
  const int64_t b0 = int64_t(blockIdx.y) * a.rows_per_cta;
  const int nrows = int(a.batch - b0 < a.rows_per_cta ? a.batch - b0 : a.rows_per_cta);

  if (tid == 0)
    for (int s = 0; s < kStepStages; ++s) mbar_init(&full[s], 1);
  __syncthreads();

  // the copies of row r into stage r % kStepStages (thread 0)
  const uint32_t hbytes = uint32_t(nch) * N * 4, rbytes = uint32_t(nch) * S::kES;
  const uint32_t bcbytes = uint32_t(N * S::kES);
  auto issue = [&](int r) {
    const int s = r % kStepStages;
    const int64_t b = b0 + r;
    const uint32_t st = sb + uint32_t(s * S::kStage);
    mbar_arrive_expect_tx(&full[s], hbytes + 3 * rbytes + 2 * bcbytes);
    bulk_g2s(st + S::kHOff, a.h_in + (b * a.Di + d0) * N, hbytes, &full[s]);
    bulk_g2s(st + S::kXOff, static_cast<const IO*>(a.xp) + b * a.Di + d0, rbytes, &full[s]);
    bulk_g2s(st + S::kZOff, static_cast<const IO*>(a.z) + b * a.Di + d0, rbytes, &full[s]);
    bulk_g2s(st + S::kDtOff, static_cast<const IO*>(a.dt) + b * a.Di + d0, rbytes, &full[s]);
    bulk_g2s(st + S::kBOff, static_cast<const IO*>(a.B) + b * N, bcbytes, &full[s]);
    bulk_g2s(st + S::kCOff, static_cast<const IO*>(a.C) + b * N, bcbytes, &full[s]);
  };
  int issued = nrows < kStepStages ? nrows : kStepStages;
  if (tid == 0)
    for (int r = 0; r < issued; ++r) issue(r);

  // per-channel parameters, once per CTA
  float A2[kS];
#pragma unroll
  for (int s = 0; s < kS; ++s)
    A2[s] = M::neg_exp(__ldg(a.A_log + d * N + j * kS + s)) * M::a_scale();
  const float4 w = __ldg(reinterpret_cast<const float4*>(a.conv_w + d * 4));
  const float cb = a.conv_b ? __ldg(a.conv_b + d) : 0.0f;
  const float dtb = __ldg(a.dt_bias + d);
  const float Dd = __ldg(a.D + d);

  const IO* cs_in = static_cast<const IO*>(a.cs_in);
  IO* cs_out = static_cast<IO*>(a.cs_out);
  // conv state of the first row, loaded ahead (lane 0 of each channel)
  float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f;
  if (j == 0 && active && nrows > 0) {
    const IO* c = cs_in + (b0 * a.Di + d) * 3;
    s0 = IOT<IO>::to_f(c[0]); s1 = IOT<IO>::to_f(c[1]); s2 = IOT<IO>::to_f(c[2]);
  }

  bool ok = true;
  for (int r = 0; r < nrows; ++r) {
    const int s = r % kStepStages;
    const int64_t b = b0 + r;
    ok = __syncthreads_and(mbar_wait(&full[s], uint32_t(r / kStepStages) & 1u, a.status));
    if (!ok) break;
    const uint32_t st = sb + uint32_t(s * S::kStage);
    // next row's conv state, in flight while this row computes
    float n0 = 0.0f, n1 = 0.0f, n2 = 0.0f;
    if (j == 0 && active && r + 1 < nrows) {
      const IO* c = cs_in + ((b + 1) * a.Di + d) * 3;
      n0 = IOT<IO>::to_f(c[0]); n1 = IOT<IO>::to_f(c[1]); n2 = IOT<IO>::to_f(c[2]);
    }
    float h[kS], Bv[kS], Cv[kS];
    const float4* hs = reinterpret_cast<const float4*>(smem + s * S::kStage + S::kHOff) +
                       (chl * N + j * kS) / 4;
#pragma unroll
    for (int i = 0; i < kS / 4; ++i) {
      const float4 v = hs[i];
      h[4 * i] = v.x; h[4 * i + 1] = v.y; h[4 * i + 2] = v.z; h[4 * i + 3] = v.w;
    }
    lds_io_n<IO, kS>(st + S::kBOff + j * kS * S::kES, Bv);
    lds_io_n<IO, kS>(st + S::kCOff + j * kS * S::kES, Cv);
    const float xt = lds_io1<IO>(st + S::kXOff + chl * S::kES);
    const float zt = lds_io1<IO>(st + S::kZOff + chl * S::kES);
    const float dtr = lds_io1<IO>(st + S::kDtOff + chl * S::kES);
    // the per-channel scalars, on both lanes of the channel (measured faster than computing
    // them on lane 0 and handing them to lane 1 by shuffle: 40.9 against 45.1 us on 256 x 5120)
    const int src = (tid & 31) & ~1;
    const float c0 = __shfl_sync(0xffffffffu, s0, src);
    const float c1 = __shfl_sync(0xffffffffu, s1, src);
    const float c2 = __shfl_sync(0xffffffffu, s2, src);
    const float pre = cb + w.x * c0 + w.y * c1 + w.z * c2 + w.w * xt;
    const float u = kPrecise ? M::silu(pre) : silu_tanh(pre);
    const float delta = kPrecise ? M::softplus(dtr + dtb) : softplus_lg2(dtr + dtb);
    const float du = delta * u;
    float part = 0.0f;
#pragma unroll
    for (int k = 0; k < kS; ++k) {
      h[k] = M::decay(delta, A2[k]) * h[k] + du * Bv[k];
      part += Cv[k] * h[k];
    }
    part += __shfl_xor_sync(0xffffffffu, part, 1);

    // this row's outputs: state slab and y row to staging, conv state straight out
    const int ob = r % kStepOut;
    unsigned char* out = smem + S::kOutOff + ob * S::kOut;
    float4* ho = reinterpret_cast<float4*>(out) + (chl * N + j * kS) / 4;
#pragma unroll
    for (int i = 0; i < kS / 4; ++i)
      ho[i] = make_float4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
    if (j == 0) {
      const float yv = (part + Dd * u) * (kPrecise ? M::silu(zt) : silu_tanh(zt));
      reinterpret_cast<IO*>(out + S::kOutH)[chl] = IOT<IO>::from_f(yv);
      if (active) {
        IO* c = cs_out + (b * a.Di + d) * 3;
        c[0] = IOT<IO>::from_f(c1);
        c[1] = IOT<IO>::from_f(c2);
        c[2] = IOT<IO>::from_f(xt);
      }
    }
    s0 = n0; s1 = n1; s2 = n2;
    // the staging writes become visible to the bulk-copy (async) proxy; the store that last
    // read the buffer the next row writes (row r + 1 - kStepOut) must be done reading it
    fence_proxy_async();
    if (tid == 0) bulk_wait_read<kStepOut - 2>();
    __syncthreads();
    if (tid == 0) {
      bulk_s2g(a.h_out + (b * a.Di + d0) * N, sb + uint32_t(S::kOutOff + ob * S::kOut), hbytes);
      bulk_s2g(static_cast<IO*>(a.y) + b * a.Di + d0,
               sb + uint32_t(S::kOutOff + ob * S::kOut + S::kOutH), rbytes);
      bulk_commit();
      // every thread is done with stage s: refill it with row r + kStepStages
      if (r + kStepStages < nrows) {
        issue(r + kStepStages);
        ++issued;
      }
    }
  }
  if (tid == 0) {
    bulk_wait_all();
    if (!ok) {
      // the copies this CTA started must land before it exits
      for (int r = issued - kStepStages < 0 ? 0 : issued - kStepStages; r < issued; ++r)
        mbar_wait(&full[r % kStepStages], uint32_t(r / kStepStages) & 1u, nullptr);
    }
  }
}

}  // namespace mm
