// Fused forward of the selective-SSM mixer core for sm_100a.
//
// Work decomposition (warp-specialised CTA)
//   CTA        = one batch row b, a tile of kCh = 32 channels, one time chunk; 4 prep
//                warps and 4 scan warps.
//   prep warps = lane c is channel c.  Prep warp 0 also issues the TMA copies.  For each
//                32-step tile, prep warp w handles steps [8w, 8w+8): it widens B and C
//                to fp32 and computes the per-(t, d) scalars of the operator -- causal
//                conv + SiLU (u), Delta = softplus(dt_raw + dt_bias), Delta*u, D*u and
//                SiLU(z) -- once per (t, d), keeping the conv window in registers.
//   scan warps = 8 channels x 4 lanes.  Lane (chl = lane & 7, j = lane >> 3) owns states
//                n in [j*kS, (j+1)*kS), kS = d_state / 4, of channel chl; j is uniform in
//                each 8-lane phase so the B/C reads are phase broadcasts.  Per group of 4
//                steps ("quad") every lane reads Delta and Delta*u of the 4 steps, advances
//                its states, and the partial readouts C.h are reduce-scattered over the 4
//                lanes of the channel so that lane j finishes step 4q + j (gate, store).
//
// Data movement
//   Raw tiles of x' (with a 4-row halo for the causal conv), z, dt_raw, B and C stream
//   into a 3-deep ring with TMA (3-D tensor maps, no multicast).  Negative or past-the-end
//   time coordinates read zeros (the causal left padding at t < 0).  Prepared tiles (fp32
//   B/C and the scalars) go through a 2-deep ring between prep and scan warps; the scalar
//   records are 64 bytes per (quad, channel) with their 16-byte units XOR-swizzled by
//   channel so that both sides access shared memory without bank conflicts.
//
// Time chunks (long sequences)
//   A chunk c > 0 starts from the state carried out of chunks 0..c-1.  The chunk-state
//   pass (kPrepass = true) runs the same recurrence over chunks 0..nchunks-2 and writes
//   each chunk's pair (P, H): decay product prod_t exp(Delta_t A) and end state from zero.
//   The main pass folds h = P*h + H over the earlier chunks to get its initial state.
//   Steps past the chunk end get Delta = Delta*u = 0, which leaves the state unchanged.
//
// Packed documents and initial state (kExt kernels; niverel-mamba 0.1.0, section "seq_idx
// strict reset")
//   Where seq_idx[b, t] != seq_idx[b, t-1] both states restart from zero at step t: the prep
//   warps drop the conv taps that lie before t, and hand the scan a decay step of +inf
//   (exp(+inf * A) = 0, A clamped strictly negative) while Delta*u is unchanged, so the scan
//   and the chunk pairs need no extra work.  An initial state (h_in, conv_state_in, either
//   optional, any mode) seeds chunk 0's recurrence and conv window and the carry fold.
//
// Every mbarrier wait is bounded (sm100_primitives.cuh): a warp that gives up leaves its
// loop, the CTA meets at a final barrier, waits (bounded) for the copies it started,
// records MAMBA_ERR_TIMEOUT in the status word and returns without writing states.
#pragma once

#include <cuda.h>
#include <float.h>

#include <type_traits>

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
  float* ckpt;          // kCkpt: the state at the start of every 16-step tile,
                        // fp32 [batch, ceil(L/16), d_inner, N] (main pass only)
  int* status;          // device status word
  int64_t L, Di;
  int64_t chunk_len;    // multiple of kTileT
  int nchunks;
  // Failure injection for tests (-1 = off): block (0, 0, 0) arms tile `inject_skip_tile`'s
  // barrier but issues none of its copies, so the waits on it run out.
  int inject_skip_tile;
};

// Extra inputs of the kExt kernels (each may be null).  Only those kernels take them, so the
// plain kernels' parameters stay as they are.
struct FwdExt {
  const int32_t* seq_idx;  // [batch, L] document ids
  const float* h_in;       // [batch, d_inner, N] initial state
  const void* cs_in;       // [batch, d_inner, 3] initial conv window
};
struct FwdParamsExt : FwdParams {
  FwdExt ext;
};
template <bool kExt>
using FwdArgs = typename std::conditional<kExt, FwdParamsExt, FwdParams>::type;

constexpr int kCh = 32;          // channels per CTA
constexpr int kTileT = 32;       // time steps per tile
constexpr int kQuads = kTileT / 4;
constexpr int kHalo = 4;         // x' rows loaded before each tile (3 needed)
constexpr int kStages = 3;       // raw TMA ring depth
constexpr int kPrepBufs = 2;     // prepared-tile ring depth
constexpr int kScanWarps = 4;
constexpr int kPrepWarps = 4;
constexpr int kPrepSteps = kTileT / kPrepWarps;  // steps per prep warp per tile
constexpr int kScanThreads = 32 * kScanWarps;
constexpr int kFwdThreads = 32 * (kScanWarps + kPrepWarps);
constexpr int kScRec = 64;       // bytes per (quad, channel) scalar record

template <typename IO, int N>
struct FwdSmem {
  static constexpr int kRow = kCh * int(sizeof(IO));            // 64 or 128 bytes
  static constexpr int kXBytes = (kTileT + kHalo) * kRow;
  static constexpr int kZBytes = kTileT * kRow;
  static constexpr int kBBytes = kTileT * N * int(sizeof(IO));
  static constexpr int align1k(int v) { return (v + 1023) / 1024 * 1024; }
  // raw stage (TMA destinations)
  static constexpr int kXOff = 0;
  static constexpr int kZOff = align1k(kXBytes);
  static constexpr int kDtOff = kZOff + align1k(kZBytes);
  static constexpr int kBOff = kDtOff + align1k(kZBytes);
  static constexpr int kCOff = kBOff + align1k(kBBytes);
  static constexpr int kRawStage = kCOff + align1k(kBBytes);
  // prepared tile: fp32 B/C records [t][j]{B[kS], C[kS]}, then the scalar records [q][c]
  static constexpr int kBCRec = 2 * (N / 4) * 4;                // fp32: 32 (N=16), 16 (N=8)
  static constexpr int kBCfBytes = kTileT * 4 * kBCRec;
  static constexpr int kScOff = align1k(kBCfBytes);
  static constexpr int kPrepBytes = kScOff + kQuads * kCh * kScRec;
  static constexpr int kPrepBase = kStages * kRawStage;
  static constexpr int kBarOff = kPrepBase + kPrepBufs * kPrepBytes;
  static constexpr int kTotal = kBarOff + 8 * (2 * kStages + 2 * kPrepBufs) + 16;
  static constexpr int kDynamic = kTotal + 1024;  // slack to align the base to 1 KiB
};

// Byte offset of (row, col) in a swizzled tile with kRow-byte rows (64B or 128B swizzle:
// the 16-byte unit index is XORed with address bits 7.. of the row start).
template <int kRow>
__device__ __forceinline__ uint32_t swz(int row, int col_bytes) {
  const uint32_t a = uint32_t(row) * kRow + uint32_t(col_bytes);
  return a ^ (((a >> 7) & uint32_t(kRow / 16 - 1)) << 4);
}

// Offset of 16-byte unit u of the scalar record of (quad q, channel c).
__device__ __forceinline__ uint32_t sc_unit(int q, int c, int u) {
  return uint32_t((q * kCh + c) * kScRec + ((u ^ ((c >> 1) & 3)) << 4));
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

__device__ __forceinline__ void sts_f32x4(uint32_t a, float x, float y, float z, float w);

// The two bf16 halves of a 32-bit word as fp32 (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// B[kS] and C[kS] (I/O type) of one (t, j) into one fp32 record {B[kS], C[kS]} (C left 0
// when b_only).  Widening here, once per CTA, spares the scan lanes of all 32 channels the
// conversion.
template <typename IO, int kS>
__device__ __forceinline__ void widen_record(uint32_t dst, uint32_t b, uint32_t c, bool b_only) {
  static_assert(kS == 2 || kS == 4, "2 or 4 states per lane");
  float v[2 * kS];
  if constexpr (sizeof(IO) == 4) {
    if constexpr (kS == 4) {
      const float4 bv = lds_f32x4(b);
      const float4 cv = b_only ? make_float4(0.f, 0.f, 0.f, 0.f) : lds_f32x4(c);
      v[0] = bv.x; v[1] = bv.y; v[2] = bv.z; v[3] = bv.w;
      v[4] = cv.x; v[5] = cv.y; v[6] = cv.z; v[7] = cv.w;
    } else {
      v[0] = lds_f32(b); v[1] = lds_f32(b + 4);
      v[2] = b_only ? 0.0f : lds_f32(c); v[3] = b_only ? 0.0f : lds_f32(c + 4);
    }
  } else {
    uint32_t w[kS];   // kS/2 words of B, then kS/2 words of C
    if constexpr (kS == 4) {
      asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "r"(b));
      w[2] = w[3] = 0;
      if (!b_only) asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w[2]), "=r"(w[3]) : "r"(c));
    } else {
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w[0]) : "r"(b));
      w[1] = 0;
      if (!b_only) asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w[1]) : "r"(c));
    }
#pragma unroll
    for (int i = 0; i < kS; ++i) {
      v[2 * i] = bf16_lo(w[i]);
      v[2 * i + 1] = bf16_hi(w[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < 2 * kS; i += 4) sts_f32x4(dst + 4 * i, v[i], v[i + 1], v[i + 2], v[i + 3]);
}

__device__ __forceinline__ void sts_f32x4(uint32_t a, float x, float y, float z, float w) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(x), "f"(y), "f"(z),
               "f"(w) : "memory");
}

template <int N, typename IO, bool kPrecise, bool kPrepass, bool kExt, bool kCkpt = false>
__global__ void __launch_bounds__(kFwdThreads)
fwd_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_z,
           const __grid_constant__ CUtensorMap tm_dt, const __grid_constant__ CUtensorMap tm_B,
           const __grid_constant__ CUtensorMap tm_C, const FwdArgs<kExt> p) {
  using M = Math<kPrecise>;
  using S = FwdSmem<IO, N>;
  constexpr int kS = N / 4;
  constexpr int kRow = S::kRow;
  constexpr int kEs = int(sizeof(IO));
  static_assert(kPrecise == (sizeof(IO) == 4), "fp32 I/O takes the precise math, bf16 the fast");

  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  unsigned char* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sb = smem_addr(smem);                 // 1 KiB-aligned shared address
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOff);  // raw tile landed
  uint64_t* raw_free = full + kStages;                              // prep warps done with it
  uint64_t* prep_ready = raw_free + kStages;                        // prepared tile written
  uint64_t* prep_free = prep_ready + kPrepBufs;                     // scan warps done with it

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int d0 = blockIdx.x * kCh;
  const int b = blockIdx.y;
  const int c = blockIdx.z;
  const int64_t t_begin = int64_t(c) * p.chunk_len;
  const int64_t t_end = t_begin + p.chunk_len < p.L ? t_begin + p.chunk_len : p.L;
  const int ntiles = int((t_end - t_begin + kTileT - 1) / kTileT);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&raw_free[s], kPrepWarps);
    }
    for (int r = 0; r < kPrepBufs; ++r) {
      mbar_init(&prep_ready[r], kPrepWarps);
      mbar_init(&prep_free[r], kScanWarps);
    }
  }
  __syncthreads();

  constexpr uint32_t kTxBytes =
      uint32_t(S::kXBytes + (kPrepass ? 1 : 2) * S::kZBytes + (kPrepass ? 1 : 2) * S::kBBytes);

  if (warp >= kScanWarps) {
    // ============================================================ prep warps
    const int w = warp - kScanWarps;  // steps [kPrepSteps*w, kPrepSteps*(w+1)) of each tile
    const bool issuer = (w == 0);
    const int cl = lane;               // channel within the CTA tile
    const bool active = d0 + cl < p.Di;
    const int64_t d = active ? d0 + cl : 0;
    const float w0 = __ldg(p.conv_w + d * 4 + 0), w1 = __ldg(p.conv_w + d * 4 + 1);
    const float w2 = __ldg(p.conv_w + d * 4 + 2), w3 = __ldg(p.conv_w + d * 4 + 3);
    const float cb = p.conv_b ? __ldg(p.conv_b + d) : 0.0f;
    const float dtb = __ldg(p.dt_bias + d);
    const float Dd = kPrepass ? 0.0f : __ldg(p.D + d);
    const int col = cl * kEs;

    int issued = 0;
    auto issue = [&](int k) {
      const int s = k % kStages;
      const bool skip = k == p.inject_skip_tile && blockIdx.x == 0 && blockIdx.y == 0 &&
                        blockIdx.z == 0;
      if (lane == 0) mbar_arrive_expect_tx(&full[s], kTxBytes);
      if (lane == 0 && !skip) {
        const uint32_t st = sb + uint32_t(s * S::kRawStage);
        const int tt = int(t_begin) + k * kTileT;
        constexpr uint32_t kSwzAlign = 1024, kPlainAlign = 128;
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
    if (issuer)
      for (int k = 0; k < ntiles && k < kStages; ++k) issue(k);

    bool good = true;
    for (int k = 0; k < ntiles; ++k) {
      const int s = k % kStages, r = k % kPrepBufs;
      bool got = mbar_wait(&full[s], uint32_t(k / kStages) & 1u, p.status);
      if (k >= kPrepBufs)
        got = got && mbar_wait(&prep_free[r], uint32_t(k / kPrepBufs - 1) & 1u, p.status);
      good = __all_sync(0xffffffffu, got);
      if (!good) break;
      const uint32_t st = sb + uint32_t(s * S::kRawStage);
      const uint32_t pr = sb + uint32_t(S::kPrepBase + r * S::kPrepBytes);
      const int64_t tt = t_begin + int64_t(k) * kTileT;

      // B and C re-laid out for this warp's steps as [t][j]{B[kS], C[kS]} (no conversion):
      // lane (t, j) copies B[t][j*kS ..] and C[t][j*kS ..] into one record
      {
        for (int idx = lane; idx < kPrepSteps * 4; idx += 32) {
          const int t = kPrepSteps * w + idx / 4, jj = idx % 4;
          const uint32_t src = uint32_t(t * N * kEs + jj * kS * kEs);
          const uint32_t dst = pr + uint32_t((t * 4 + jj) * S::kBCRec);
          widen_record<IO, kS>(dst, st + S::kBOff + src, st + S::kCOff + src, kPrepass);
        }
      }

      // scalars of this warp's steps for channel cl; x' tile row r holds t = tt - 4 + r
      const int t0 = kPrepSteps * w;
      float xa = lds_io<IO>(st + S::kXOff + swz<kRow>(t0 + 1, col));
      float xb = lds_io<IO>(st + S::kXOff + swz<kRow>(t0 + 2, col));
      float xc = lds_io<IO>(st + S::kXOff + swz<kRow>(t0 + 3, col));
      [[maybe_unused]] uint32_t resets = 0;   // bit i + 3: reset at step tt + t0 + i (i >= -3)
      if constexpr (kExt) {
        if (p.ext.cs_in && c == 0 && k == 0 && w == 0 && active) {
          // t < 0 of the row: the cached window instead of the zero padding
          const IO* cw = static_cast<const IO*>(p.ext.cs_in) + (int64_t(b) * p.Di + d) * 3;
          xa = IOT<IO>::to_f(cw[0]);
          xb = IOT<IO>::to_f(cw[1]);
          xc = IOT<IO>::to_f(cw[2]);
        }
      }
      // document ids of steps tt + t0 - 3 .. tt + t0 + kPrepSteps - 1: a reset at step T is
      // an id change between T - 1 and T; the row's first step never resets
      if constexpr (kExt) if (p.ext.seq_idx) {
        // lane l reads the id of step T0 - 4 + l (l < kPrepSteps + 4) and compares it with
        // lane l - 1's: one load, one shuffle and one vote per warp and tile
        const int64_t T = tt + t0 - 4 + lane;
        const bool in = T >= 0 && T < p.L && lane < kPrepSteps + 4;
        const int32_t cur = in ? __ldg(p.ext.seq_idx + int64_t(b) * p.L + T) : 0;
        const int32_t prv = __shfl_up_sync(0xffffffffu, cur, 1);
        const bool reset = in && lane >= 1 && T >= 1 && cur != prv;
        resets = __ballot_sync(0xffffffffu, reset) >> 1;   // bit i + 3 <- lane i + 4
      }
      // One tile of per-(t, d) work; kMasked applies the document resets (the plain path
      // is the kMasked = false instance, and a tile without resets takes it too).
      auto prep_steps = [&](auto masked_tag) {
        constexpr bool kMasked = decltype(masked_tag)::value;
#pragma unroll
      for (int qq = 0; qq < kPrepSteps / 4; ++qq) {
        const int q = t0 / 4 + qq;
        float dv[4], duv[4];
        [[maybe_unused]] float skv[4], szv[4];
        // per-(t, d) transcendentals on MUFU (SiLU by tanh.approx, softplus by ex2 + lg2):
        // measured 3.6 % faster on the 130M-class layer and the long sequence than one MUFU
        // op each with the reciprocal and log1p on the FMA pipe
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int t = 4 * q + i;
          const float xt = lds_io<IO>(st + S::kXOff + swz<kRow>(t + 4, col));
          float pre;
          if constexpr (kMasked) {
            // taps before the document's first step are zero
            const int r = 4 * qq + i + 3;   // bit of step t
            const bool m1 = !((resets >> r) & 1u);
            const bool m2 = m1 && !((resets >> (r - 1)) & 1u);
            const bool m3 = m2 && !((resets >> (r - 2)) & 1u);
            pre = cb + w0 * (m3 ? xa : 0.0f) + w1 * (m2 ? xb : 0.0f) + w2 * (m1 ? xc : 0.0f) + w3 * xt;
          } else {
            pre = cb + w0 * xa + w1 * xb + w2 * xc + w3 * xt;
          }
          xa = xb; xb = xc; xc = xt;
          const float u = kPrecise ? M::silu(pre) : silu_tanh(pre);
          const bool valid = tt + t < t_end;
          const float dtv = lds_io<IO>(st + S::kDtOff + swz<kRow>(t, col)) + dtb;
          const float dl = kPrecise ? M::softplus(dtv) : softplus_lg2(dtv);
          dv[i] = valid ? dl : 0.0f;
          duv[i] = valid ? dl * u : 0.0f;
          if constexpr (kMasked)
            if (valid && ((resets >> (4 * qq + i + 3)) & 1u))
              dv[i] = __int_as_float(0x7f800000);   // +inf: this step's decay is 0
          if constexpr (!kPrepass) {
            skv[i] = Dd * u;
            const float zv = lds_io<IO>(st + S::kZOff + swz<kRow>(t, col));
            szv[i] = kPrecise ? M::silu(zv) : silu_tanh(zv);
          }
        }
        const uint32_t rec = pr + S::kScOff;
        sts_f32x4(rec + sc_unit(q, cl, 0), dv[0], dv[1], dv[2], dv[3]);
        sts_f32x4(rec + sc_unit(q, cl, 1), duv[0], duv[1], duv[2], duv[3]);
        if constexpr (!kPrepass) {
          sts_f32x4(rec + sc_unit(q, cl, 2), skv[0], skv[1], skv[2], skv[3]);
          sts_f32x4(rec + sc_unit(q, cl, 3), szv[0], szv[1], szv[2], szv[3]);
        }
      }
      };
      if (kExt && resets != 0)   // warp-uniform
        prep_steps(std::true_type{});
      else
        prep_steps(std::false_type{});
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&prep_ready[r]);
        mbar_arrive(&raw_free[s]);
      }
      // new conv state: last 3 entries of xpad, x'[L-3+i] (the initial window or zeros for
      // negative positions); with documents, slots older than the last document's first
      // step are zero (slot i needs no reset at steps L-2+i .. L-1)
      if (!kPrepass && w == kPrepWarps - 1 && k == ntiles - 1 && c == p.nchunks - 1 && p.cs_out && active) {
        IO* cs = static_cast<IO*>(p.cs_out) + (int64_t(b) * p.Di + d) * 3;
        if constexpr (kExt) {
          bool keep0 = true, keep1 = true;
          if (p.ext.seq_idx) {
            const int32_t* sq = p.ext.seq_idx + int64_t(b) * p.L;
            const bool r1 = p.L - 1 >= 1 && __ldg(sq + p.L - 1) != __ldg(sq + p.L - 2);
            const bool r2 = p.L - 2 >= 1 && __ldg(sq + p.L - 2) != __ldg(sq + p.L - 3);
            keep1 = !r1;
            keep0 = !r1 && !r2;
          }
#pragma unroll
          for (int i = 0; i < 3; ++i) {
            const int64_t pos = p.L - 3 + i;
            float v;
            if (pos < 0 && p.ext.cs_in)
              v = IOT<IO>::to_f(static_cast<const IO*>(p.ext.cs_in)[(int64_t(b) * p.Di + d) * 3 + (p.L + i)]);
            else
              v = lds_io<IO>(st + S::kXOff + swz<kRow>(int(pos - (tt - kHalo)), col));
            if ((i == 0 && !keep0) || (i == 1 && !keep1)) v = 0.0f;
            cs[i] = IOT<IO>::from_f(v);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 3; ++i) {
            const int rr = int(p.L - 3 + i - (tt - kHalo));
            cs[i] = IOT<IO>::from_f(lds_io<IO>(st + S::kXOff + swz<kRow>(rr, col)));
          }
        }
      }
      // refill this raw stage with tile k + kStages once both prep warps are done with it
      if (issuer && k + kStages < ntiles) {
        good = __all_sync(0xffffffffu,
                          mbar_wait(&raw_free[s], uint32_t(k / kStages) & 1u, p.status));
        if (!good) break;
        issue(k + kStages);
      }
    }
    named_bar_sync(0, kFwdThreads);
    // drain: every copy this CTA started must land before the CTA exits
    if (issuer && lane == 0 && !good) {
      for (int k = issued - kStages < 0 ? 0 : issued - kStages; k < issued; ++k)
        mbar_wait(&full[k % kStages], uint32_t(k / kStages) & 1u, nullptr);
    }
    return;
  }

  // ============================================================== scan warps
  const int chl = lane & 7;
  const int j = lane >> 3;
  const int cl = warp * 8 + chl;  // channel within the CTA tile
  // d_inner % 8 == 0: a warp's 8 channels are all in range or all out of range; an
  // out-of-range warp still walks the tiles (it releases every buffer) but stores nothing.
  const bool active = d0 + cl < p.Di;
  const int64_t d = active ? d0 + cl : 0;
  float A2[kS], h[kS], P[kS];
#pragma unroll
  for (int s = 0; s < kS; ++s) {
    // A = -exp(A_log) (held times log2 e on the fast path); clamped finite so that a
    // masked step (Delta = 0) multiplies to exactly 0 and decays by exactly 1.
    A2[s] = fmaxf(M::neg_exp(__ldg(p.A_log + d * N + j * kS + s)) * M::a_scale(), -FLT_MAX);
    // with resets, also strictly negative, so that a reset step (+inf) decays to exactly 0
    if constexpr (kExt) A2[s] = fminf(A2[s], -FLT_MIN);
    h[s] = 0.0f;
    P[s] = 1.0f;
  }
  if constexpr (!kPrepass) {
    // chunk c starts from the initial state carried through chunks 0..c-1
    if constexpr (kExt) if (p.ext.h_in) {
      const float* hi = p.ext.h_in + (int64_t(b) * p.Di + d) * N + j * kS;
#pragma unroll
      for (int s = 0; s < kS; ++s) h[s] = __ldg(hi + s);
    }
    for (int cc = 0; cc < c; ++cc) {
      const int64_t o = ((int64_t(b) * (p.nchunks - 1) + cc) * p.Di + d) * N + j * kS;
#pragma unroll
      for (int s = 0; s < kS; ++s) h[s] = p.ws_P[o + s] * h[s] + p.ws_H[o + s];
    }
  }
  // packed copies for the fast path (pairs of states)
  f32x2 A2p[kS / 2], hp[kS / 2], Pp[kS / 2];
#pragma unroll
  for (int pp = 0; pp < kS / 2; ++pp) {
    A2p[pp] = pk2(A2[2 * pp], A2[2 * pp + 1]);
    hp[pp] = pk2(h[2 * pp], h[2 * pp + 1]);
    Pp[pp] = pk2(1.0f, 1.0f);
  }

  // checkpoints (main pass, when asked): the state entering the 16-step tile that starts at
  // step t < L; chunk 0 writes the row's first, every chunk those that its own steps end
  [[maybe_unused]] auto put_ckpt = [&](int64_t t) {
    if constexpr (kCkpt && !kPrepass) {
      if (active && t < p.L) {
        float v[kS];
        if constexpr (!kPrecise) {
#pragma unroll
          for (int pp = 0; pp < kS / 2; ++pp) upk2(hp[pp], v[2 * pp], v[2 * pp + 1]);
        } else {
#pragma unroll
          for (int s = 0; s < kS; ++s) v[s] = h[s];
        }
        float* o = p.ckpt + ((int64_t(b) * ((p.L + 15) / 16) + t / 16) * p.Di + d) * N + j * kS;
        if constexpr (kS == 4) __stcg(reinterpret_cast<float4*>(o), make_float4(v[0], v[1], v[2], v[3]));
        else __stcg(reinterpret_cast<float2*>(o), make_float2(v[0], v[1]));
      }
    }
  };
  if (c == 0) put_ckpt(0);

  IO* yrow = static_cast<IO*>(p.y) + (int64_t(b) * p.L + t_begin + j) * p.Di + d;
  bool ok = true;
  for (int k = 0; k < ntiles; ++k) {
    const int r = k % kPrepBufs;
    ok = __all_sync(0xffffffffu,
                    mbar_wait(&prep_ready[r], uint32_t(k / kPrepBufs) & 1u, p.status));
    if (!ok) break;
    const uint32_t pr = sb + uint32_t(S::kPrepBase + r * S::kPrepBytes);
    const uint32_t bcf = pr + uint32_t(j * S::kBCRec);
    const uint32_t rec = pr + S::kScOff;
    const int64_t rem = t_end - (t_begin + int64_t(k) * kTileT) - j;  // my step valid if 4q < rem

#pragma unroll 2
    for (int q = 0; q < kQuads; ++q) {
      const float4 dv = lds_f32x4(rec + sc_unit(q, cl, 0));
      const float4 duv = lds_f32x4(rec + sc_unit(q, cl, 1));
      const float di[4] = {dv.x, dv.y, dv.z, dv.w};
      const float dui[4] = {duv.x, duv.y, duv.z, duv.w};
      float yp[4];
      if constexpr (!kPrecise) {
        // fast path: states in packed pairs; per step and pair one f32x2 multiply for
        // Delta*A, two ex2, one f32x2 multiply for Delta*u*B and f32x2 FMAs for h and C.h
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t row = bcf + uint32_t((4 * q + i) * 4 * S::kBCRec);
          const f32x2 d2 = pk2(di[i], di[i]), du2 = pk2(dui[i], dui[i]);
          f32x2 Bp[kS / 2], Cp[kS / 2];
          if constexpr (kS == 4) {   // fp32 record {B0..B3, C0..C3}
            const float4 bv = lds_f32x4(row);
            Bp[0] = pk2(bv.x, bv.y); Bp[1] = pk2(bv.z, bv.w);
            if constexpr (!kPrepass) {
              const float4 cv = lds_f32x4(row + 16);
              Cp[0] = pk2(cv.x, cv.y); Cp[1] = pk2(cv.z, cv.w);
            } else {
              Cp[0] = Cp[1] = pk2(0.0f, 0.0f);
            }
          } else {                   // fp32 record {B0, B1, C0, C1}
            const float4 v = lds_f32x4(row);
            Bp[0] = pk2(v.x, v.y); Cp[0] = pk2(v.z, v.w);
          }
          f32x2 acc2 = pk2(0.0f, 0.0f);
#pragma unroll
          for (int pp = 0; pp < kS / 2; ++pp) {
            float xl, xh;
            upk2(mul2(d2, A2p[pp]), xl, xh);
            const f32x2 a2 = pk2(ex2_approx(xl), ex2_approx(xh));
            hp[pp] = fma2(a2, hp[pp], mul2(du2, Bp[pp]));
            if constexpr (kPrepass) Pp[pp] = mul2(Pp[pp], a2);
            else acc2 = fma2(Cp[pp], hp[pp], acc2);
          }
          float al, ah;
          upk2(acc2, al, ah);
          yp[i] = al + ah;
        }
      } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t row = bcf + uint32_t((4 * q + i) * 4 * S::kBCRec);
        float Bv[kS], Cv[kS];   // fp32 record {B[kS], C[kS]}
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
      }
      if constexpr (!kPrepass) {
        // reduce-scatter over j (lane bits 4 then 3): lane j ends with step 4q+j's sum
        const bool hi = (j & 2) != 0;
        float k0 = hi ? yp[2] : yp[0], k1 = hi ? yp[3] : yp[1];
        const float s0 = hi ? yp[0] : yp[2], s1 = hi ? yp[1] : yp[3];
        k0 += __shfl_xor_sync(0xffffffffu, s0, 16);
        k1 += __shfl_xor_sync(0xffffffffu, s1, 16);
        const bool odd = (j & 1) != 0;
        float kp = odd ? k1 : k0;
        const float sp = odd ? k0 : k1;
        kp += __shfl_xor_sync(0xffffffffu, sp, 8);
        const float skip = lds_f32(rec + sc_unit(q, cl, 2) + 4 * j);
        const float sz = lds_f32(rec + sc_unit(q, cl, 3) + 4 * j);
        if (4 * q < rem && active) yrow[int64_t(4 * q) * p.Di] = IOT<IO>::from_f((kp + skip) * sz);
        if ((q & 3) == 3) put_ckpt(t_begin + int64_t(k) * kTileT + 4 * q + 4);
      }
    }
    yrow += int64_t(kTileT) * p.Di;
    __syncwarp();
    if (lane == 0) mbar_arrive(&prep_free[r]);
  }

  named_bar_sync(0, kFwdThreads);  // pairs with the prep warps' barrier
  if (!ok || !active) return;
  if constexpr (!kPrecise) {
#pragma unroll
    for (int pp = 0; pp < kS / 2; ++pp) {
      upk2(hp[pp], h[2 * pp], h[2 * pp + 1]);
      upk2(Pp[pp], P[2 * pp], P[2 * pp + 1]);
    }
  }

  if constexpr (kPrepass) {
    const int64_t o = ((int64_t(b) * (p.nchunks - 1) + c) * p.Di + d) * N + j * kS;
#pragma unroll
    for (int s = 0; s < kS; ++s) {
      p.ws_P[o + s] = P[s];
      p.ws_H[o + s] = h[s];
    }
  } else if (c == p.nchunks - 1 && p.h_out) {
    float* ho = p.h_out + (int64_t(b) * p.Di + d) * N + j * kS;
    if constexpr (kS == 4) {
      *reinterpret_cast<float4*>(ho) = make_float4(h[0], h[1], h[2], h[3]);
    } else {
      *reinterpret_cast<float2*>(ho) = make_float2(h[0], h[1]);
    }
  }
}

}  // namespace mm
