// Mamba2 selective scan (the SSD layer) forward, main pass on the 5th-generation tensor cores
// (tcgen05): the same chunked evaluation as ssd_kernel.cuh (niverel-mamba 0.1.0, sections
// "The weight contract" and "Measured tolerances"), for rows without document resets.
//
// Per chunk of kQ = 64 steps, with cs the in-chunk cumulative sum of Delta A (log2 units)
// and H [headdim p x d_state n] the state entering the chunk:
//   G  = C B^T                                   (M 64 t, N 64 s, K n)       K-major A and B
//   Y1 = C H^T        (H as bf16 hi + lo planes)  (M 64 t, N 64 p, K n)       K-major A and B
//   Y2 = (M o G) x    (M o G as hi + lo planes)   (M 64 t, N 64 p, K 64 s)    x MN-major
//   U  = (w o x)^T B  (w o x rounded to bf16)     (M 64 p, N n, K 64 s)       both MN-major
//   y_t = 2^cs_t Y1[t] + Y2[t] + D x_t (times SiLU(z_t)),   H <- 2^cs_last H + U
// with M[t, s] = 2^(cs_t - cs_s) Delta_s for s <= t and w_s = 2^(cs_last - cs_s) Delta_s.
// The accumulators live in TMEM (an M = 64 accumulator puts row m in lane
// (m mod 16) + 32 floor(m / 16)); the operand tiles in shared memory use the 128-byte
// swizzle the TMA copies write (64-element rows, 8-row atoms of 1024 bytes).
//
// CTA = one (batch row, head, time segment), 10 warps:
//   warp 9 (copy warp): lane 0 issues the TMA copies of each chunk's C, B and x tiles into a
//     3-deep ring, refilling a stage as soon as the math warps release it;
//   warp 8 (MMA warp): lane 0 issues every tcgen05.mma, committing each group to an mbarrier;
//   warps 0..7 (math warps, warp w reads TMEM lanes 32 (w mod 4) .. + 31, column half w / 4):
//     Delta and cs (warp 3), the mask of G into bf16 hi/lo planes and w o x, the outputs from
//     Y1 and Y2, and the state: H is held in registers (row p = 16 (w mod 4) + lane mod 16,
//     a quarter of the n columns per lane), updated from U and written back as the hi/lo
//     bf16 planes that the next chunk's C H^T reads.  An M = 64 accumulator's rows sit in lanes
//     0..15 of each quarter; the 16x32bx2 load shape hands lanes 16..31 of the warp the
//     second half of the same rows' columns, so all lanes work.
//   Per chunk k the math warps: mask G_k (warp 3 then forms chunk k + 1's cs), write the
//   outputs of chunk k - 1 while (M o G_k) x and U_k run, update the state -- after which
//   the MMA warp can start C H^T of chunk k + 1.  The tensor pipe is the scarce unit (an
//   M = 64, N = 64, K = 16 product takes about 47 clocks, N = 128 about 67), so the MMA warp
//   keeps it fed: G of chunk k + 1 is issued right behind U_k and runs while the math warps
//   update the state, C H^T of chunk k + 1 runs while they mask G_{k+1}, and the copies are
//   left to their own warp.  G, Y1 and Y2 are
//   double-buffered in TMEM, the tiles triple-buffered in shared memory.
// Numerics: bf16 inputs enter exactly; the masked G and the state used by C H^T enter as
// hi + lo bf16 pairs, w o x is rounded once to bf16 (round to nearest); accumulation is fp32
// and the carried state itself stays fp32 in registers.
//
// Every wait is bounded: a warp that gives up records MAMBA_ERR_TIMEOUT in *status and leaves
// its loop; the copy warp waits (bounded) for its copies in flight and the MMA warp for its
// products before the CTA leaves and TMEM is freed.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "device_math.cuh"
#include "sm100_primitives.cuh"
#include "ssd_kernel.cuh"

namespace ssd {
namespace tc {

constexpr int kMathWarps = 8;
constexpr int kMmaWarp = kMathWarps;      // issues every tcgen05.mma, owns TMEM
constexpr int kCopyWarp = kMathWarps + 1; // issues the TMA copies
constexpr int kThreads = 32 * (kMathWarps + 2);
constexpr int kCS = kMathWarps / 4;  // math warps per TMEM lane quarter: each takes 1/kCS of the columns
constexpr int kCW = 64 / kCS;        // columns of a 64-column accumulator per math warp
constexpr int kLW = kCW / 2;         // ... per lane
constexpr int kNS = 3;             // TMA ring depth (chunks in flight)
// The MMA warp (warp 8) shares sub-partition 0 with math warps 0 and 4, and its
// tcgen05.mma issue slows to about half rate when they issue back to back; the math work
// that is not tied to TMEM lane quarter 0 therefore runs on the other sub-partitions: the
// cumulative sums on warp kCsWarp, w o x on the six math warps with warp % 4 != 0.
constexpr int kCsWarp = 3;

// dt_raw of steps 2 lane and 2 lane + 1 of the next kDtAhead chunks, as raw bf16 bits (the
// loads land in their registers without a consumer in between, so nothing waits for them
// until the chunk's cumulative sum is formed kDtAhead chunks later).  Slot = chunk mod
// kDtAhead, chosen by a switch so that the array stays in registers.
constexpr int kDtAhead = 4;
struct DtRing {
  uint32_t v[2 * kDtAhead];
  __device__ __forceinline__ void load(int slot, const __nv_bfloat16* dt, int64_t row0, int64_t L,
                                       int H, int h, int64_t t) {
    const unsigned short* p = reinterpret_cast<const unsigned short*>(dt) + (row0 + t) * H + h;
    switch (slot) {
      case 0: v[0] = 0u; v[1] = 0u; if (t < L) v[0] = __ldg(p); if (t + 1 < L) v[1] = __ldg(p + H); break;
      case 1: v[2] = 0u; v[3] = 0u; if (t < L) v[2] = __ldg(p); if (t + 1 < L) v[3] = __ldg(p + H); break;
      case 2: v[4] = 0u; v[5] = 0u; if (t < L) v[4] = __ldg(p); if (t + 1 < L) v[5] = __ldg(p + H); break;
      default: v[6] = 0u; v[7] = 0u; if (t < L) v[6] = __ldg(p); if (t + 1 < L) v[7] = __ldg(p + H); break;
    }
  }
  __device__ __forceinline__ void take(int slot, float& d0, float& d1) const {
    uint32_t r0, r1;
    switch (slot) {
      case 0: r0 = v[0]; r1 = v[1]; break;
      case 1: r0 = v[2]; r1 = v[3]; break;
      case 2: r0 = v[4]; r1 = v[5]; break;
      default: r0 = v[6]; r1 = v[7]; break;
    }
    d0 = __uint_as_float(r0 << 16);
    d1 = __uint_as_float(r1 << 16);
  }
};
static_assert(kDtAhead == 4, "DtRing has four slots");
constexpr int kPanel = kQ * 128;   // 64 rows of 128 bytes: one swizzled operand panel
// bf16 planes of the masked G and of the state that C H^T reads: two each (hi = bf16(v),
// lo = bf16(v - hi)).  Rounded once, either term carries an error of 2^-9 times the sum of
// its products' magnitudes, which with a carried-in state of order one and d_state 128
// exceeds the output tolerance on rare elements (measured: one plane for the state, 1 element
// in 82k at 1.5x the bound; one plane for the masked G, 1 in 422k at 1.2x).
constexpr int kMGPl = 2;
constexpr int kHPl = 2;

template <int N>
struct Smem {
  static constexpr int NP = N / 64;                // 64-wide panels of d_state
  static constexpr int kC = 0;                     // C [64 t][N n]
  static constexpr int kB = NP * kPanel;           // B [64 s][N n]
  static constexpr int kX = 2 * NP * kPanel;       // x [64 s][64 p]
  static constexpr int kStage = (2 * NP + 1) * kPanel;
  static constexpr int kMG = kNS * kStage;         // masked G [64 t][64 s], bf16 planes
  static constexpr int kXw = kMG + kMGPl * kPanel; // w o x [64 s][64 p]
  static constexpr int kH = kXw + kPanel;          // H [64 p][N n], bf16 planes
  static constexpr int kCs = kH + kHPl * NP * kPanel;   // [3][kQ] cs (log2), chunk k in k % 3
  static constexpr int kDl = kCs + 3 * kQ * 4;     // [3][kQ] Delta
  static constexpr int kBar = kDl + 3 * kQ * 4;
  // full[kNS], empty[kNS], g_done[2], y_done[2], u_done, mg_ready, h_ready
  static constexpr int kNBar = 2 * kNS + 7;
  static constexpr int kTotal = kBar + 8 * kNBar + 16;
  static constexpr int kDynamic = kTotal + 1024;   // slack to align to 1 KiB
  // TMEM: G, Y1 and Y2 (64 columns each, two buffers by chunk parity), U (N columns)
  static constexpr uint32_t kTG = 0, kTY1 = 128, kTY2 = 256, kTU = 384;
  static constexpr uint32_t kTmemCols = 512;
};

// All math warps agree on a flag at named barrier `id` (each of `threads` threads votes).
__device__ __forceinline__ bool bar_and(int id, int threads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "barrier.cta.red.and.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r) : "r"(uint32_t(v)), "r"(id), "r"(threads) : "memory");
  return r != 0;
}

// kW consecutive 32-bit columns of an M = 64 accumulator's row 16 (warp % 4) + lane % 16:
// lanes 0..15 from column col, lanes 16..31 from column col + kW.
template <int kW>
__device__ __forceinline__ void ld_half(uint32_t taddr, float (&v)[kW]) {
  if constexpr (kW == 32) mm::tmem_ld_half32<32>(taddr, v);
  else mm::tmem_ld_half16<16>(taddr, v);
}

// Byte offset of element (row r, column c) of a 64-column swizzled panel.
__device__ __forceinline__ uint32_t pofs(int r, int c) {
  return uint32_t(r * 128 + ((((c >> 3) ^ r) & 7) << 4) + (c & 7) * 2);
}

template <int N, bool kGate>
__global__ void __launch_bounds__(kThreads, 1)
ssd_tc_kernel(const __grid_constant__ CUtensorMap tm_C, const __grid_constant__ CUtensorMap tm_B,
              const __grid_constant__ CUtensorMap tm_x, const SsdArgs a, int* status) {
  using S = Smem<N>;
  constexpr int NP = S::NP;
  constexpr int NH = N / kCS;                      // state columns per math warp
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = mm::smem_addr(smem_raw);
  unsigned char* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sb = mm::smem_addr(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint64_t* full = bars;                // [kNS] a chunk's tiles landed
  uint64_t* empty = bars + kNS;         // [kNS] the math warps are done with a stage
  uint64_t* g_done = bars + 2 * kNS;    // [2] G of chunk k (barrier k & 1) is in TMEM
  uint64_t* y_done = g_done + 2;        // [2] Y1 and Y2 of chunk k (barrier k & 1) are in TMEM
  uint64_t* u_done = y_done + 2;        // U of the chunk is in TMEM
  uint64_t* mg_ready = u_done + 1;      // the masked G and w o x are in shared memory
  uint64_t* h_ready = mg_ready + 1;     // the bf16 planes of the state entering a chunk
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + S::kNBar);
  float* cs_all = reinterpret_cast<float*>(smem + S::kCs);
  float* dl_all = reinterpret_cast<float*>(smem + S::kDl);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x;
  const int64_t b = blockIdx.y;
  const int seg = blockIdx.z;
  const int grp = h / (a.H / a.G);
  const int64_t L = a.L;
  const int64_t nchunks = (L + kQ - 1) / kQ;
  const int64_t c_begin = int64_t(seg) * a.cps;
  const int64_t c_end = c_begin + a.cps < nchunks ? c_begin + a.cps : nchunks;
  const int nck = c_end > c_begin ? int(c_end - c_begin) : 0;
  const int64_t bh = b * a.H + h;

  if (tid == 0) {
    for (int i = 0; i < kNS; ++i) {
      mm::mbar_init(&full[i], 1);
      mm::mbar_init(&empty[i], kMathWarps);
    }
    mm::mbar_init(&g_done[0], 1);
    mm::mbar_init(&g_done[1], 1);
    mm::mbar_init(&y_done[0], 1);
    mm::mbar_init(&y_done[1], 1);
    mm::mbar_init(u_done, 1);
    mm::mbar_init(mg_ready, kMathWarps);
    mm::mbar_init(h_ready, kMathWarps);
  }
  if (warp == kMmaWarp) {
    mm::tmem_alloc(tmem_slot, S::kTmemCols);
    mm::tmem_relinquish();
  }
  mm::tc_fence_before();
  __syncthreads();
  mm::tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == kCopyWarp) {
    // ================================================================== copy warp
    // the stage of chunk k - kNS takes chunk k once the math warps are done with it (they
    // finish a chunk's outputs during the next chunk, after its products completed)
    auto issue = [&](int k) {
      const int s = k % kNS;
      const int t0 = int((c_begin + k) * kQ);
      const uint32_t st = sb + uint32_t(s * S::kStage);
      mm::mbar_arrive_expect_tx(&full[s], uint32_t(S::kStage));
      for (int pn = 0; pn < NP; ++pn) {
        mm::tma_load_4d(st + S::kC + pn * kPanel, &tm_C, &full[s], pn * 64, grp, t0, int(b), 1024,
                        2, status);
        mm::tma_load_4d(st + S::kB + pn * kPanel, &tm_B, &full[s], pn * 64, grp, t0, int(b), 1024,
                        2, status);
      }
      mm::tma_load_4d(st + S::kX, &tm_x, &full[s], 0, h, t0, int(b), 1024, 2, status);
    };
    bool good = true;
    if (lane == 0)
      for (int k = 0; k < nck && k < kNS; ++k) issue(k);
    int issued = nck < kNS ? nck : kNS;
    __syncwarp();
    for (int k = kNS; good && k < nck; ++k) {
      good = __all_sync(0xffffffffu, mm::mbar_wait(&empty[(k - kNS) % kNS],
                                                   uint32_t((k - kNS) / kNS) & 1u, status));
      if (!good) break;
      if (lane == 0) issue(k);
      __syncwarp();
      issued = k + 1;
    }
    mm::named_bar_sync(0, kThreads);
    // nothing may still write the stages when the CTA leaves (after a failure elsewhere the
    // last copies may not have been waited for)
    if (lane == 0)
      for (int k = issued - kNS < 0 ? 0 : issued - kNS; k < issued; ++k)
        mm::mbar_wait(&full[k % kNS], uint32_t(k / kNS) & 1u, nullptr);
    __syncwarp();
    return;
  }

  if (warp == kMmaWarp) {
    // =================================================================== MMA warp
    bool good = true;
    uint64_t* last_bar = nullptr;   // the barrier of the last commit, and its phase
    uint32_t last_par = 0;
    // G of chunk k into its parity buffer (the buffer's previous G, chunk k - 2, was masked
    // before mg_ready of chunk k - 2, which this warp waited for)
    auto issue_g = [&](int k) -> bool {
      const int s = k % kNS;
      const uint32_t st = sb + uint32_t(s * S::kStage);
      if (!__all_sync(0xffffffffu, mm::mbar_wait(&full[s], uint32_t(k / kNS) & 1u, status)))
        return false;
      if (lane == 0) {
        mm::tc_fence_after();
        constexpr uint32_t idG = mm::umma_idesc_bf16_f32_mj<64, 64, 0, 0>();
        const uint32_t dc = mm::umma_desc_lo(st + S::kC, 16), db = mm::umma_desc_lo(st + S::kB, 16);
#pragma unroll
        for (int kk = 0; kk < N / 16; ++kk) {
          const uint32_t o = uint32_t((kk >> 2) * kPanel + (kk & 3) * 32) >> 4;
          mm::umma_bf16_lo(tbase + S::kTG + uint32_t(k & 1) * 64u, dc + o, db + o, idG,
                           kk > 0 ? 1u : 0u);
        }
        mm::umma_commit(&g_done[k & 1]);
        last_bar = &g_done[k & 1];
        last_par = uint32_t(k >> 1) & 1u;
      }
      __syncwarp();
      return true;
    };
    if (nck > 0) good = issue_g(0);
    for (int k = 0; good && k < nck; ++k) {
      const int s = k % kNS;
      const uint32_t st = sb + uint32_t(s * S::kStage);
      const uint32_t ty1 = S::kTY1 + uint32_t(k & 1) * 64u, ty2 = S::kTY2 + uint32_t(k & 1) * 64u;
      // C H^T takes the state entering this chunk, into this chunk's Y1 buffer
      good = __all_sync(0xffffffffu, mm::mbar_wait(h_ready, uint32_t(k) & 1u, status));
      if (!good) break;
      if (lane == 0) {
        mm::tc_fence_after();
        constexpr uint32_t idY = mm::umma_idesc_bf16_f32_mj<64, 64, 0, 0>();
        const uint32_t dc = mm::umma_desc_lo(st + S::kC, 16), dh = mm::umma_desc_lo(sb + S::kH, 16);
#pragma unroll
        for (int pl = 0; pl < kHPl; ++pl)
#pragma unroll
          for (int kk = 0; kk < N / 16; ++kk) {
            const uint32_t o = uint32_t((kk >> 2) * kPanel + (kk & 3) * 32) >> 4;
            mm::umma_bf16_lo(tbase + ty1, dc + o, dh + uint32_t(pl * NP * kPanel >> 4) + o, idY,
                             pl + kk > 0 ? 1u : 0u);
          }
      }
      __syncwarp();
      good = __all_sync(0xffffffffu, mm::mbar_wait(mg_ready, uint32_t(k) & 1u, status));
      if (!good) break;
      if (lane == 0) {
        mm::tc_fence_after();
        constexpr uint32_t idY2 = mm::umma_idesc_bf16_f32_mj<64, 64, 0, 1>();
        const uint32_t dm = mm::umma_desc_lo(sb + S::kMG, 16);
        const uint32_t dx = mm::umma_desc_lo(st + S::kX, kPanel);
#pragma unroll
        for (int pl = 0; pl < kMGPl; ++pl)
#pragma unroll
          for (int kk = 0; kk < kQ / 16; ++kk)
            mm::umma_bf16_lo(tbase + ty2, dm + uint32_t((pl * kPanel + kk * 32) >> 4),
                             dx + uint32_t(kk * 2048 >> 4), idY2, pl + kk > 0 ? 1u : 0u);
        mm::umma_commit(&y_done[k & 1]);
        constexpr uint32_t idU = mm::umma_idesc_bf16_f32_mj<64, N, 1, 1>();
        const uint32_t dw = mm::umma_desc_lo(sb + S::kXw, kPanel);
        const uint32_t dbm = mm::umma_desc_lo(st + S::kB, kPanel);
#pragma unroll
        for (int kk = 0; kk < kQ / 16; ++kk)
          mm::umma_bf16_lo(tbase + S::kTU, dw + uint32_t(kk * 2048 >> 4),
                           dbm + uint32_t(kk * 2048 >> 4), idU, kk > 0 ? 1u : 0u);
        mm::umma_commit(u_done);
        last_bar = u_done;
        last_par = uint32_t(k) & 1u;
      }
      __syncwarp();
      // the next chunk's G runs while the math warps update the state
      if (k + 1 < nck) {
        good = issue_g(k + 1);
        if (!good) break;
      }
    }
    mm::named_bar_sync(0, kThreads);
    // nothing may still write TMEM when it is freed
    if (lane == 0 && last_bar) mm::mbar_wait(last_bar, last_par, nullptr);
    __syncwarp();
    mm::tc_fence_after();
    mm::tmem_dealloc(tbase, S::kTmemCols);
    return;
  }

  // ================================================================== math warps
  const int q = warp & 3, hf = warp >> 2;          // TMEM lane quarter, column block
  // An M = 64 accumulator holds row m in TMEM lane (m mod 16) + 32 (m / 16): lanes 0..15
  // of the warp load the first half of their rows' columns, lanes 16..31 the second half.
  const int part = lane >> 4;                      // 0: first half of the columns, 1: second
  const int r = 16 * q + (lane & 15);              // accumulator row of this lane (t, or p)
  const uint32_t tq = tbase + (uint32_t(32 * q) << 16);
  const float A2 = -expf(a.A_log[h]) * mm::kLog2e;
  const float bias = a.dt_bias[h];
  const float Dh = a.D[h];
  const bool has_h_in = a.h_in != nullptr;
  constexpr int NH2 = NH / 2;                      // state columns per lane
  const int ncol0 = hf * NH + part * NH2;          // this lane's first state column

  // the state entering the segment: row p = r, columns [ncol0, ncol0 + NH2)
  float H[NH2];
#pragma unroll
  for (int i = 0; i < NH2; ++i) H[i] = 0.0f;
  {
    const int64_t col0 = int64_t(r) * N + ncol0;
    if (has_h_in) {
      const float* hi = a.nseg > 1 ? a.ws_H + (bh * a.nseg + a.nseg - 1) * int64_t(kP * N)
                                   : a.h_in + bh * int64_t(kP * N);
#pragma unroll
      for (int i = 0; i < NH2; i += 4) {
        const float4 v = *reinterpret_cast<const float4*>(hi + col0 + i);
        H[i] = v.x; H[i + 1] = v.y; H[i + 2] = v.z; H[i + 3] = v.w;
      }
    }
    for (int sp = 0; sp < seg; ++sp) {
      const float f = mm::ex2_approx(a.ws_A[bh * (a.nseg - 1) + sp]);
      const float* hs = a.ws_H + (bh * a.nseg + sp) * int64_t(kP * N);
#pragma unroll
      for (int i = 0; i < NH2; i += 4) {
        const float4 v = *reinterpret_cast<const float4*>(hs + col0 + i);
        H[i] = fmaf(f, H[i], v.x); H[i + 1] = fmaf(f, H[i + 1], v.y);
        H[i + 2] = fmaf(f, H[i + 2], v.z); H[i + 3] = fmaf(f, H[i + 3], v.w);
      }
    }
  }
  // the state's bf16 planes (B operand of C H^T): row p = r, this lane's columns
  auto put_state = [&]() {
#pragma unroll
    for (int i = 0; i < NH2; i += 8) {
      const int n = ncol0 + i;
      const uint32_t off = uint32_t((n >> 6) * kPanel) + pofs(r, n & 63);
      if constexpr (kHPl == 2) {
        uint4 vh, vl;
        split_bf16(H[i], H[i + 1], vh.x, vl.x);
        split_bf16(H[i + 2], H[i + 3], vh.y, vl.y);
        split_bf16(H[i + 4], H[i + 5], vh.z, vl.z);
        split_bf16(H[i + 6], H[i + 7], vh.w, vl.w);
        sts_u128(sb + S::kH + off, vh);
        sts_u128(sb + S::kH + uint32_t(NP * kPanel) + off, vl);
      } else {
        sts_u128(sb + S::kH + off,
                 make_uint4(pack_bf16(H[i], H[i + 1]), pack_bf16(H[i + 2], H[i + 3]),
                            pack_bf16(H[i + 4], H[i + 5]), pack_bf16(H[i + 6], H[i + 7])));
      }
    }
    mm::fence_async_shared();
    mm::tc_fence_before();
    __syncwarp();
    if (lane == 0) mm::mbar_arrive(h_ready);
  };
  put_state();

  // warp kCsWarp: dt_raw of steps 2 lane, 2 lane + 1 of a chunk (loaded kDtAhead chunks
  // ahead), then Delta and the inclusive cumulative sum of Delta A (log2 units) over it into
  // the chunk's buffer (k mod 3)
  DtRing dtr;
  auto load_dt = [&](int k) {   // chunk k of the segment into slot k mod kDtAhead
    dtr.load(k % kDtAhead, a.dt, b * L, L, a.H, h, (c_begin + k) * kQ + 2 * lane);
  };
  auto chunk_cs = [&](int k) {   // warp kCsWarp; dt of chunk k loaded
    float* cs = cs_all + (k % 3) * kQ;
    float* dl = dl_all + (k % 3) * kQ;
    const int64_t t = (c_begin + k) * kQ + 2 * lane;
    float r0, r1;
    dtr.take(k % kDtAhead, r0, r1);
    const float d0 = t < L ? mm::Math<false>::softplus(r0 + bias) : 0.f;
    const float d1 = t + 1 < L ? mm::Math<false>::softplus(r1 + bias) : 0.f;
    if (k + kDtAhead < nck) load_dt(k + kDtAhead);
    const float e0 = d0 * A2, e1 = d1 * A2;
    float sum = e0 + e1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float v = __shfl_up_sync(0xffffffffu, sum, o);
      if (lane >= o) sum += v;
    }
    float ex = __shfl_up_sync(0xffffffffu, sum, 1);
    if (lane == 0) ex = 0.f;
    cs[2 * lane] = ex + e0;
    cs[2 * lane + 1] = ex + e0 + e1;
    dl[2 * lane] = d0;
    dl[2 * lane + 1] = d1;
  };
  if (warp == kCsWarp && nck > 0) {
    for (int k = 0; k < kDtAhead && k < nck; ++k) load_dt(k);
    chunk_cs(0);
  }

  // the outputs of chunk k: y_t = 2^cs_t Y1[t] + Y2[t] + D x_t (times SiLU(z_t)), t = r, p in
  // the half; then the chunk's stage is free
  auto epilogue = [&](int k) -> bool {
    if (!__all_sync(0xffffffffu, mm::mbar_wait(&y_done[k & 1], uint32_t(k >> 1) & 1u, status)))
      return false;
    mm::tc_fence_after();
    const uint32_t ty1 = S::kTY1 + uint32_t(k & 1) * 64u, ty2 = S::kTY2 + uint32_t(k & 1) * 64u;
    const uint32_t st = sb + uint32_t((k % kNS) * S::kStage);
    const float* cs = cs_all + (k % 3) * kQ;
    float y1[kLW], y2[kLW];
    ld_half(tq + ty1 + uint32_t(kCW * hf), y1);
    ld_half(tq + ty2 + uint32_t(kCW * hf), y2);
    mm::tmem_wait_ld();
    const int64_t t = (c_begin + k) * kQ + r;
    if (t < L) {
      const float et = mm::ex2_approx(cs[r]);
      const int p0 = kCW * hf + kLW * part;
      const int64_t row = ((b * L + t) * a.H + h) * kP + p0;
#pragma unroll
      for (int j = 0; j < kLW / 8; ++j) {
        const uint4 xv = lds_u128(st + S::kX + pofs(r, p0 + 8 * j));
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
        uint4 zv = make_uint4(0, 0, 0, 0);
        if constexpr (kGate) zv = *reinterpret_cast<const uint4*>(a.z + row + 8 * j);
        const uint32_t zw[4] = {zv.x, zv.y, zv.z, zv.w};
        uint32_t ow[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = 8 * j + 2 * e;
          float o0 = fmaf(et, y1[c], y2[c]) + Dh * bf16_lo(xw[e]);
          float o1 = fmaf(et, y1[c + 1], y2[c + 1]) + Dh * bf16_hi(xw[e]);
          if constexpr (kGate) {
            o0 *= mm::Math<false>::silu(bf16_lo(zw[e]));
            o1 *= mm::Math<false>::silu(bf16_hi(zw[e]));
          }
          ow[e] = pack_bf16(o0, o1);
        }
        *reinterpret_cast<uint4*>(a.y + row + 8 * j) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
      }
    }
    mm::tc_fence_before();
    __syncwarp();
    if (lane == 0) mm::mbar_arrive(&empty[k % kNS]);
    return true;
  };

  // Every math warp passes the same named barrier once per chunk, where all agree whether to
  // go on: a wait that gave up in one warp stops them all at the next chunk, never at an
  // unbounded barrier.  Per chunk k: the mask (then warp 0 forms chunk k + 1's cs), the
  // outputs of chunk k - 1 (while this chunk's products run), then the state update, after
  // which the next chunk's C H^T can start.
  bool ok = true;
  for (int k = 0; k < nck; ++k) {
    const int s = k % kNS;
    const uint32_t st = sb + uint32_t(s * S::kStage);
    const float* cs = cs_all + (k % 3) * kQ;
    const float* dl = dl_all + (k % 3) * kQ;
    ok = bar_and(1, 32 * kMathWarps, ok);      // this chunk's cs and Delta visible
    if (!ok) break;
    const float csl = cs[kQ - 1];

    // ---- the mask of G: M[t, s] = G[t, s] 2^(cs_t - cs_s) Delta_s for s <= t, as hi/lo planes
    ok = __all_sync(0xffffffffu, mm::mbar_wait(&full[s], uint32_t(k / kNS) & 1u, status)) &&
         __all_sync(0xffffffffu, mm::mbar_wait(&g_done[k & 1], uint32_t(k >> 1) & 1u, status));
    if (!ok) continue;
    mm::tc_fence_after();
    {
      float g[kLW];
      ld_half(tq + S::kTG + uint32_t(k & 1) * 64u + uint32_t(kCW * hf), g);
      mm::tmem_wait_ld();
      const int c0 = kCW * hf + kLW * part;        // this lane's kLW columns s
      float csv[kLW], dlv[kLW];
#pragma unroll
      for (int i = 0; i < kLW; i += 4) {
        const float4 cv = *reinterpret_cast<const float4*>(cs + c0 + i);
        const float4 dv = *reinterpret_cast<const float4*>(dl + c0 + i);
        csv[i] = cv.x; csv[i + 1] = cv.y; csv[i + 2] = cv.z; csv[i + 3] = cv.w;
        dlv[i] = dv.x; dlv[i + 1] = dv.y; dlv[i + 2] = dv.z; dlv[i + 3] = dv.w;
      }
      const float ct = cs[r];
#pragma unroll
      for (int j = 0; j < kLW / 8; ++j) {
        uint32_t pw[4];
        [[maybe_unused]] uint32_t pl[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i0 = 8 * j + 2 * e;
          const float v0 = c0 + i0 <= r ? g[i0] * mm::ex2_approx(ct - csv[i0]) * dlv[i0] : 0.f;
          const float v1 = c0 + i0 + 1 <= r ? g[i0 + 1] * mm::ex2_approx(ct - csv[i0 + 1]) * dlv[i0 + 1] : 0.f;
          if constexpr (kMGPl == 2) split_bf16(v0, v1, pw[e], pl[e]);
          else pw[e] = pack_bf16(v0, v1);
        }
        const uint32_t off = pofs(r, c0 + 8 * j);
        sts_u128(sb + S::kMG + off, make_uint4(pw[0], pw[1], pw[2], pw[3]));
        if constexpr (kMGPl == 2)
          sts_u128(sb + S::kMG + uint32_t(kPanel) + off, make_uint4(pl[0], pl[1], pl[2], pl[3]));
      }
    }
    // w o x, w_s = 2^(cs_last - cs_s) Delta_s, in 8-element pieces (row pc / 8, columns
    // 8 (pc mod 8) ..): the 192 threads of the math warps off sub-partition 0 take pieces
    // u, u + 192, ...
    if (q != 0) {
      const int u = (warp - 1 - (warp >> 2)) * 32 + lane;
      for (int pc = u; pc < kQ * kP / 8; pc += 6 * 32) {
        const int row = pc >> 3;
        const float w = mm::ex2_approx(csl - cs[row]) * dl[row];
        const uint32_t off = pofs(row, (pc & 7) * 8);
        const uint4 v = lds_u128(st + S::kX + off);
        uint4 o;
        o.x = pack_bf16(w * bf16_lo(v.x), w * bf16_hi(v.x));
        o.y = pack_bf16(w * bf16_lo(v.y), w * bf16_hi(v.y));
        o.z = pack_bf16(w * bf16_lo(v.z), w * bf16_hi(v.z));
        o.w = pack_bf16(w * bf16_lo(v.w), w * bf16_hi(v.w));
        sts_u128(sb + S::kXw + off, o);
      }
    }
    mm::fence_async_shared();
    mm::tc_fence_before();
    __syncwarp();
    if (lane == 0) mm::mbar_arrive(mg_ready);
    if (warp == kCsWarp && k + 1 < nck) chunk_cs(k + 1);   // read by all after the next barrier

    // ---- the outputs of the previous chunk, while this chunk's (M o G) x and U run
    if (k > 0) {
      ok = epilogue(k - 1);
      if (!ok) continue;
    }

    // ---- the state: H <- 2^cs_last H + U, then its bf16 planes for the next chunk (u_done
    // also means this chunk's C H^T and (M o G) x are complete)
    ok = __all_sync(0xffffffffu, mm::mbar_wait(u_done, uint32_t(k) & 1u, status));
    if (!ok) continue;
    mm::tc_fence_after();
    {
      const float dec = mm::ex2_approx(csl);
      // this lane's NH2 columns of U: the first NH2 of the (q, hf) block's NH for lanes 0..15,
      // the last NH2 for lanes 16..31
      float u[NH2];
      ld_half(tq + S::kTU + uint32_t(hf * NH), u);
      mm::tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < NH2; ++i) H[i] = fmaf(dec, H[i], u[i]);
    }
    put_state();
  }
  if (ok && nck > 0) ok = epilogue(nck - 1);

  if (nck > 0) ok = bar_and(1, 32 * kMathWarps, ok);   // a failure in the last chunk counts
  mm::named_bar_sync(0, kThreads);   // pairs with the copy and MMA warps' barriers
  // the last segment leaves the final state
  if (ok && seg == a.nseg - 1 && a.h_out) {
    float* ho = a.h_out + bh * int64_t(kP * N) + int64_t(r) * N + ncol0;
#pragma unroll
    for (int i = 0; i < NH2; i += 4)
      *reinterpret_cast<float4*>(ho + i) = make_float4(H[i], H[i + 1], H[i + 2], H[i + 3]);
  }
}


// ---------------------------------------------------------------------------------------
// The state pass on the tensor cores: CTA z < nseg - 1 of row b, head h leaves the end state
// of its segment started from zero, sum_k 2^(cs_last,k ...) U_k, in ws_H slot z and the
// segment's summed Delta A log2 e in ws_A; segment 0 also copies h_in into slot nseg - 1 (the
// main pass reads the carried-in state from there, so that its last segment may write h_out
// over h_in).  Per chunk only U = (w o x)^T B runs (B and x tiles, no C), and the state
// update H <- 2^cs_last H + U.  Same warp roles as the main pass; 82 KB of shared memory and
// N TMEM columns, so two CTAs share an SM.
template <int N>
struct StateSmem {
  static constexpr int NP = N / 64;
  static constexpr int kB = 0;                     // B [64 s][N n]
  static constexpr int kX = NP * kPanel;           // x [64 s][64 p]
  static constexpr int kStage = (NP + 1) * kPanel;
  static constexpr int kXw = kNS * kStage;         // w o x [64 s][64 p]
  static constexpr int kCs = kXw + kPanel;         // [3][kQ] cs (log2 units)
  static constexpr int kDl = kCs + 3 * kQ * 4;     // [3][kQ] Delta
  static constexpr int kBar = kDl + 3 * kQ * 4;
  // full[kNS], empty[kNS], u_done, mg_ready
  static constexpr int kNBar = 2 * kNS + 2;
  static constexpr int kTotal = kBar + 8 * kNBar + 16;
  static constexpr int kDynamic = kTotal + 1024;
  static constexpr uint32_t kTmemCols = N;         // U
};

template <int N>
__global__ void __launch_bounds__(kThreads, 2)
ssd_tc_state_kernel(const __grid_constant__ CUtensorMap tm_B,
                    const __grid_constant__ CUtensorMap tm_x, const SsdArgs a, int* status) {
  using S = StateSmem<N>;
  constexpr int NP = S::NP;
  constexpr int NH = N / kCS;
  constexpr int NH2 = NH / 2;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = mm::smem_addr(smem_raw);
  unsigned char* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sb = mm::smem_addr(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + kNS;
  uint64_t* u_done = bars + 2 * kNS;
  uint64_t* mg_ready = u_done + 1;     // w o x is in shared memory
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + S::kNBar);
  float* cs_all = reinterpret_cast<float*>(smem + S::kCs);
  float* dl_all = reinterpret_cast<float*>(smem + S::kDl);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x;
  const int64_t b = blockIdx.y;
  const int seg = blockIdx.z;
  const int grp = h / (a.H / a.G);
  const int64_t L = a.L;
  const int64_t nchunks = (L + kQ - 1) / kQ;
  const int64_t c_begin = int64_t(seg) * a.cps;
  const int64_t c_end = c_begin + a.cps < nchunks ? c_begin + a.cps : nchunks;
  const int nck = c_end > c_begin ? int(c_end - c_begin) : 0;
  const int64_t bh = b * a.H + h;

  if (tid == 0) {
    for (int i = 0; i < kNS; ++i) {
      mm::mbar_init(&full[i], 1);
      mm::mbar_init(&empty[i], kMathWarps);
    }
    mm::mbar_init(u_done, 1);
    mm::mbar_init(mg_ready, kMathWarps);
  }
  if (warp == kMmaWarp) {
    mm::tmem_alloc(tmem_slot, S::kTmemCols);
    mm::tmem_relinquish();
  }
  mm::tc_fence_before();
  __syncthreads();
  mm::tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == kCopyWarp) {
    // ================================================================== copy warp
    auto issue = [&](int k) {
      const int s = k % kNS;
      const int t0 = int((c_begin + k) * kQ);
      const uint32_t st = sb + uint32_t(s * S::kStage);
      mm::mbar_arrive_expect_tx(&full[s], uint32_t(S::kStage));
      for (int pn = 0; pn < NP; ++pn)
        mm::tma_load_4d(st + S::kB + pn * kPanel, &tm_B, &full[s], pn * 64, grp, t0, int(b), 1024,
                        2, status);
      mm::tma_load_4d(st + S::kX, &tm_x, &full[s], 0, h, t0, int(b), 1024, 2, status);
    };
    bool good = true;
    if (lane == 0)
      for (int k = 0; k < nck && k < kNS; ++k) issue(k);
    int issued = nck < kNS ? nck : kNS;
    __syncwarp();
    for (int k = kNS; good && k < nck; ++k) {
      good = __all_sync(0xffffffffu, mm::mbar_wait(&empty[(k - kNS) % kNS],
                                                   uint32_t((k - kNS) / kNS) & 1u, status));
      if (!good) break;
      if (lane == 0) issue(k);
      __syncwarp();
      issued = k + 1;
    }
    mm::named_bar_sync(0, kThreads);
    if (lane == 0)
      for (int k = issued - kNS < 0 ? 0 : issued - kNS; k < issued; ++k)
        mm::mbar_wait(&full[k % kNS], uint32_t(k / kNS) & 1u, nullptr);
    __syncwarp();
    return;
  }

  if (warp == kMmaWarp) {
    // =================================================================== MMA warp
    bool good = true;
    int last = -1;   // the chunk of the last commit
    for (int k = 0; good && k < nck; ++k) {
      const int s = k % kNS;
      const uint32_t st = sb + uint32_t(s * S::kStage);
      // U_k overwrites U_{k-1}: the math warps read it before they signalled mg_ready of k
      good = __all_sync(0xffffffffu, mm::mbar_wait(&full[s], uint32_t(k / kNS) & 1u, status)) &&
             __all_sync(0xffffffffu, mm::mbar_wait(mg_ready, uint32_t(k) & 1u, status));
      if (!good) break;
      if (lane == 0) {
        mm::tc_fence_after();
        constexpr uint32_t idU = mm::umma_idesc_bf16_f32_mj<64, N, 1, 1>();
        const uint32_t dw = mm::umma_desc_lo(sb + S::kXw, kPanel);
        const uint32_t dbm = mm::umma_desc_lo(st + S::kB, kPanel);
#pragma unroll
        for (int kk = 0; kk < kQ / 16; ++kk)
          mm::umma_bf16_lo(tbase, dw + uint32_t(kk * 2048 >> 4), dbm + uint32_t(kk * 2048 >> 4),
                           idU, kk > 0 ? 1u : 0u);
        mm::umma_commit(u_done);
      }
      __syncwarp();
      last = k;
    }
    mm::named_bar_sync(0, kThreads);
    // nothing may still write TMEM when it is freed
    if (lane == 0 && last >= 0) mm::mbar_wait(u_done, uint32_t(last) & 1u, nullptr);
    __syncwarp();
    mm::tc_fence_after();
    mm::tmem_dealloc(tbase, S::kTmemCols);
    return;
  }

  // ================================================================== math warps
  const int q = warp & 3, hf = warp >> 2;
  const int part = lane >> 4;
  const int r = 16 * q + (lane & 15);
  const uint32_t tq = tbase + (uint32_t(32 * q) << 16);
  const float A2 = -expf(a.A_log[h]) * mm::kLog2e;
  const float bias = a.dt_bias[h];
  const int ncol0 = hf * NH + part * NH2;
  const int64_t col0 = int64_t(r) * N + ncol0;

  if (seg == 0 && a.h_in) {   // the copy of h_in the main pass starts from
    const float* hi = a.h_in + bh * int64_t(kP * N);
    float* hc = a.ws_H + (bh * a.nseg + a.nseg - 1) * int64_t(kP * N);
#pragma unroll
    for (int i = 0; i < NH2; i += 4)
      *reinterpret_cast<float4*>(hc + col0 + i) = *reinterpret_cast<const float4*>(hi + col0 + i);
  }
  float H[NH2];
#pragma unroll
  for (int i = 0; i < NH2; ++i) H[i] = 0.0f;
  float seg_a = 0.0f;

  DtRing dtr;
  auto load_dt = [&](int k) {   // chunk k of the segment into slot k mod kDtAhead
    dtr.load(k % kDtAhead, a.dt, b * L, L, a.H, h, (c_begin + k) * kQ + 2 * lane);
  };
  auto chunk_cs = [&](int k) {   // warp kCsWarp; dt of chunk k loaded
    float* cs = cs_all + (k % 3) * kQ;
    float* dl = dl_all + (k % 3) * kQ;
    const int64_t t = (c_begin + k) * kQ + 2 * lane;
    float r0, r1;
    dtr.take(k % kDtAhead, r0, r1);
    const float d0 = t < L ? mm::Math<false>::softplus(r0 + bias) : 0.f;
    const float d1 = t + 1 < L ? mm::Math<false>::softplus(r1 + bias) : 0.f;
    if (k + kDtAhead < nck) load_dt(k + kDtAhead);
    const float e0 = d0 * A2, e1 = d1 * A2;
    float sum = e0 + e1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float v = __shfl_up_sync(0xffffffffu, sum, o);
      if (lane >= o) sum += v;
    }
    float ex = __shfl_up_sync(0xffffffffu, sum, 1);
    if (lane == 0) ex = 0.f;
    cs[2 * lane] = ex + e0;
    cs[2 * lane + 1] = ex + e0 + e1;
    dl[2 * lane] = d0;
    dl[2 * lane + 1] = d1;
  };
  if (warp == kCsWarp && nck > 0) {
    for (int k = 0; k < kDtAhead && k < nck; ++k) load_dt(k);
    chunk_cs(0);
  }

  bool ok = true;
  for (int k = 0; k < nck; ++k) {
    const int s = k % kNS;
    const uint32_t st = sb + uint32_t(s * S::kStage);
    const float* cs = cs_all + (k % 3) * kQ;
    const float* dl = dl_all + (k % 3) * kQ;
    ok = bar_and(1, 32 * kMathWarps, ok);      // this chunk's cs and Delta visible
    if (!ok) break;
    const float csl = cs[kQ - 1];
    seg_a += csl;
    ok = __all_sync(0xffffffffu, mm::mbar_wait(&full[s], uint32_t(k / kNS) & 1u, status));
    if (!ok) continue;
    // w o x, w_s = 2^(cs_last - cs_s) Delta_s, in 8-element pieces: the 192 threads of the
    // math warps off sub-partition 0 take pieces u, u + 192, ...
    if (q != 0) {
      const int u = (warp - 1 - (warp >> 2)) * 32 + lane;
      for (int pc = u; pc < kQ * kP / 8; pc += 6 * 32) {
        const int row = pc >> 3;
        const float w = mm::ex2_approx(csl - cs[row]) * dl[row];
        const uint32_t off = pofs(row, (pc & 7) * 8);
        const uint4 v = lds_u128(st + S::kX + off);
        uint4 o;
        o.x = pack_bf16(w * bf16_lo(v.x), w * bf16_hi(v.x));
        o.y = pack_bf16(w * bf16_lo(v.y), w * bf16_hi(v.y));
        o.z = pack_bf16(w * bf16_lo(v.z), w * bf16_hi(v.z));
        o.w = pack_bf16(w * bf16_lo(v.w), w * bf16_hi(v.w));
        sts_u128(sb + S::kXw + off, o);
      }
    }
    mm::fence_async_shared();
    mm::tc_fence_before();
    __syncwarp();
    if (lane == 0) mm::mbar_arrive(mg_ready);
    if (warp == kCsWarp && k + 1 < nck) chunk_cs(k + 1);   // read by all after the next barrier

    ok = __all_sync(0xffffffffu, mm::mbar_wait(u_done, uint32_t(k) & 1u, status));
    if (!ok) continue;
    mm::tc_fence_after();
    {
      const float dec = mm::ex2_approx(csl);
      float u[NH2];
      ld_half(tq + uint32_t(hf * NH), u);
      mm::tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < NH2; ++i) H[i] = fmaf(dec, H[i], u[i]);
    }
    mm::tc_fence_before();
    __syncwarp();
    if (lane == 0) mm::mbar_arrive(&empty[s]);   // the stage's tiles and U are read
  }
  if (nck > 0) ok = bar_and(1, 32 * kMathWarps, ok);
  mm::named_bar_sync(0, kThreads);
  if (ok && seg < a.nseg - 1) {
    float* out = a.ws_H + (bh * a.nseg + seg) * int64_t(kP * N) + col0;
#pragma unroll
    for (int i = 0; i < NH2; i += 4)
      *reinterpret_cast<float4*>(out + i) = make_float4(H[i], H[i + 1], H[i + 2], H[i + 3]);
    if (tid == 0) a.ws_A[bh * (a.nseg - 1) + seg] = seg_a;
  }
}

}  // namespace tc
}  // namespace ssd
