// Fused forward of the selective-SSM mixer core for bf16 I/O on sm_100a (calm-mamba 0.1.4,
// section "Mamba operator", steps 2 and 4-6): causal conv + SiLU, Delta = softplus(dt_raw +
// dt_bias), the selective scan h = exp(Delta*A)*h + Delta*B*u, y = C.h + D*u, the gate
// y*SiLU(z), and the final states.
//
// Work decomposition
//   CTA    = 32 channels of one batch row over one time chunk ("unit"); 4G scan warps in G
//            time groups of 4, plus one producer warp.
//   tile   = 32 time steps, staged by TMA (3-D tensor maps, no multicast) into a ring of
//            kStages; negative time coordinates read zeros (the causal left padding).
//   producer warp: issues the copies of x' (with a 4-row halo for the conv), z, dt_raw, B
//            and C, and widens each tile's B and C once into fp32 records [t][j]{B[kS],C[kS]}
//            that all 32 channels' lanes read.
//   scan lane (chl = lane & 7, j = lane >> 3) of warp w of group g: channel 8w + chl, states
//            n in [j*kS, (j+1)*kS), kS = N/4.  For each quad (4 steps) of its group's part of
//            the tile the lane first computes the per-(t, d) scalars of step 4q + j -- conv,
//            SiLU, softplus, Delta*u, D*u, SiLU(z) -- once per (t, d); the 4 lanes of a
//            channel swap Delta and Delta*u through shared memory, then all advance their
//            states over the quad; the readouts C.h are reduce-scattered so that lane j
//            finishes (gates, stores) step 4q + j, whose D*u and SiLU(z) it already holds.
//
// Time groups: the two-level scan (G > 1).  Group g scans steps [g*R, (g+1)*R) of every tile
// (R = 32/G) from a zero state, keeping the running decay product P_t and C_t*P_t per step
// next to its local readouts.  The state entering its block, h_in, is the end state of the
// block before it, handed along a chain through shared memory (group g-1, or group G-1 of
// the previous tile for g = 0): its own end state is P*h_in + h_local, and each readout
// gets the term sum_n C_t[n] P_t[n] h_in[n].  That is the (a, b)-pair composition
// (a1, b1) o (a2, b2) = (a1 a2, a2 b1 + b2) applied once per block, so G blocks of a tile
// advance in parallel while the carried prefix moves along the chain.
//
// Chunks (kChained): a long row is cut into chunks whose units are claimed in order from a
// counter; the unit of chunk c > 0 starts from the end state that chunk c - 1 left in the
// workspace (a flag per warp with release/acquire ordering), so nothing is recomputed.
//
// Packed documents and initial state (kExt; niverel-mamba 0.1.0, section "seq_idx strict
// reset"): where seq_idx changes both states restart at that step -- conv taps before it are
// dropped and its decay input becomes +inf (exp(+inf*A) = 0 with A clamped strictly
// negative), which also zeroes P, so the carried h_in stops there.  h_in / conv_state_in seed
// the first chunk.
//
// Every wait (mbarriers, the chain, the chunk flags) is bounded: a warp that gives up leaves
// its loop, records MAMBA_ERR_TIMEOUT in the status word, and the CTA exits cleanly.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <float.h>

#include "device_math.cuh"
#include "sm100_primitives.cuh"

namespace mm {
namespace f2 {

constexpr int kCh = 32;        // channels per CTA
constexpr int kTileT = 32;     // steps per tile
constexpr int kHalo = 4;       // x' rows before each tile (3 needed)
constexpr int kMaxDtBlocks = 2;  // fused dt projection: dt_rank up to 128, K blocks of 64

// TMA ring depth: 3 for one time group with the dt projection fused (its operands would
// otherwise keep three CTAs from sharing an SM), else 4
__host__ __device__ constexpr int ring_depth(int G, int KB) { return KB > 0 && G == 1 ? 3 : 4; }
constexpr int kGroupWarps = 4; // scan warps per time group (8 channels x 4 lanes each)

// scan warps, the producer warp, and (the dt projection fused with G > 1) the product warp
template <int G, int KB = 0>
__host__ __device__ constexpr int threads() {
  return 32 * (kGroupWarps * G + 1 + (KB > 0 && G > 1 ? 1 : 0));
}

struct Params {
  const float* A_log;
  const float* D;
  const float* conv_w;
  const float* conv_b;      // may be null
  const float* dt_bias;
  __nv_bfloat16* y;
  float* h_out;             // may be null
  __nv_bfloat16* cs_out;    // may be null
  int* status;              // device status word
  const int32_t* seq_idx;   // kExt, may be null
  const float* h_in;        // kExt, may be null
  const __nv_bfloat16* cs_in;  // kExt, may be null
  int* unit_counter;        // kChained
  int* carry_flag;          // kChained: [tiles][kGroupWarps]
  float* carry;             // kChained: [tiles][kCh][N]
  float* ckpt;              // kCkpt: the state at the start of every 16-step tile,
                            // fp32 [batch, ceil(L/16), d_inner, N]
  int64_t L, Di;
  int64_t chunk_len;        // multiple of kTileT
  int nchunks, ntd, batch;
  int inject_skip_tile;     // test hook: -1 = off
  int dt_rank;              // KB > 0: columns of dt_low and W_dt (<= 64 * KB)
};

// KB = K blocks of the fused dt projection (0: dt_raw is an input)
template <int N, int G, int KB = 0>
struct Smem {
  static constexpr bool kDtProj = KB > 0;
  static constexpr int kStages = ring_depth(G, KB);
  static constexpr int kS = N / 4;
  static constexpr int kRow = kCh * 2;                         // 64-byte rows (bf16)
  static constexpr int align1k(int v) { return (v + 1023) / 1024 * 1024; }
  static constexpr int kXOff = 0;
  static constexpr int kZOff = align1k((kTileT + kHalo) * kRow);
  // dt_raw tile (bf16, 64-byte swizzle) -- or, with the dt projection fused, the tile's
  // dt_low rows (bf16, 128-byte swizzle, K blocks of 64), which the product in fp32 then
  // overwrites once the tensor cores have read them: [t][32], channel c of step t at word
  // t*32 + (c ^ 8*(t & 3)), so that both the producer's row writes and the scan lanes'
  // reads (steps 4q..4q+3 x 8 channels) hit 32 distinct banks
  static constexpr int kDtOff = kZOff + align1k(kTileT * kRow);
  static constexpr int kDtBytes = kDtProj ? KB * kTileT * 128 : align1k(kTileT * kRow);
  static constexpr int kBOff = kDtOff + kDtBytes;
  static constexpr int kCOff = kBOff + align1k(kTileT * N * 2);
  static constexpr int kBCRec = 2 * kS * 4;                    // fp32 {B[kS], C[kS]}
  static constexpr int kBCfOff = kCOff + align1k(kTileT * N * 2);
  static constexpr int kStage = kBCfOff + align1k(kTileT * 4 * kBCRec);
  static constexpr int kXchOff = kStages * kStage;             // Delta / Delta*u swap
  static constexpr int kXchRec = 48;                           // {Delta[4]}, {Delta*u[4]}, pad
  static constexpr int kXchWarp = 2 * 8 * kXchRec;             // quad parity x channels
  static constexpr int kSlotOff = kXchOff + kGroupWarps * G * kXchWarp;
  static constexpr int kSlotBytes = G > 1 ? G * kGroupWarps * 32 * kS * 4 : 0;
  // KB > 0: W_dt of the CTA's channels as the M = 128 operand (rows 32..127 zero), per K block
  static constexpr int kWOff = align1k(kSlotOff + kSlotBytes);
  static constexpr int kWBytes = KB * 128 * 128;
  static constexpr int kBarOff = kWOff + kWBytes;
  static constexpr int kBars = 3 * kStages + G * kGroupWarps + 2;   // + W landed, MMA done
  static constexpr int kTotal = kBarOff + 8 * kBars + 16;      // + the TMEM address
  static constexpr int kDynamic = kTotal + 1024;               // slack to align to 1 KiB
};

__device__ __forceinline__ float bf(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// Byte offset of (row, col) in a TMA tile with 64-byte rows and the 64-byte swizzle.
__device__ __forceinline__ uint32_t swz64(int row, int col_bytes) {
  const uint32_t a = uint32_t(row) * 64u + uint32_t(col_bytes);
  return a ^ (((a >> 7) & 3u) << 4);
}

__device__ __forceinline__ void sts_v4(uint32_t a, float x, float y, float z, float w) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(x), "f"(y), "f"(z),
               "f"(w) : "memory");
}
__device__ __forceinline__ void sts_v2(uint32_t a, float x, float y) {
  asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(a), "f"(x), "f"(y) : "memory");
}
__device__ __forceinline__ float2 lds_v2(uint32_t a) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
  return v;
}

// Document resets of the tile's steps tt-4 .. tt+31: bit i set when step tt-4+i starts a new
// document (its id differs from the previous step's; step 0 never does).  One warp, two
// loads per lane.
__device__ __forceinline__ uint64_t tile_resets(const int32_t* seq, int64_t tt, int64_t L,
                                                int lane) {
  const int64_t s_lo = tt - 4 + lane, s_hi = tt + 28 + lane;
  const bool in_lo = s_lo >= 0 && s_lo < L, in_hi = lane < 4 && s_hi >= 0 && s_hi < L;
  const int32_t lo = in_lo ? __ldg(seq + s_lo) : 0;
  const int32_t hi = in_hi ? __ldg(seq + s_hi) : 0;
  const int32_t lo_prev = __shfl_up_sync(0xffffffffu, lo, 1);
  const int32_t lo_31 = __shfl_sync(0xffffffffu, lo, 31);
  const int32_t hi_up = __shfl_up_sync(0xffffffffu, hi, 1);
  const int32_t hi_prev = lane == 0 ? lo_31 : hi_up;
  const bool r_lo = in_lo && lane >= 1 && s_lo >= 1 && lo != lo_prev;
  const bool r_hi = in_hi && s_hi >= 1 && hi != hi_prev;
  return uint64_t(__ballot_sync(0xffffffffu, r_lo)) |
         (uint64_t(__ballot_sync(0xffffffffu, r_hi)) << 32);
}

template <int N, bool kExt, int G, bool kChained, int KB = 0, bool kCkpt = false>
__global__ void __launch_bounds__(threads<G, KB>(), G == 1 ? 3 : 1)
fwd2_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_z,
            const __grid_constant__ CUtensorMap tm_dt, const __grid_constant__ CUtensorMap tm_B,
            const __grid_constant__ CUtensorMap tm_C, const __grid_constant__ CUtensorMap tm_w,
            const Params p) {
  using S = Smem<N, G, KB>;
  constexpr bool kDtProj = KB > 0;
  constexpr int kStages = S::kStages;
  constexpr int kS = N / 4;
  constexpr int kP = kS / 2;              // f32x2 pairs per lane
  constexpr int R = kTileT / G;           // steps per group per tile
  constexpr int QG = R / 4;               // quads per group per tile
  constexpr int kScanWarps = kGroupWarps * G;
  constexpr int kThreads = threads<G, KB>();
  // the products run on a warp of their own beside many scan warps (whose tiles come fast),
  // else on the producer warp
  constexpr bool kMmaWarp = kDtProj && G > 1;
  constexpr bool kProdMma = kDtProj && !kMmaWarp;
  constexpr int kDLane = kMmaWarp ? 32 : 0;
  static_assert(!kMmaWarp || (kGroupWarps * G + 1) % 4 == 1, "product warp reads TMEM lanes 32..63");
  static_assert(!kProdMma || (kGroupWarps * G) % 4 == 0, "producer reads TMEM lanes 0..31");
  static_assert(G == 1 || G == 2 || G == 4, "1, 2 or 4 time groups");
  static_assert(N == 8 || N == 16, "d_state 8 or 16");

  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  unsigned char* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sb = smem_addr(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOff);   // tile landed
  uint64_t* bc_ready = full + kStages;                               // B/C widened
  uint64_t* empty = bc_ready + kStages;                              // all scan warps done
  uint64_t* end_ready = empty + kStages;                             // [G][kGroupWarps]
  uint64_t* w_bar = end_ready + G * kGroupWarps;                     // kDtProj: W_dt landed
  uint64_t* mma_bar = w_bar + 1;                                     // kDtProj: product done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_bar + 1);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int tile = 0, d0 = int(blockIdx.x) * kCh, b = int(blockIdx.y), c = int(blockIdx.z);
  if constexpr (kChained) {
    __shared__ int s_unit;
    if (tid == 0) s_unit = atomicAdd(p.unit_counter, 1);
    __syncthreads();
    const int tiles_total = p.batch * p.ntd;
    tile = s_unit % tiles_total;
    c = s_unit / tiles_total;
    b = tile / p.ntd;
    d0 = (tile % p.ntd) * kCh;
  }
  const int64_t t_begin = int64_t(c) * p.chunk_len;
  const int64_t t_end = t_begin + p.chunk_len < p.L ? t_begin + p.chunk_len : p.L;
  const int ntiles = int((t_end - t_begin + kTileT - 1) / kTileT);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&bc_ready[s], kMmaWarp ? 2 : 1);   // B/C widened (and the product read back)
      mbar_init(&empty[s], kScanWarps);
    }
    for (int i = 0; i < G * kGroupWarps; ++i) mbar_init(&end_ready[i], 1);
    mbar_init(w_bar, 1);
    mbar_init(mma_bar, 1);
  }
  __syncthreads();

  // ---- the fused dt projection (KB > 0): dt_raw of tile k = W_dt (channels x rank) *
  // dt_low (steps x rank)^T on the tensor cores, D[channel][step] in 32 TMEM columns of lanes
  // kDLane..kDLane+31 (the lanes the issuing warp may read: warp index mod 4 = kDLane / 32).
  // The product is read back over the tile's consumed dt_low rows in the swizzled fp32 layout
  // the prep reads, and the next tile's product is issued right after, so that it runs while
  // the warp waits for the next tile.
  [[maybe_unused]] uint32_t tbase = 0;
  [[maybe_unused]] int mma_issued = 0, mma_waited = 0;
  [[maybe_unused]] auto dt_setup = [&]() {
    tmem_alloc(tmem_slot, 32);
    tmem_relinquish();
    // the M = 128 operand: W_dt's 32 rows at kDLane by TMA, the other 96 rows zero
    const uint32_t wb = sb + uint32_t(S::kWOff);
    for (int kb = 0; kb < KB; ++kb)
      for (int i = lane; i < 96 * 8; i += 32) {
        const int chunk = i < kDLane * 8 ? i : i + 32 * 8;   // 16-byte chunks, 8 per row
        sts_v4(wb + uint32_t(kb * 16384 + chunk * 16), 0.f, 0.f, 0.f, 0.f);
      }
    fence_async_shared();
    __syncwarp();
    tc_fence_before();
    __syncwarp();
    tc_fence_after();
    tbase = *tmem_slot;
    if (lane == 0) {
      mbar_arrive_expect_tx(w_bar, uint32_t(KB * 32 * 128));
      for (int kb = 0; kb < KB; ++kb)
        tma_load_2d(wb + uint32_t(kb * 16384 + kDLane * 128), &tm_w, w_bar, kb * 64, d0, 1024, 2,
                    p.status);
    }
    __syncwarp();
  };
  [[maybe_unused]] auto dt_issue = [&](int k) -> bool {
    const int s = k % kStages;
    if (!__all_sync(0xffffffffu, mbar_wait(&full[s], uint32_t(k / kStages) & 1u, p.status)))
      return false;
    if (k == 0 && !__all_sync(0xffffffffu, mbar_wait(w_bar, 0, p.status))) return false;
    if (lane == 0) {
      tc_fence_after();
      const uint32_t st = sb + uint32_t(s * S::kStage);
      constexpr uint32_t idesc = umma_idesc_bf16_f32<128, kTileT>();
      int n = 0;
      for (int kb = 0; kb < KB; ++kb)
        for (int kk = 0; kk < 4 && kb * 64 + kk * 16 < p.dt_rank; ++kk, ++n)
          umma_bf16(tbase, umma_desc_sw128(sb + uint32_t(S::kWOff + kb * 16384 + kk * 32)),
                    umma_desc_sw128(st + uint32_t(S::kDtOff + kb * kTileT * 128 + kk * 32)), idesc,
                    n > 0 ? 1u : 0u);
      umma_commit(mma_bar);
    }
    __syncwarp();
    ++mma_issued;
    return true;
  };
  [[maybe_unused]] auto dt_readback = [&](int k) -> bool {
    if (!__all_sync(0xffffffffu, mbar_wait(mma_bar, uint32_t(k) & 1u, p.status))) return false;
    ++mma_waited;
    tc_fence_after();
    float v[kTileT];
    tmem_ld32(tbase + (uint32_t(kDLane) << 16), v);
    tmem_wait_ld();
    const uint32_t dt32 = sb + uint32_t((k % kStages) * S::kStage + S::kDtOff);
#pragma unroll
    for (int t = 0; t < kTileT; ++t)
      sts_f32(dt32 + uint32_t((t * 32 + (lane ^ ((t & 3) << 3))) * 4), v[t]);
    // these generic writes precede the refill's TMA writes to the same bytes
    fence_async_shared();
    tc_fence_before();
    __syncwarp();
    return true;
  };
  [[maybe_unused]] auto dt_teardown = [&]() {
    // W_dt's copy must have landed and no product may still be writing the accumulator
    if (mma_issued == 0) mbar_wait(w_bar, 0, nullptr);
    if (mma_issued > mma_waited) mbar_wait(mma_bar, uint32_t(mma_issued - 1) & 1u, nullptr);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tbase, 32);
  };

  if constexpr (kMmaWarp) {
    if (warp == kScanWarps + 1) {
      // ============================================================== product warp
      dt_setup();
      bool good = dt_issue(0);
      for (int k = 0; good && k < ntiles; ++k) {
        good = dt_readback(k);
        if (!good) break;
        if (lane == 0) mbar_arrive(&bc_ready[k % kStages]);
        if (k + 1 < ntiles) good = dt_issue(k + 1);
      }
      named_bar_sync(0, kThreads);
      dt_teardown();
      return;
    }
  }

  if (warp == kScanWarps) {
    // ================================================================ producer warp
    const uint32_t kTx = uint32_t((kTileT + kHalo) * S::kRow + kTileT * S::kRow +
                                  (kDtProj ? KB * kTileT * 128 : kTileT * S::kRow) +
                                  2 * kTileT * N * 2);
    if constexpr (kProdMma) dt_setup();
    int issued = 0;
    auto issue = [&](int k) {
      const int s = k % kStages;
      const bool skip = k == p.inject_skip_tile && d0 == 0 && b == 0 && c == 0;
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], kTx);
        if (!skip) {
          const uint32_t st = sb + uint32_t(s * S::kStage);
          const int tt = int(t_begin) + k * kTileT;
          tma_load_3d(st + S::kXOff, &tm_x, &full[s], d0, tt - kHalo, b, 1024, 2, p.status);
          tma_load_3d(st + S::kZOff, &tm_z, &full[s], d0, tt, b, 1024, 2, p.status);
          if constexpr (kDtProj) {
            for (int kb = 0; kb < KB; ++kb)
              tma_load_3d(st + S::kDtOff + kb * kTileT * 128, &tm_dt, &full[s], kb * 64, tt, b,
                          1024, 2, p.status);
          } else {
            tma_load_3d(st + S::kDtOff, &tm_dt, &full[s], d0, tt, b, 1024, 2, p.status);
          }
          tma_load_3d(st + S::kBOff, &tm_B, &full[s], 0, tt, b, 128, 2, p.status);
          tma_load_3d(st + S::kCOff, &tm_C, &full[s], 0, tt, b, 128, 2, p.status);
        }
      }
      __syncwarp();
      issued = k + 1;
    };
    for (int k = 0; k < ntiles && k < kStages; ++k) issue(k);
    bool good = true;
    if constexpr (kProdMma) good = dt_issue(0);
    for (int k = 0; good && k < ntiles; ++k) {
      const int s = k % kStages;
      good = __all_sync(0xffffffffu, mbar_wait(&full[s], uint32_t(k / kStages) & 1u, p.status));
      if (!good) break;
      // widen B and C of this tile: record (t, jj) = {B[t][jj*kS ..], C[t][jj*kS ..]}
      const uint32_t st = sb + uint32_t(s * S::kStage);
#pragma unroll
      for (int idx = lane; idx < kTileT * 4; idx += 32) {
        const int t = idx >> 2, jj = idx & 3;
        const uint32_t src = uint32_t((t * N + jj * kS) * 2);
        const uint32_t dst = st + S::kBCfOff + uint32_t(idx * S::kBCRec);
        if constexpr (kS == 4) {
          uint32_t b0, b1, c0, c1;
          asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(b0), "=r"(b1) : "r"(st + S::kBOff + src));
          asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(c0), "=r"(c1) : "r"(st + S::kCOff + src));
          sts_v4(dst, bf(b0 & 0xffffu), bf(b0 >> 16), bf(b1 & 0xffffu), bf(b1 >> 16));
          sts_v4(dst + 16, bf(c0 & 0xffffu), bf(c0 >> 16), bf(c1 & 0xffffu), bf(c1 >> 16));
        } else {
          uint32_t b0, c0;
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(b0) : "r"(st + S::kBOff + src));
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(c0) : "r"(st + S::kCOff + src));
          sts_v4(dst, bf(b0 & 0xffffu), bf(b0 >> 16), bf(c0 & 0xffffu), bf(c0 >> 16));
        }
      }
      if constexpr (kProdMma) {
        good = dt_readback(k);
        if (!good) break;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bc_ready[s]);
      if constexpr (kProdMma) {
        if (k + 1 < ntiles) {
          good = dt_issue(k + 1);
          if (!good) break;
        }
      }
      // refill the stage of the previous tile once every scan warp is done with it
      if (k >= 1 && k - 1 + kStages < ntiles) {
        const int sp = (k - 1) % kStages;
        good = __all_sync(0xffffffffu,
                          mbar_wait(&empty[sp], uint32_t((k - 1) / kStages) & 1u, p.status));
        if (!good) break;
        issue(k - 1 + kStages);
      }
    }
    named_bar_sync(0, kThreads);
    if (!good && lane == 0) {
      // every copy this CTA started must land before it exits
      for (int k = issued - kStages < 0 ? 0 : issued - kStages; k < issued; ++k)
        mbar_wait(&full[k % kStages], uint32_t(k / kStages) & 1u, nullptr);
    }
    if constexpr (kProdMma) dt_teardown();
    return;
  }
  // ================================================================== scan warps
  const int g = warp / kGroupWarps;       // time group
  const int w4 = warp % kGroupWarps;      // channel slice of the group
  const int chl = lane & 7, j = lane >> 3;
  const int cl = w4 * 8 + chl;            // channel within the CTA
  // d_inner % 8 == 0: a warp's 8 channels are all in range or all out; an out-of-range warp
  // still walks the tiles (it releases every stage and passes the chain) but stores nothing
  const bool active = d0 + cl < p.Di;
  const int64_t d = active ? d0 + cl : 0;

  // per-channel parameters of the prep; A (times log2 e) of this lane's states
  const float4 cw = __ldg(reinterpret_cast<const float4*>(p.conv_w + d * 4));
  const float cb = p.conv_b ? __ldg(p.conv_b + d) : 0.0f;
  const float dtb = __ldg(p.dt_bias + d);
  const float Dd = __ldg(p.D + d);
  f32x2 A2p[kP];
#pragma unroll
  for (int pp = 0; pp < kP; ++pp) {
    float a[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      // A = -exp(A_log) times log2 e, clamped finite (a masked step, Delta = 0, decays by
      // exactly 1); with documents also strictly negative (a reset step decays to exactly 0)
      a[e] = fmaxf(-ex2_approx(__ldg(p.A_log + d * N + j * kS + 2 * pp + e) * kLog2e) * kLog2e,
                   -FLT_MAX);
      if constexpr (kExt) a[e] = fminf(a[e], -FLT_MIN);
    }
    A2p[pp] = pk2(a[0], a[1]);
  }

  // the state entering the unit (group 0's first block)
  float h0[kS];
#pragma unroll
  for (int s = 0; s < kS; ++s) h0[s] = 0.0f;
  bool ok = true;
  if (g == 0) {
    if (kChained && c > 0) {
      if (active)
        ok = wait_flag_geq(p.carry_flag + tile * kGroupWarps + w4, c, p.status);
      ok = __all_sync(0xffffffffu, ok);
      if (ok && active) {
        const float* src = p.carry + (int64_t(tile) * kCh + cl) * N + j * kS;
#pragma unroll
        for (int s = 0; s < kS; ++s) h0[s] = __ldcg(src + s);
      }
    } else if (kExt && c == 0 && p.h_in) {
      const float* hi = p.h_in + (int64_t(b) * p.Di + d) * N + j * kS;
#pragma unroll
      for (int s = 0; s < kS; ++s) h0[s] = __ldg(hi + s);
    }
  }
  f32x2 hp[kP];     // G == 1: the state itself; G > 1: the local state of the block
#pragma unroll
  for (int pp = 0; pp < kP; ++pp) hp[pp] = pk2(h0[2 * pp], h0[2 * pp + 1]);
  f32x2 hin[kP];    // G > 1: the state entering the block
#pragma unroll
  for (int pp = 0; pp < kP; ++pp) hin[pp] = hp[pp];

  // the state entering the 16-step tile that starts at step t < L, when checkpoints are asked
  [[maybe_unused]] auto put_ckpt = [&](int64_t t, const f32x2* hv) {
    if (kCkpt && active && t < p.L) {
      float v[kS];
#pragma unroll
      for (int pp = 0; pp < kP; ++pp) upk2(hv[pp], v[2 * pp], v[2 * pp + 1]);
      float* o = p.ckpt + ((int64_t(b) * ((p.L + 15) / 16) + t / 16) * p.Di + d) * N + j * kS;
      if constexpr (kS == 4) __stcg(reinterpret_cast<float4*>(o), make_float4(v[0], v[1], v[2], v[3]));
      else __stcg(reinterpret_cast<float2*>(o), make_float2(v[0], v[1]));
    }
  };
  if (kCkpt && G > 1 && c == 0 && g == 0) put_ckpt(0, hp);

  const uint32_t xch = sb + uint32_t(S::kXchOff + warp * S::kXchWarp);
  __nv_bfloat16* yrow = p.y + (int64_t(b) * p.L + t_begin + j) * p.Di + d;
  const int col = cl * 2;
  // swizzled offsets of this lane's prep loads for quads of either parity (the 64-byte
  // swizzle repeats every 8 rows, so quad qq + 2 reads 512 bytes further on)
  uint32_t xoff[2][4], dtoff[2], zoff[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int t = (g * QG + e) * 4 + j;
#pragma unroll
    for (int m = 0; m < 4; ++m) xoff[e][m] = uint32_t(S::kXOff) + swz64(t + 1 + m, col);
    dtoff[e] = kDtProj ? uint32_t(S::kDtOff + (t * 32 + (cl ^ (j << 3))) * 4)
                       : uint32_t(S::kDtOff) + swz64(t, col);
    zoff[e] = uint32_t(S::kZOff) + swz64(t, col);
  }

  for (int k = 0; ok && k < ntiles; ++k) {
    const int s = k % kStages;
    ok = __all_sync(0xffffffffu, mbar_wait(&bc_ready[s], uint32_t(k / kStages) & 1u, p.status));
    if (!ok) break;
    const uint32_t st = sb + uint32_t(s * S::kStage);
    const int64_t tt = t_begin + int64_t(k) * kTileT;
    const int64_t valid_n = t_end - tt;             // steps of this tile inside the chunk
    __nv_bfloat16* ytile = yrow + int64_t(k) * kTileT * p.Di;   // step j of the tile

    [[maybe_unused]] uint64_t rs = 0;
    if constexpr (kExt) if (p.seq_idx) rs = tile_resets(p.seq_idx + int64_t(b) * p.L, tt, p.L, lane);
    f32x2 Pp[kP];
    [[maybe_unused]] f32x2 CP[G > 1 ? R : 1][kP];
    [[maybe_unused]] float yl[G > 1 ? R : 4];
    [[maybe_unused]] float skip[QG], szg[QG];
#pragma unroll
    for (int pp = 0; pp < kP; ++pp) {
      Pp[pp] = pk2(1.0f, 1.0f);
      if constexpr (G > 1) hp[pp] = pk2(0.0f, 0.0f);
    }
    // reduce-scatter of one quad's readouts over the 4 lanes of a channel, gate, store
    auto emit = [&](int qq, const float* yp, float sk, float sz) {
      const bool hi = (j & 2) != 0;
      float k0 = hi ? yp[2] : yp[0], k1 = hi ? yp[3] : yp[1];
      const float s0 = hi ? yp[0] : yp[2], s1 = hi ? yp[1] : yp[3];
      k0 += __shfl_xor_sync(0xffffffffu, s0, 16);
      k1 += __shfl_xor_sync(0xffffffffu, s1, 16);
      const bool odd = (j & 1) != 0;
      float kp = odd ? k1 : k0;
      const float sp = odd ? k0 : k1;
      kp += __shfl_xor_sync(0xffffffffu, sp, 8);
      const int t = (g * QG + qq) * 4 + j;
      if (t < valid_n && active) ytile[(g * QG + qq) * 4 * p.Di] = __float2bfloat16_rn((kp + sk) * sz);
    };
#pragma unroll
    for (int qq = 0; qq < QG; ++qq) {
      // ---- prep: the per-(t, d) scalars of step t = 4q + j (q = g*QG + qq), once per (t, d)
      const int t = (g * QG + qq) * 4 + j;          // step within the tile
      const uint32_t rb = st + uint32_t(512 * (qq >> 1));   // the swizzle repeats every 8 rows
      const int e = qq & 1;
      // x' tile row r holds step tt - 4 + r: taps x'[t-3..t] are rows t+1..t+4
      float x3 = bf(lds_u16(rb + xoff[e][0]));
      float x2 = bf(lds_u16(rb + xoff[e][1]));
      float x1 = bf(lds_u16(rb + xoff[e][2]));
      const float x0 = bf(lds_u16(rb + xoff[e][3]));
      if constexpr (kExt) {
        if (p.cs_in && c == 0 && k == 0 && t < 3) {
          // steps before the row: the cached window instead of the zero padding
          const __nv_bfloat16* cwin = p.cs_in + (int64_t(b) * p.Di + d) * 3;
          if (t < 1) x1 = __bfloat162float(cwin[2]);
          if (t < 2) x2 = __bfloat162float(cwin[1 + t]);
          x3 = __bfloat162float(cwin[t]);
        }
        if (p.seq_idx) {
          // a tap lies before the document's first step when a reset sits between them
          const bool r0 = (rs >> (t + 4)) & 1u, r1 = (rs >> (t + 3)) & 1u, r2 = (rs >> (t + 2)) & 1u;
          if (r0) x1 = 0.0f;
          if (r0 || r1) x2 = 0.0f;
          if (r0 || r1 || r2) x3 = 0.0f;
        }
      }
      const float pre = fmaf(cw.w, x0, fmaf(cw.z, x1, fmaf(cw.y, x2, fmaf(cw.x, x3, cb))));
      const float u = silu_tanh(pre);
      const float dtv = kDtProj ? lds_f32(st + dtoff[e] + uint32_t((qq >> 1) * 8 * 32 * 4))
                                : bf(lds_u16(rb + dtoff[e]));
      const float dl = softplus_lg2(dtv + dtb);
      const bool valid = t < valid_n;
      float dlt = valid ? dl : 0.0f;
      const float du = valid ? dl * u : 0.0f;
      if constexpr (kExt)
        if (valid && ((rs >> (t + 4)) & 1u)) dlt = __int_as_float(0x7f800000);   // decay 0
      const float sk = Dd * u;
      const float sz = silu_tanh(bf(lds_u16(rb + zoff[e])));
      // swap area of quad parity qq & 1: channel chl's {Delta[4], Delta*u[4]} (48-byte records:
      // both the lanes' 4-byte stores and the 16-byte loads are free of bank conflicts).  Two
      // areas suffice: quad qq + 2 overwrites quad qq's only after the __syncwarp of quad
      // qq + 1, which every lane reaches after its loads of quad qq.
      const uint32_t xa = xch + uint32_t(((qq & 1) * 8 + chl) * S::kXchRec);
      sts_f32(xa + 4 * j, dlt);
      sts_f32(xa + 16 + 4 * j, du);
      __syncwarp();

      // ---- scan of the quad
      const int q = g * QG + qq;
      const float4 dv = lds_f32x4(xa);
      const float4 duv = lds_f32x4(xa + 16);
      const float di[4] = {dv.x, dv.y, dv.z, dv.w};
      const float dui[4] = {duv.x, duv.y, duv.z, duv.w};
      float yq[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t row = st + S::kBCfOff + uint32_t(((4 * q + i) * 4 + j) * S::kBCRec);
        f32x2 Bp[kP], Cp[kP];
        if constexpr (kS == 4) {
          const float4 bv = lds_f32x4(row);
          const float4 cv = lds_f32x4(row + 16);
          Bp[0] = pk2(bv.x, bv.y); Bp[1] = pk2(bv.z, bv.w);
          Cp[0] = pk2(cv.x, cv.y); Cp[1] = pk2(cv.z, cv.w);
        } else {
          const float4 v = lds_f32x4(row);
          Bp[0] = pk2(v.x, v.y); Cp[0] = pk2(v.z, v.w);
        }
        const f32x2 d2 = pk2(di[i], di[i]), du2 = pk2(dui[i], dui[i]);
        f32x2 acc = pk2(0.0f, 0.0f);
#pragma unroll
        for (int pp = 0; pp < kP; ++pp) {
          float xl, xh;
          upk2(mul2(d2, A2p[pp]), xl, xh);
          const f32x2 a2 = pk2(ex2_approx(xl), ex2_approx(xh));
          hp[pp] = fma2(a2, hp[pp], mul2(du2, Bp[pp]));
          acc = fma2(Cp[pp], hp[pp], acc);
          if constexpr (G > 1) {
            Pp[pp] = mul2(Pp[pp], a2);
            CP[4 * qq + i][pp] = mul2(Cp[pp], Pp[pp]);
          }
        }
        float al, ah;
        upk2(acc, al, ah);
        yq[i] = al + ah;
      }
      if constexpr (G == 1) {
        emit(qq, yq, sk, sz);
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) yl[4 * qq + i] = yq[i];
        skip[qq] = sk;
        szg[qq] = sz;
      }
    }

    // ---- the chain (G > 1): the state entering this block, and this block's end state
    if constexpr (G > 1) {
      const int src_g = g == 0 ? G - 1 : g - 1;
      if (g > 0 || k > 0) {
        const uint32_t par = uint32_t(g == 0 ? k - 1 : k) & 1u;
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&end_ready[src_g * kGroupWarps + w4], par, p.status));
        if (!ok) break;
        const uint32_t sa = sb + uint32_t(S::kSlotOff + ((src_g * kGroupWarps + w4) * 32 + lane) * kS * 4);
        if constexpr (kS == 4) {
          const float4 v = lds_f32x4(sa);
          hin[0] = pk2(v.x, v.y); hin[1] = pk2(v.z, v.w);
        } else {
          const float2 v = lds_v2(sa);
          hin[0] = pk2(v.x, v.y);
        }
      }
      f32x2 endp[kP];
#pragma unroll
      for (int pp = 0; pp < kP; ++pp) endp[pp] = fma2(Pp[pp], hin[pp], hp[pp]);
      // checkpoints (when asked): the blocks that end on a 16-step boundary leave the state
      // entering the next 16-step tile
      if (kCkpt && (R * (g + 1)) % 16 == 0) put_ckpt(tt + R * (g + 1), endp);
      if (g < G - 1 || k < ntiles - 1) {
        const uint32_t da = sb + uint32_t(S::kSlotOff + ((g * kGroupWarps + w4) * 32 + lane) * kS * 4);
        float e[kS];
#pragma unroll
        for (int pp = 0; pp < kP; ++pp) upk2(endp[pp], e[2 * pp], e[2 * pp + 1]);
        if constexpr (kS == 4) sts_v4(da, e[0], e[1], e[2], e[3]);
        else sts_v2(da, e[0], e[1]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&end_ready[g * kGroupWarps + w4]);
      } else {
#pragma unroll
        for (int pp = 0; pp < kP; ++pp) hp[pp] = endp[pp];   // the unit's end state
      }
      // the readouts' share of the carried state, then the outputs
#pragma unroll
      for (int t = 0; t < R; ++t) {
        f32x2 corr = pk2(0.0f, 0.0f);
#pragma unroll
        for (int pp = 0; pp < kP; ++pp) corr = fma2(CP[t][pp], hin[pp], corr);
        float c0, c1;
        upk2(corr, c0, c1);
        yl[t] += c0 + c1;
      }
#pragma unroll
      for (int qq = 0; qq < QG; ++qq) emit(qq, &yl[4 * qq], skip[qq], szg[qq]);
    }

    // ---- the new conv state: the last 3 entries of xpad (x'[L-3..L-1], or the cached
    // window / zeros before the row); with documents, slots older than the last document's
    // first step are zero
    if (g == 0 && j == 0 && k == ntiles - 1 && c == p.nchunks - 1 && p.cs_out && active) {
      bool keep0 = true, keep1 = true;
      if constexpr (kExt) if (p.seq_idx) {
        const bool r1 = (rs >> (p.L - 1 - (tt - 4))) & 1u;   // reset at L-1
        const bool r2 = p.L >= 2 && ((rs >> (p.L - 2 - (tt - 4))) & 1u);   // reset at L-2
        keep1 = !r1;
        keep0 = !r1 && !r2;
      }
      __nv_bfloat16* cso = p.cs_out + (int64_t(b) * p.Di + d) * 3;
#pragma unroll
      for (int i = 0; i < 3; ++i) {
        const int64_t pos = p.L - 3 + i;
        float v;
        if (kExt && pos < 0 && p.cs_in) v = __bfloat162float(p.cs_in[(int64_t(b) * p.Di + d) * 3 + (p.L + i)]);
        else v = bf(lds_u16(st + S::kXOff + swz64(int(pos - (tt - 4)), col)));
        if ((i == 0 && !keep0) || (i == 1 && !keep1)) v = 0.0f;
        cso[i] = __float2bfloat16_rn(v);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  named_bar_sync(0, kThreads);   // pairs with the producer's barrier
  if (!ok || !active || (G > 1 && g != G - 1)) return;
  // the unit's end state: to the next chunk, or out
  float h[kS];
#pragma unroll
  for (int pp = 0; pp < kP; ++pp) upk2(hp[pp], h[2 * pp], h[2 * pp + 1]);
  if (kChained && c < p.nchunks - 1) {
    float* dst = p.carry + (int64_t(tile) * kCh + cl) * N + j * kS;
#pragma unroll
    for (int s = 0; s < kS; ++s) __stcg(dst + s, h[s]);
    __threadfence();
    __syncwarp();
    if (lane == 0) st_release_gpu(p.carry_flag + tile * kGroupWarps + w4, c + 1);
  } else if (c == p.nchunks - 1 && p.h_out) {
    float* ho = p.h_out + (int64_t(b) * p.Di + d) * N + j * kS;
    if constexpr (kS == 4) *reinterpret_cast<float4*>(ho) = make_float4(h[0], h[1], h[2], h[3]);
    else *reinterpret_cast<float2*>(ho) = make_float2(h[0], h[1]);
  }
}

}  // namespace f2
}  // namespace mm
