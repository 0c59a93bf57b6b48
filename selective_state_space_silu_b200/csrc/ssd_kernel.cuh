// Mamba2 selective scan (the SSD layer) forward: chunked evaluation on the tensor cores.
//
// The recurrence (niverel-mamba 0.1.0, sections "The weight contract" and "Measured
// tolerances"; the Mamba recurrence of calm-mamba 0.1.4, "Mamba operator", with one
// scalar A, Delta and D per head and one B/C pair per group of heads):
//
//   Delta_t = softplus(dt_raw[t] + dt_bias),  A = -exp(A_log)
//   h[p, n] <- exp(Delta_t A) h[p, n] + Delta_t x_t[p] B_t[n]
//   y_t[p]   = C_t . h[p, :] + D x_t[p]          (times SiLU(z_t[p]) when z is given)
//
// evaluated chunk by chunk (kQ = 64 steps).  With cs_t the in-chunk cumulative sum of
// Delta A (held in log2 units) and H the state entering the chunk:
//
//   Y   = (M o C B^T) x  +  diag(exp(cs)) C H^T  +  D x,   M[t, s] = exp(cs_t - cs_s) Delta_s
//                                                                    for s <= t, else 0
//   H  <- exp(cs_last) H + (w o x)^T B,                  w_s = exp(cs_last - cs_s) Delta_s
//
// (the decay between two steps of a chunk is a difference of that cumulative sum, as the
// pages describe for the reference kernels).  One CTA of 4 warps owns one (batch row,
// head, time segment) and walks the segment's chunks in order; the state H (headdim 64 x
// d_state) stays in the fp32 accumulators of the state GEMM for the whole segment -- it
// never goes to HBM.  Sequences of few (row, head) pairs are cut into segments, each
// started from the earlier ones' end states (see the kernel below); document resets
// (seq_idx) mask the chunk's products.
//
// Work split per chunk (warp w):
//   * M o C B^T: the 10 causal 16 x 16 blocks of the 64 x 64 matrix, 3/3/2/2 per warp,
//     masked and written to shared memory;
//   * the outputs Y for all 64 steps and headdim columns [16w, 16w + 16): the inter-chunk
//     term C H^T takes its B operand straight from this warp's own rows of H (the state
//     GEMM's accumulators hold rows p in [16w, 16w + 16)), then (M o C B^T) x from shared
//     memory;
//   * the state update for rows p in [16w, 16w + 16).
//
// Every product runs on mma.sync m16n8k16 (bf16 operands, fp32 accumulation); operand
// tiles come from shared memory through ldmatrix (XOR-swizzled rows, no bank conflicts).
// The per-chunk tiles (x, B, C) are double-buffered with cp.async: the next chunk's copy
// runs under this chunk's math.
//
// Numerics: the inputs are bf16 and enter the products exactly.  The two fp32
// intermediates that feed the outputs -- H for the inter-chunk term and the masked
// C B^T -- are split into a bf16 pair hi + lo (hi = bf16(v), lo = bf16(v - hi)), so they
// enter the products with a relative error of about 2^-17; only the Delta-weighted x of
// the state update is rounded once to bf16 (relative 2^-9), and it only feeds the state,
// whose own accumulation is fp32.  A single bf16 copy of H measured errors of 3 % of the
// output RMS on outputs that cancel a large carried state.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "device_math.cuh"
#include "sm100_primitives.cuh"

namespace ssd {

constexpr int kP = 64;         // headdim
constexpr int kQ = 64;         // chunk length (steps)
constexpr int kThreads = 128;  // 4 warps

struct SsdArgs {
  const __nv_bfloat16* x;   // [Bt, L, H, P]
  const __nv_bfloat16* dt;  // [Bt, L, H]
  const float* A_log;       // [H]
  const __nv_bfloat16* B;   // [Bt, L, G, N]
  const __nv_bfloat16* C;   // [Bt, L, G, N]
  const float* D;           // [H]
  const float* dt_bias;     // [H]
  const __nv_bfloat16* z;   // [Bt, L, H, P] or null
  const float* h_in;        // [Bt, H, P, N] or null
  const int32_t* seq_idx;   // [Bt, L] or null: the state resets where the id changes
  __nv_bfloat16* y;         // [Bt, L, H, P]
  float* h_out;             // [Bt, H, P, N] or null
  // time segments: CTA z covers chunks [z cps, (z + 1) cps); segments 0 .. nseg - 2 leave
  // their local end state (from zero) and summed Delta A log2 e in the workspace; slot
  // nseg - 1 of ws_H holds a copy of h_in made by the state pass, so that the main pass
  // never reads h_in while its last segment writes h_out (which may be the same buffer)
  float* ws_H;              // [Bt, H, nseg, P, N]
  float* ws_A;              // [Bt, H, nseg - 1]
  int64_t L;
  int H, G;
  int nseg, cps;
};

// Shared memory: two stages of (C, B, x) chunk tiles (B and x only for the state pass),
// then the masked C B^T (hi and lo planes; main pass only), w o x, cs, Delta and the
// in-chunk reset positions.
template <int N, bool kPre>
struct SsdSmem {
  static constexpr int kBC = kQ * N * 2;
  static constexpr int kX = kQ * kP * 2;
  static constexpr int kOffB = kPre ? 0 : kBC;  // within a stage; C at 0 (main pass)
  static constexpr int kOffX = kOffB + kBC;
  static constexpr int kStage = kOffX + kX;
  static constexpr int kG = kPre ? 0 : kQ * kQ * 2;  // one bf16 plane of the 64 x 64 matrix
  static constexpr int kOffGhi = 2 * kStage;
  static constexpr int kOffGlo = kOffGhi + kG;
  static constexpr int kOffXw = kOffGlo + kG;
  static constexpr int kOffCs = kOffXw + kQ * kP * 2;
  static constexpr int kOffDl = kOffCs + kQ * 4;
  static constexpr int kOffRs = kOffDl + kQ * 4;  // int: last reset position <= t, or -1
  static constexpr int kBytes = kOffRs + kQ * 4;
};

// The causal 16 x 16 blocks (t block, s block) of the chunk's 64 x 64 matrix, by warp.
__device__ __forceinline__ void gblock(int warp, int i, int& tb, int& sb) {
  // warp 0: (3,0) (3,1) (0,0); warp 1: (3,2) (3,3) (1,0); warp 2: (2,0) (2,1); warp 3: (2,2) (1,1)
  // as 4-bit fields at position 3 warp + i (no local-memory table)
  constexpr unsigned long long kT = 0x012022133033ull, kS = 0x012010032010ull;
  const int sh = 4 * (3 * warp + i);
  tb = int((kT >> sh) & 0xf);
  sb = int((kS >> sh) & 0xf);
}

// v as a bf16 pair hi + lo with hi = bf16(v) and lo = bf16(v - hi), both packed for two
// adjacent elements.
__device__ __forceinline__ void split_bf16(float v0, float v1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  const float r0 = v0 - __uint_as_float(hi << 16), r1 = v1 - __uint_as_float(hi & 0xffff0000u);
  const __nv_bfloat162 l = __floats2bfloat162_rn(r0, r1);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Byte offset of 16-byte piece k of row r in a tile of R pieces per row (R >= 8): the
// piece index is XORed with the row's low 3 bits, so the 8 rows an ldmatrix reads at one
// column fall in 8 different bank groups.
__device__ __forceinline__ uint32_t swz(int r, int k, int R) {
  return uint32_t((r * R + (k ^ (r & 7))) << 4);
}

__device__ __forceinline__ void ldsm_x4(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(a));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(a));
}

// d += A (16x16, row) * B (16x8, col), bf16 operands, fp32 accumulators.
__device__ __forceinline__ void mma16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two fp32 values as a bf16 pair (round to nearest even); lo in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// 16-byte global -> shared copy; `valid` false fills the 16 bytes with zeros (reads none).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
               ::"r"(dst), "l"(src), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts_u32(uint32_t a, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ uint4 lds_u128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts_u128(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
               ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// Grid (H, Bt, nseg) -- (H, Bt, nseg - 1) for the state pass; kThreads threads;
// SsdSmem<N, kPre>::kBytes of dynamic shared memory.
//
// kPre (state pass): run segment z from a zero state over B and x only and leave its end
// state and its summed Delta A in the workspace.  Main pass: start segment z from h_in
// (zero when absent) folded with the end states of segments 0 .. z - 1,
//   H <- 2^(sum of segment s's Delta A log2 e) H + H_s,
// produce y for the segment's chunks, and (last segment) write h_out.
//
// kSeq (documents, niverel-mamba 0.1.0, section "seq_idx strict reset"): the state is
// zeroed before every step t > 0 whose seq_idx differs from step t - 1's.  With rs_t the
// last reset position <= t inside the chunk (-1 for none): M[t, s] keeps only s >= rs_t,
// the inter-chunk term of step t only when rs_t < 0, the state update only steps
// s >= rs_last, and the carried state decays by 0 instead of 2^cs_last when the chunk holds
// a reset; a segment holding a reset folds with factor 0.
template <int N, bool kGate, bool kPre, bool kSeq>
__global__ void __launch_bounds__(kThreads, kPre ? 4 : 2) ssd_fwd_kernel(const SsdArgs a) {
  using S = SsdSmem<N, kPre>;
  constexpr int R = N / 8;   // 16-byte pieces per row of B and C
  constexpr int NT = N / 8;  // 8-column tiles of the state
  static_assert(N % 16 == 0 && R >= 8, "d_state must be a multiple of 16, at least 64");
  extern __shared__ __align__(128) unsigned char smem[];
  const uint32_t sbase = mm::smem_addr(smem);
  const uint32_t sGhi = sbase + S::kOffGhi, sGlo = sbase + S::kOffGlo, sXw = sbase + S::kOffXw;
  float* cs2 = reinterpret_cast<float*>(smem + S::kOffCs);  // in-chunk cumsum of Delta A log2 e
  float* dls = reinterpret_cast<float*>(smem + S::kOffDl);  // Delta
  int* rsp = reinterpret_cast<int*>(smem + S::kOffRs);      // last reset position <= t, or -1

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tig = lane & 3;  // mma fragment row / column pair
  const int mi = lane >> 3, ri = lane & 7;  // ldmatrix: matrix and row this lane addresses
  const int h = blockIdx.x;
  const int64_t b = blockIdx.y;
  const int seg = blockIdx.z;
  const int grp = h / (a.H / a.G);
  const int64_t L = a.L;
  const int64_t nchunks = (L + kQ - 1) / kQ;
  const int64_t c_begin = int64_t(seg) * a.cps;
  const int64_t c_end = c_begin + a.cps < nchunks ? c_begin + a.cps : nchunks;
  const float A2 = -expf(a.A_log[h]) * mm::kLog2e;  // A log2(e)
  const float bias = a.dt_bias[h];
  const bool has_h_in = !kPre && a.h_in != nullptr;
  const int64_t bh = b * a.H + h;

  // H: rows p0 = 16 warp + g and p0 + 8, columns n = 8 j + 2 tig (+1)
  const int p0 = 16 * warp + g;
  float hacc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) hacc[j][0] = hacc[j][1] = hacc[j][2] = hacc[j][3] = 0.f;
  if constexpr (kPre) {
    if (seg == 0 && a.h_in) {  // the copy of h_in the main pass starts from
      const float* hi = a.h_in + bh * int64_t(kP * N);
      float* hc = a.ws_H + (bh * a.nseg + a.nseg - 1) * int64_t(kP * N);
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        *reinterpret_cast<float2*>(hc + p0 * N + 8 * j + 2 * tig) =
            *reinterpret_cast<const float2*>(hi + p0 * N + 8 * j + 2 * tig);
        *reinterpret_cast<float2*>(hc + (p0 + 8) * N + 8 * j + 2 * tig) =
            *reinterpret_cast<const float2*>(hi + (p0 + 8) * N + 8 * j + 2 * tig);
      }
    }
  } else {
    if (has_h_in) {
      const float* hi = a.nseg > 1 ? a.ws_H + (bh * a.nseg + a.nseg - 1) * int64_t(kP * N)
                                   : a.h_in + bh * int64_t(kP * N);
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        const float2 v0 = *reinterpret_cast<const float2*>(hi + p0 * N + 8 * j + 2 * tig);
        const float2 v1 = *reinterpret_cast<const float2*>(hi + (p0 + 8) * N + 8 * j + 2 * tig);
        hacc[j][0] = v0.x; hacc[j][1] = v0.y; hacc[j][2] = v1.x; hacc[j][3] = v1.y;
      }
    }
    for (int sp = 0; sp < seg; ++sp) {  // fold the end states of the earlier segments
      const float f = mm::ex2_approx(a.ws_A[bh * (a.nseg - 1) + sp]);
      const float* hs = a.ws_H + (bh * a.nseg + sp) * int64_t(kP * N);
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        const float2 v0 = *reinterpret_cast<const float2*>(hs + p0 * N + 8 * j + 2 * tig);
        const float2 v1 = *reinterpret_cast<const float2*>(hs + (p0 + 8) * N + 8 * j + 2 * tig);
        hacc[j][0] = fmaf(f, hacc[j][0], v0.x); hacc[j][1] = fmaf(f, hacc[j][1], v0.y);
        hacc[j][2] = fmaf(f, hacc[j][2], v1.x); hacc[j][3] = fmaf(f, hacc[j][3], v1.y);
      }
    }
  }

  // chunk c's (C,) B and x tiles into stage st; rows past L are zero-filled
  auto load_chunk = [&](int64_t c, int st) {
    const int64_t t0 = c * kQ;
    const uint32_t s0 = sbase + st * S::kStage;
    for (int i = tid; i < kQ * R; i += kThreads) {
      const int r = i / R, k = i % R;
      const int64_t t = t0 + r;
      const bool ok = t < L;
      const int64_t row = ((b * L + (ok ? t : 0)) * a.G + grp) * N + 8 * k;
      if constexpr (!kPre) cp_async16(s0 + swz(r, k, R), a.C + row, ok);
      cp_async16(s0 + S::kOffB + swz(r, k, R), a.B + row, ok);
    }
    for (int i = tid; i < kQ * 8; i += kThreads) {
      const int r = i >> 3, k = i & 7;
      const int64_t t = t0 + r;
      const bool ok = t < L;
      const int64_t row = ((b * L + (ok ? t : 0)) * a.H + h) * kP + 8 * k;
      cp_async16(s0 + S::kOffX + swz(r, k, 8), a.x + row, ok);
    }
    cp_async_commit();
  };
  // warp 0 holds dt_raw (and seq_idx) of steps 2 lane and 2 lane + 1 of the next chunk,
  // and lane 0 the seq_idx of the step before the chunk
  float dtn0 = 0.f, dtn1 = 0.f;
  int32_t idn0 = 0, idn1 = 0, idp = 0;
  auto load_dt = [&](int64_t c) {
    const int64_t t = c * kQ + 2 * lane;
    dtn0 = t < L ? __bfloat162float(a.dt[(b * L + t) * a.H + h]) : 0.f;
    dtn1 = t + 1 < L ? __bfloat162float(a.dt[(b * L + t + 1) * a.H + h]) : 0.f;
    if constexpr (kSeq) {
      const int32_t* ids = a.seq_idx + b * L;
      idn0 = t < L ? ids[t] : 0;
      idn1 = t + 1 < L ? ids[t + 1] : 0;
      if (lane == 0) idp = c > 0 ? ids[c * kQ - 1] : idn0;
    }
  };

  float seg_a = 0.f;  // state pass: summed Delta A log2 e of the segment
  if (c_begin < c_end) {
    load_chunk(c_begin, 0);
    if (warp == 0) load_dt(c_begin);
  }
  for (int64_t c = c_begin; c < c_end; ++c) {
    const int st = int((c - c_begin) & 1);
    const int64_t t0 = c * kQ;
    const uint32_t sC = sbase + st * S::kStage, sB = sC + S::kOffB, sX = sC + S::kOffX;
    const bool has_state = c > 0 || has_h_in;
    cp_async_wait_all();
    __syncthreads();  // this chunk's tiles are in; every warp is done with the previous chunk
    if (c + 1 < c_end) load_chunk(c + 1, st ^ 1);

    // Delta and the inclusive cumulative sum of Delta A (log2 units) over the chunk
    if (warp == 0) {
      const int64_t t = t0 + 2 * lane;
      const float d0 = t < L ? mm::Math<false>::softplus(dtn0 + bias) : 0.f;
      const float d1 = t + 1 < L ? mm::Math<false>::softplus(dtn1 + bias) : 0.f;
      if constexpr (kSeq) {
        // reset flags of steps 2 lane, 2 lane + 1 (none past L, none at t = 0), then the
        // last reset position <= t by a max-scan over the lanes
        const int32_t i0 = idn0, i1 = idn1;
        const int32_t prev = __shfl_up_sync(0xffffffffu, i1, 1);
        const bool r0 = t < L && (lane == 0 ? (t > 0 && i0 != idp) : i0 != prev);
        const bool r1 = t + 1 < L && i1 != i0;
        int m = r1 ? 2 * lane + 1 : (r0 ? 2 * lane : -1);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, m, o);
          if (lane >= o) m = max(m, v);
        }
        int mex = __shfl_up_sync(0xffffffffu, m, 1);
        if (lane == 0) mex = -1;
        const int rs0 = r0 ? 2 * lane : mex;
        rsp[2 * lane] = rs0;
        rsp[2 * lane + 1] = r1 ? 2 * lane + 1 : rs0;
      }
      if (c + 1 < c_end) load_dt(c + 1);
      const float e0 = d0 * A2, e1 = d1 * A2;
      float s = e0 + e1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float v = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += v;
      }
      float ex = __shfl_up_sync(0xffffffffu, s, 1);
      if (lane == 0) ex = 0.f;
      cs2[2 * lane] = ex + e0;
      cs2[2 * lane + 1] = ex + e0 + e1;
      dls[2 * lane] = d0;
      dls[2 * lane + 1] = d1;
    }

    // before Delta is known: this warp's causal blocks of C B^T and the inter-chunk term
    // C H^T for headdim columns [16 warp, 16 warp + 16), H's B operand (hi + lo) taken from
    // this warp's own state rows
    const int nblk = warp < 2 ? 3 : 2;
    float gacc[3][2][4];
    float yacc[4][2][4];
    if constexpr (!kPre) {
#pragma unroll
      for (int i = 0; i < 3; ++i) {
#pragma unroll
        for (int j = 0; j < 2; ++j) gacc[i][j][0] = gacc[i][j][1] = gacc[i][j][2] = gacc[i][j][3] = 0.f;
        if (i < nblk) {
          int tb, sb;
          gblock(warp, i, tb, sb);
#pragma unroll
          for (int kk = 0; kk < N / 16; ++kk) {
            uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
            ldsm_x4(sC + swz(16 * tb + (mi & 1) * 8 + ri, 2 * kk + (mi >> 1), R), a0, a1, a2, a3);
            ldsm_x4(sB + swz(16 * sb + (mi >> 1) * 8 + ri, 2 * kk + (mi & 1), R), b0, b1, b2, b3);
            mma16816(gacc[i][0], a0, a1, a2, a3, b0, b1);
            mma16816(gacc[i][1], a0, a1, a2, a3, b2, b3);
          }
        }
      }
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int np = 0; np < 2; ++np) yacc[mt][np][0] = yacc[mt][np][1] = yacc[mt][np][2] = yacc[mt][np][3] = 0.f;
      if (has_state) {
#pragma unroll
        for (int kk = 0; kk < N / 16; ++kk) {
          uint32_t bhi[2][2], blo[2][2];
#pragma unroll
          for (int np = 0; np < 2; ++np) {
            split_bf16(hacc[2 * kk][2 * np], hacc[2 * kk][2 * np + 1], bhi[np][0], blo[np][0]);
            split_bf16(hacc[2 * kk + 1][2 * np], hacc[2 * kk + 1][2 * np + 1], bhi[np][1], blo[np][1]);
          }
#pragma unroll
          for (int mt = 0; mt < 4; ++mt) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(sC + swz(16 * mt + (mi & 1) * 8 + ri, 2 * kk + (mi >> 1), R), a0, a1, a2, a3);
            mma16816(yacc[mt][0], a0, a1, a2, a3, bhi[0][0], bhi[0][1]);
            mma16816(yacc[mt][1], a0, a1, a2, a3, bhi[1][0], bhi[1][1]);
          }
#pragma unroll
          for (int mt = 0; mt < 4; ++mt) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(sC + swz(16 * mt + (mi & 1) * 8 + ri, 2 * kk + (mi >> 1), R), a0, a1, a2, a3);
            mma16816(yacc[mt][0], a0, a1, a2, a3, blo[0][0], blo[0][1]);
            mma16816(yacc[mt][1], a0, a1, a2, a3, blo[1][0], blo[1][1]);
          }
        }
      }
    }
    __syncthreads();  // cs2 and dls visible

    const float csl = cs2[kQ - 1];
    const int rsl = kSeq ? rsp[kQ - 1] : -1;  // last reset in the chunk
    if constexpr (kPre) seg_a = rsl >= 0 ? -INFINITY : seg_a + csl;
    // w o x for the state update: w_s = 2^(cs2_last - cs2_s) Delta_s (0 before a reset)
    for (int i = tid; i < kQ * 8; i += kThreads) {
      const int r = i >> 3, k = i & 7;
      const uint32_t off = swz(r, k, 8);
      const float w = r >= rsl ? mm::ex2_approx(csl - cs2[r]) * dls[r] : 0.f;
      const uint4 v = lds_u128(sX + off);
      uint4 o;
      o.x = pack_bf16(w * bf16_lo(v.x), w * bf16_hi(v.x));
      o.y = pack_bf16(w * bf16_lo(v.y), w * bf16_hi(v.y));
      o.z = pack_bf16(w * bf16_lo(v.z), w * bf16_hi(v.z));
      o.w = pack_bf16(w * bf16_lo(v.w), w * bf16_hi(v.w));
      sts_u128(sXw + off, o);
    }

    if constexpr (!kPre) {
      // mask the blocks: M[t, s] = 2^(cs2_t - cs2_s) Delta_s for s <= t; hi / lo planes [t][s]
#pragma unroll
      for (int i = 0; i < 3; ++i) {
        if (i < nblk) {
          int tb, sb;
          gblock(warp, i, tb, sb);
          const int t0r = 16 * tb + g, t1r = t0r + 8;
          const float ct0 = cs2[t0r], ct1 = cs2[t1r];
          const int lo0 = kSeq ? rsp[t0r] : 0, lo1 = kSeq ? rsp[t1r] : 0;  // same document: s >= lo
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int s0 = 16 * sb + 8 * j + 2 * tig, s1 = s0 + 1;
            const float cs0 = cs2[s0], cs1 = cs2[s1], w0 = dls[s0], w1 = dls[s1];
            const float v00 = s0 <= t0r && s0 >= lo0 ? gacc[i][j][0] * mm::ex2_approx(ct0 - cs0) * w0 : 0.f;
            const float v01 = s1 <= t0r && s1 >= lo0 ? gacc[i][j][1] * mm::ex2_approx(ct0 - cs1) * w1 : 0.f;
            const float v10 = s0 <= t1r && s0 >= lo1 ? gacc[i][j][2] * mm::ex2_approx(ct1 - cs0) * w0 : 0.f;
            const float v11 = s1 <= t1r && s1 >= lo1 ? gacc[i][j][3] * mm::ex2_approx(ct1 - cs1) * w1 : 0.f;
            uint32_t hi, lo;
            split_bf16(v00, v01, hi, lo);
            sts_u32(sGhi + swz(t0r, 2 * sb + j, 8) + 4 * tig, hi);
            sts_u32(sGlo + swz(t0r, 2 * sb + j, 8) + 4 * tig, lo);
            split_bf16(v10, v11, hi, lo);
            sts_u32(sGhi + swz(t1r, 2 * sb + j, 8) + 4 * tig, hi);
            sts_u32(sGlo + swz(t1r, 2 * sb + j, 8) + 4 * tig, lo);
          }
        }
      }
      if (has_state) {  // the inter-chunk term decays by 2^cs2_t at step t (0 after a reset)
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          const int ta = 16 * mt + g, tb2 = ta + 8;
          const float e0 = (!kSeq || rsp[ta] < 0) ? mm::ex2_approx(cs2[ta]) : 0.f;
          const float e1 = (!kSeq || rsp[tb2] < 0) ? mm::ex2_approx(cs2[tb2]) : 0.f;
#pragma unroll
          for (int np = 0; np < 2; ++np) {
            yacc[mt][np][0] *= e0; yacc[mt][np][1] *= e0; yacc[mt][np][2] *= e1; yacc[mt][np][3] *= e1;
          }
        }
      }
    }
    __syncthreads();  // M o C B^T and w o x visible

    if constexpr (!kPre) {
      // Y += (M o C B^T) x for s blocks kb <= t block mt
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
          if (kb <= mt) {
            uint32_t h0, h1, h2, h3, l0, l1, l2, l3, b0, b1, b2, b3;
            const uint32_t ga = swz(16 * mt + (mi & 1) * 8 + ri, 2 * kb + (mi >> 1), 8);
            ldsm_x4(sGhi + ga, h0, h1, h2, h3);
            ldsm_x4(sGlo + ga, l0, l1, l2, l3);
            ldsm_x4_t(sX + swz(16 * kb + (mi & 1) * 8 + ri, 2 * warp + (mi >> 1), 8), b0, b1, b2, b3);
            mma16816(yacc[mt][0], h0, h1, h2, h3, b0, b1);
            mma16816(yacc[mt][1], h0, h1, h2, h3, b2, b3);
            mma16816(yacc[mt][0], l0, l1, l2, l3, b0, b1);
            mma16816(yacc[mt][1], l0, l1, l2, l3, b2, b3);
          }
        }
      }

      // out = (Y + D x) [* SiLU(z)], bf16 pairs at (t = 16 mt + g (+8), p = 16 warp + 8 np + 2 tig)
      const float Dh = a.D[h];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int tr = 16 * mt + g + 8 * hf;
          const int64_t t = t0 + tr;
          if (t < L) {
            const int64_t row = ((b * L + t) * a.H + h) * kP;
#pragma unroll
            for (int np = 0; np < 2; ++np) {
              const int p = 16 * warp + 8 * np + 2 * tig;
              const uint32_t xv = lds_u32(sX + swz(tr, 2 * warp + np, 8) + 4 * tig);
              float o0 = yacc[mt][np][2 * hf] + Dh * bf16_lo(xv);
              float o1 = yacc[mt][np][2 * hf + 1] + Dh * bf16_hi(xv);
              if constexpr (kGate) {
                const uint32_t zv = *reinterpret_cast<const uint32_t*>(a.z + row + p);
                o0 *= mm::Math<false>::silu(bf16_lo(zv));
                o1 *= mm::Math<false>::silu(bf16_hi(zv));
              }
              *reinterpret_cast<uint32_t*>(a.y + row + p) = pack_bf16(o0, o1);
            }
          }
        }
      }
    }

    // H <- 2^cs2_last H + (w o x)^T B   (rows p of this warp, all n)
    const float dec = rsl < 0 ? mm::ex2_approx(csl) : 0.f;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      hacc[j][0] *= dec; hacc[j][1] *= dec; hacc[j][2] *= dec; hacc[j][3] *= dec;
    }
#pragma unroll
    for (int kk = 0; kk < kQ / 16; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4_t(sXw + swz(16 * kk + (mi >> 1) * 8 + ri, 2 * warp + (mi & 1), 8), a0, a1, a2, a3);
#pragma unroll
      for (int jp = 0; jp < NT / 2; ++jp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sB + swz(16 * kk + (mi & 1) * 8 + ri, 2 * jp + (mi >> 1), R), b0, b1, b2, b3);
        mma16816(hacc[2 * jp], a0, a1, a2, a3, b0, b1);
        mma16816(hacc[2 * jp + 1], a0, a1, a2, a3, b2, b3);
      }
    }
  }

  float* out = nullptr;
  if constexpr (kPre) {
    out = a.ws_H + (bh * a.nseg + seg) * int64_t(kP * N);
    if (tid == 0) a.ws_A[bh * (a.nseg - 1) + seg] = seg_a;
  } else {
    if (seg == a.nseg - 1) out = a.h_out;
    if (out) out += bh * int64_t(kP * N);
  }
  if (out) {
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      *reinterpret_cast<float2*>(out + p0 * N + 8 * j + 2 * tig) = make_float2(hacc[j][0], hacc[j][1]);
      *reinterpret_cast<float2*>(out + (p0 + 8) * N + 8 * j + 2 * tig) = make_float2(hacc[j][2], hacc[j][3]);
    }
  }
}

}  // namespace ssd
