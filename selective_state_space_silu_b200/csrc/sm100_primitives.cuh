// sm_100a building blocks: mbarriers, TMA tensor loads, bounded waits.
//
// Every wait here is bounded by the GPU's global timer: after kWaitLimitNs without
// progress it records an error code in the caller's status word and reports failure, so
// a kernel can stop cleanly instead of hanging.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace mm {

constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s
constexpr int kStatusTimeout = 6;                               // MAMBA_ERR_TIMEOUT
constexpr int kStatusBadCopy = 7;  // a TMA copy failed its alignment self-check (not issued)

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
               ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// Waits for the phase with `parity` to complete.  Returns false if it has not completed
// within kWaitLimitNs, recording MAMBA_ERR_TIMEOUT in *status (if status is not null).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 63u && global_ns() - t0 > kWaitLimitNs) {
      if (status) atomicExch(status, kStatusTimeout);
      return false;
    }
  }
}

__device__ __forceinline__ void st_release_gpu(int* p, int v) {
  asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Waits until *flag >= value (a flag another CTA of the same grid sets with a release store).
// Bounded like mbar_wait: after kWaitLimitNs records MAMBA_ERR_TIMEOUT and returns false.
__device__ __forceinline__ bool wait_flag_geq(const int* flag, int value, int* status) {
  if (ld_acquire_gpu(flag) >= value) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    __nanosleep(64);
    if (ld_acquire_gpu(flag) >= value) return true;
    if (global_ns() - t0 > kWaitLimitNs) {
      if (status) atomicExch(status, kStatusTimeout);
      return false;
    }
  }
}

// 3-D tiled TMA load (no multicast): coordinates innermost first.  Self-checked: the
// tensor map must be 64-byte aligned, the destination `dst_align`-byte aligned (1024 for
// swizzled tiles, 128 otherwise) and the innermost coordinate times the element size a
// multiple of 16 bytes; a copy that fails a check is not issued and *status records
// kStatusBadCopy (its barrier then times out and the CTA stops cleanly).
__device__ __forceinline__ bool tma_load_3d(uint32_t sdst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, uint32_t dst_align,
                                            int elem_bytes, int* status) {
  const uint64_t gmap = reinterpret_cast<uint64_t>(map);
  if ((sdst & (dst_align - 1)) != 0 || (gmap & 63u) != 0 || ((c0 * elem_bytes) & 15) != 0) {
    atomicExch(status, kStatusBadCopy);
    return false;
  }
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];"
      ::"r"(sdst), "l"(gmap), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
  return true;
}

// Shared-memory accesses by 32-bit shared-window address (always LDS/STS, never generic).
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ float4 lds_f32x4(uint32_t a) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts_f32(uint32_t a, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}

// Packed fp32 pairs (sm_100a f32x2 arithmetic): one instruction, two IEEE fp32 results.
typedef unsigned long long f32x2;
__device__ __forceinline__ f32x2 pk2(float lo, float hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void upk2(f32x2 v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// ---- 5th-generation tensor cores (tcgen05) and tensor memory ----------------------------
// Shared-memory matrix descriptor of a K-major operand in the 128-byte-swizzle layout that a
// TMA copy with CU_TENSOR_MAP_SWIZZLE_128B writes: rows of 128 bytes (64 bf16 of K), 8-row
// atoms of 1024 bytes (the atom must start 1024-byte aligned), the 16-byte chunk index XORed
// with the row index within the atom.  Fields: start address >> 4 (bits 0-13), leading byte
// offset >> 4 (16-29; unused for swizzled K-major, set to 1), stride byte offset >> 4 (32-45:
// 1024 bytes between 8-row atoms), version 1 (46-47), layout 2 = 128-byte swizzle (61-63).
// The K = 16 slice kk of a row starts 32*kk bytes further on.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// Instruction descriptor of tcgen05.mma kind::f16 with bf16 A and B, fp32 D, both K-major:
// D format (bits 4-5) = 1 (f32), A format (7-9) = 1 (bf16), B format (10-12) = 1 (bf16),
// A and B major (15, 16) = 0 (K), N >> 3 (17-22), M >> 4 (24-28).
template <int M, int N>
__host__ __device__ constexpr uint32_t umma_idesc_bf16_f32() {
  static_assert(M == 64 || M == 128, "M = 64 or 128 (cta_group::1)");
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "N a multiple of 16 up to 256");
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, issued by one thread; accumulate = 0 overwrites D.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}
// A shared-memory descriptor split in two 32-bit words: the low word holds the start address
// (bits 0..13, address >> 4) and the leading-dimension offset (bits 16..29); the high word
// the stride offset (1024 bytes: 8 rows of 128 bytes), the sm100 version bit and the
// 128-byte swizzle.  A run of products over consecutive tiles of one operand then adds an
// immediate to the low word (addresses stay below 256 KB, so the 14-bit field never carries).
__device__ __forceinline__ uint32_t umma_desc_lo(uint32_t saddr, uint32_t lbo_bytes) {
  return ((saddr >> 4) & 0x3FFFu) | (((lbo_bytes >> 4) & 0x3FFFu) << 16);
}
constexpr uint32_t kUmmaDescHiSw128 = (1024u >> 4) | (1u << 14) | (2u << 29);
// tcgen05.mma kind::f16 with descriptors given as (a_lo, hi) and (b_lo, hi).
__device__ __forceinline__ void umma_bf16_lo(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "mov.b64 da, {%1, %5};\n\t"
      "mov.b64 db, {%2, %5};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(accumulate), "r"(kUmmaDescHiSw128)
      : "memory");
}
// The mbarrier receives one arrival when every tcgen05.mma this thread issued has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_addr(bar)) : "memory");
}
// Tensor-memory allocation: warp-wide; the column base is written to *dst_smem.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_addr(dst_smem)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// 32 consecutive 32-bit columns of this thread's TMEM lane (the warp's 32-lane quarter):
// thread i of the warp gets lane (32*(warp%4) + i), columns col..col+31 of taddr.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// 16 consecutive 32-bit columns of this thread's TMEM lane (as tmem_ld32).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// The 16x32bx2 shape: threads 0..15 get lanes 32*(warp%4) + i, columns col..col+kW-1;
// threads 16..31 get the same 16 lanes, columns col+kOff..col+kOff+kW-1 (an M = 64
// accumulator keeps its rows in lanes 0..15 of each quarter, so the warp's two halves split
// a row's columns between them).
template <int kOff>
__device__ __forceinline__ void tmem_ld_half16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, "
      "%10, %11, %12, %13, %14, %15}, [%16], %17;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr), "n"(kOff));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
template <int kOff>
__device__ __forceinline__ void tmem_ld_half32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, "
      "%10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, "
      "%27, %28, %29, %30, %31}, [%32], %33;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr), "n"(kOff));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void fence_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// 2-D tiled TMA load (no multicast); same self-checks as tma_load_3d.
__device__ __forceinline__ bool tma_load_2d(uint32_t sdst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, uint32_t dst_align, int elem_bytes,
                                            int* status) {
  const uint64_t gmap = reinterpret_cast<uint64_t>(map);
  if ((sdst & (dst_align - 1)) != 0 || (gmap & 63u) != 0 || ((c0 * elem_bytes) & 15) != 0) {
    atomicExch(status, kStatusBadCopy);
    return false;
  }
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];"
      ::"r"(sdst), "l"(gmap), "r"(smem_addr(bar)), "r"(c0), "r"(c1)
      : "memory");
  return true;
}

// 4-D tiled TMA load (no multicast), self-checked like tma_load_3d.
__device__ __forceinline__ bool tma_load_4d(uint32_t sdst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3, uint32_t dst_align,
                                            int elem_bytes, int* status) {
  const uint64_t gmap = reinterpret_cast<uint64_t>(map);
  if ((sdst & (dst_align - 1)) != 0 || (gmap & 63u) != 0 || ((c0 * elem_bytes) & 15) != 0) {
    atomicExch(status, kStatusBadCopy);
    return false;
  }
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];"
      ::"r"(sdst), "l"(gmap), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
  return true;
}

// Shared-memory matrix descriptor of an MN-major operand in the 128-byte-swizzle layout:
// rows of 128 bytes hold 64 consecutive M (or N) elements of one K index, 8-row atoms of
// 1024 bytes (one atom = 8 consecutive K), atoms along K 1024 bytes apart (stride byte
// offset), 64-wide M/N panels `panel_bytes` apart (leading byte offset).  One K = 16 step of
// the instruction advances the start address by 16 rows = 2048 bytes.
__device__ __forceinline__ uint64_t umma_desc_mn_sw128(uint32_t saddr, uint32_t panel_bytes) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((panel_bytes >> 4) & 0x3FFFu) << 16) |
         (uint64_t(1024 >> 4) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// Instruction descriptor of tcgen05.mma kind::f16 (bf16 A and B, fp32 D) with the operands'
// major-ness: a_mn / b_mn = 1 for MN-major (bits 15, 16).
template <int M, int N, int AMn, int BMn>
__host__ __device__ constexpr uint32_t umma_idesc_bf16_f32_mj() {
  static_assert(M == 64 || M == 128, "M = 64 or 128 (cta_group::1)");
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "N a multiple of 16 up to 256");
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(AMn) << 15) | (uint32_t(BMn) << 16) |
         (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Named barrier that tolerates divergent arrival (non-.aligned form).
__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

}  // namespace mm
