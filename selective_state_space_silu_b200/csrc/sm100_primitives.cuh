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

// Named barrier that tolerates divergent arrival (non-.aligned form).
__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

}  // namespace mm
