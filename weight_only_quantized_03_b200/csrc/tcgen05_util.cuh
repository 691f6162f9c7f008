// tcgen05 / mbarrier helpers shared by the tensor-core GEMMs (sm_100a).
#pragma once

#include <cuda.h>  // CUtensorMap

#include "qg_internal.cuh"

namespace qg {

// Host: a TMA descriptor of a bf16 [rows][cols] row-major tensor in boxes of
// 64 columns x box_rows rows with 128-byte swizzle (rows past the end read as
// zero); false when the driver's encoder is unavailable or refuses it.
bool make_bf16_map(CUtensorMap* map, const void* base, int rows, int cols, int box_rows);
// Host: a TMA descriptor of a byte [rows][cols] row-major tensor (cols a
// multiple of 16) in boxes of box_cols x box_rows, no swizzle or (with
// swizzle128 and box_cols = 128) the 128-byte swizzle.
bool make_u8_map(CUtensorMap* map, const void* base, int rows, int cols, int box_cols,
                 int box_rows, bool swizzle128 = false);

namespace tc {

constexpr unsigned long long kWaitNs = 1000000000ull;  // every device-side wait gives up after 1 s

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// try_wait that may suspend the thread up to hint_ns (it resumes as soon as
// the phase completes), so a waiting role sleeps instead of spinning
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity,
                                                   uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
// bounded wait (limit_ns); gives up early once another role has aborted
__device__ __forceinline__ bool wait_bar_ns(uint64_t* bar, uint32_t parity, volatile int* abort,
                                            unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = now_ns();
  while (!mbar_try_wait_hint(bar, parity, 20000u)) {
    if (*abort) return false;
    if (now_ns() - t0 > limit_ns) return false;
  }
  return true;
}
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort) {
  return wait_bar_ns(bar, parity, abort, kWaitNs);
}

// K-major, 128-byte swizzle shared-memory matrix descriptor: 8-row groups
// 1024 bytes apart (SBO), leading offset 16 bytes, descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;             // LBO = 16 B (encoded >> 4)
  d |= (uint64_t)(1024u >> 4) << 32;   // SBO = 1024 B
  d |= (uint64_t)1u << 46;             // version
  d |= (uint64_t)2u << 61;             // SWIZZLE_128B
  return d;
}

// instruction descriptor: fp16 x fp16 -> fp32, both K-major, M = 128
template <int BN>
__host__ __device__ constexpr uint32_t instr_desc_f16() {
  return (1u << 4)                 // D fp32 (A, B fp16: format 0)
         | ((uint32_t)(BN >> 3) << 17)
         | ((uint32_t)(128 >> 4) << 24);
}

// instruction descriptor: bf16 x bf16 -> fp32, both K-major, M = 128
template <int BN>
__host__ __device__ constexpr uint32_t instr_desc() {
  return (1u << 4)                 // D fp32
         | (1u << 7)               // A bf16
         | (1u << 10)              // B bf16
         | ((uint32_t)(BN >> 3) << 17)
         | ((uint32_t)(128 >> 4) << 24);
}

}  // namespace tc
}  // namespace qg
