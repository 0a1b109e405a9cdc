// Device helpers shared by the kernels of the routed int4 expert layer.
// Inline PTX follows the public PTX ISA (mbarrier, cp.async.bulk, ldmatrix,
// mma.sync, lop3, griddepcontrol, tcgen05).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "layer.h"

namespace strata {

// ---------------------------------------------------------------- status word
__device__ __forceinline__ void set_status(int *status, int bit) {
  if (status) atomicOr(status, bit);
}

// ---------------------------------------------------------------- addresses
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Wait for the barrier phase, backing off with nanosleep between polls (for
// waits off the critical path, e.g. a producer waiting for a free stage).
__device__ __forceinline__ bool mbar_wait_sleepy(uint64_t *bar, uint32_t parity, int *status) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = global_timer_ns();
  unsigned ns = 32;
  while (true) {
    __nanosleep(ns);
    if (ns < 256) ns <<= 1;
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      set_status(status, STATUS_TIMEOUT);
      return false;
    }
  }
}

// try_wait with a suspend-time hint: the thread sleeps until the phase
// completes or about 1 ms passes, instead of spinning.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 1000000;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the barrier phase with a time limit.  On timeout the status word
// gets STATUS_TIMEOUT and the caller must stop waiting and wind down.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int *status) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      set_status(status, STATUS_TIMEOUT);
      return false;
    }
  }
}

// ---------------------------------------------------------------- bulk copy
// Plain (non-multicast) bulk copy global -> this CTA's shared memory; the
// completion is counted on `bar` as transaction bytes.  Both addresses and
// the size must be multiples of 16 bytes.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------- PDL
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dependency_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- loads
__device__ __forceinline__ uint32_t ld_nc_u32(const void *p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

// ---------------------------------------------------------------- tensor core (legacy)
__device__ __forceinline__ void ldmatrix_x4(uint32_t r[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// D = A * B + C, A 16x16 f16 (row), B 16x8 f16 (col), C/D 16x8 f32.
// (Not volatile: it has no side effects, so the compiler may interleave
// independent MMAs.)
__device__ __forceinline__ void mma_16816(float d[4], const uint32_t a[4], uint32_t b0,
                                          uint32_t b1, const float c[4]) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]),
        "f"(c[2]), "f"(c[3]));
}

// (a & b) ^ c in one instruction.
__device__ __forceinline__ uint32_t and_xor(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t h2_bits(__half2 v) { return *reinterpret_cast<uint32_t *>(&v); }
__device__ __forceinline__ __half2 bits_h2(uint32_t v) { return *reinterpret_cast<__half2 *>(&v); }

// Eight int4 values packed in one 32-bit word (element e in bits 4e..4e+3,
// two's complement) -> four f16x2 registers holding the exact integers
//   out[0] = (q0, q4), out[1] = (q1, q5), out[2] = (q2, q6), out[3] = (q3, q7)
// (low half first).  A nibble n with its sign bit flipped is n' = q + 8 in
// [0, 15]; OR-ing it into the mantissa of 1024.0 gives 1024 + n' (low nibble
// position) or 1024 + 16 n' (next nibble position), both exact in f16, and
// one f16 subtract (or multiply-add by 1/16) recovers q exactly.
__device__ __forceinline__ void int4x8_to_f16(uint32_t w, uint32_t out[4]) {
  const uint32_t w8 = w >> 8;
  const uint32_t a = and_xor(w, 0x000F000Fu, 0x64086408u);
  const uint32_t b = and_xor(w, 0x00F000F0u, 0x64806480u);
  const uint32_t c = and_xor(w8, 0x000F000Fu, 0x64086408u);
  const uint32_t d = and_xor(w8, 0x00F000F0u, 0x64806480u);
  const __half2 k1032 = __half2half2(__ushort_as_half(0x6408));    // 1032.0
  const __half2 k1_16 = __half2half2(__ushort_as_half(0x2C00));    // 1/16
  const __half2 km72 = __half2half2(__ushort_as_half(0xD480));     // -72.0
  out[0] = h2_bits(__hsub2(bits_h2(a), k1032));
  out[1] = h2_bits(__hfma2(bits_h2(b), k1_16, km72));
  out[2] = h2_bits(__hsub2(bits_h2(c), k1032));
  out[3] = h2_bits(__hfma2(bits_h2(d), k1_16, km72));
}

}  // namespace strata
