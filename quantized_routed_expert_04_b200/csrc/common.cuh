// Device helpers shared by the kernels of the routed int4 expert layer.
// Inline PTX follows the public PTX ISA (mbarrier, cp.async.bulk, ldmatrix,
// mma.sync, lop3, griddepcontrol, tcgen05).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "layer.h"

namespace strata {

// ---------------------------------------------------------------- status word
__device__ __forceinline__ void set_status(int *status, int bit) {
  if (status) atomicOr(status, bit);
}

// Eight bf16 activations -> eight f16, in the order in which the format's
// weight conversion produces weight pairs (so that one 16-byte load gives a
// thread its four mma B-fragment registers): 0,4,1,5,2,6,3,7 for int4
// (int4x8_to_f16), 0..7 for NVFP4 (e2m1x8_to_f16).  Sets `overflow` if an
// input rounds to an f16 infinity.
template <int FMT>
__device__ __forceinline__ uint4 pack8_bf16_to_f16(uint4 raw, bool &overflow) {
  const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&raw);
  const float2 f0 = __bfloat1622float2(b[0]), f1 = __bfloat1622float2(b[1]);
  const float2 f2 = __bfloat1622float2(b[2]), f3 = __bfloat1622float2(b[3]);
  const float m = fmaxf(fmaxf(fmaxf(fabsf(f0.x), fabsf(f0.y)), fmaxf(fabsf(f1.x), fabsf(f1.y))),
                        fmaxf(fmaxf(fabsf(f2.x), fabsf(f2.y)), fmaxf(fabsf(f3.x), fabsf(f3.y))));
  overflow = m >= kF16Overflow;
  uint4 o;
  __half2 h;
  if (FMT == kFmtInt4) {
    h = __floats2half2_rn(f0.x, f2.x); o.x = *reinterpret_cast<uint32_t *>(&h);
    h = __floats2half2_rn(f0.y, f2.y); o.y = *reinterpret_cast<uint32_t *>(&h);
    h = __floats2half2_rn(f1.x, f3.x); o.z = *reinterpret_cast<uint32_t *>(&h);
    h = __floats2half2_rn(f1.y, f3.y); o.w = *reinterpret_cast<uint32_t *>(&h);
  } else {
    h = __floats2half2_rn(f0.x, f0.y); o.x = *reinterpret_cast<uint32_t *>(&h);
    h = __floats2half2_rn(f1.x, f1.y); o.y = *reinterpret_cast<uint32_t *>(&h);
    h = __floats2half2_rn(f2.x, f2.y); o.z = *reinterpret_cast<uint32_t *>(&h);
    h = __floats2half2_rn(f3.x, f3.y); o.w = *reinterpret_cast<uint32_t *>(&h);
  }
  return o;
}

// Position of element i (of a row of packed 16-bit activations or SwiGLU
// outputs) in the format's pair order (see pack8_bf16_to_f16).
template <int FMT>
__device__ __forceinline__ int packed_pos(int i) {
  return FMT == kFmtInt4 ? (i & ~7) | (((i & 3) << 1) | ((i >> 2) & 1)) : i;
}

// Eight E2M1 codes in one 32-bit word (code e in bits 4e..4e+3) -> four
// f16x2 registers holding their exact values: out[j] = (code 2j, code 2j+1),
// low half first (the conversion instruction of sm_100a, one per byte).
__device__ __forceinline__ void e2m1x8_to_f16(uint32_t w, uint32_t out[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
      : "r"(w));
}

// One E4M3 byte (the low byte of `byte`) -> f16x2 holding its exact value
// twice.
__device__ __forceinline__ uint32_t e4m3_to_f16x2_dup(uint32_t byte) {
  const uint16_t v = (uint16_t)((byte & 0xFFu) * 0x101u);
  uint32_t d;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"(v));
  return d;
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

// Read-only global loads that bypass L1 allocation (data read once per SM).
__device__ __forceinline__ uint4 ldg_nc_v4(const void *ptr) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(ptr));
  return v;
}
__device__ __forceinline__ uint2 ldg_nc_v2(const void *ptr) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(ptr));
  return v;
}

// ---------------------------------------------------------------- bulk copy
// Hint: bring `bytes` (a multiple of 16, 16-byte aligned source) into L2 ahead
// of the copies that will read them; no completion to wait for.
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

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
// (low half first).  This is the published magic-number conversion of
// low-bit integers to f16 with one lop3 per pair (Kim et al., "Who Says
// Elephants Can't Run: Bringing Large Scale MoE Models into Cloud Scale
// Production", 2022), here in a two's-complement form: a nibble n with its
// sign bit flipped is n' = q + 8 in [0, 15]; the same lop3 that masks it ORs
// it into the mantissa of 1024.0 and flips the sign bit, giving 1024 + n'
// (low nibble position) or 1024 + 16 n' (next nibble position), both exact
// in f16, and one f16 subtract (or multiply-add by 1/16) recovers q exactly.
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


// ---------------------------------------------------------------- TMA (tiled)
// 2D tiled load (no multicast) into this CTA's shared memory; completion in
// transaction bytes on `bar`.  c0 is the innermost coordinate.
__device__ __forceinline__ void tma_load_2d(void *dst, const void *tmap, int c0, int c1,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const void *tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// ---------------------------------------------------------------- tcgen05
// Shared-memory matrix descriptor for a K-major operand in the 128-byte
// swizzle layout: rows of 128 bytes, 8-row groups 1024 bytes apart (stride
// byte offset), descriptor version 1, base offset 0 (the tile starts on a
// 1024-byte boundary; per-k16 steps inside the 128-byte row add 32 bytes to
// the start address).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);          // start address
  d |= (uint64_t)(1) << 16;                             // leading byte offset (unused)
  d |= (uint64_t)(1024 >> 4) << 32;                     // stride byte offset
  d |= (uint64_t)1 << 46;                               // version
  d |= (uint64_t)2 << 61;                               // 128-byte swizzle
  return d;
}

// Instruction descriptor of kind::f16 with f16 A and B (both K-major) and an
// f32 accumulator, shape M x N.
__device__ __forceinline__ uint32_t umma_idesc_f16(int M, int N) {
  return (1u << 4)                       // D format f32
         | (0u << 7) | (0u << 10)        // A, B format f16
         | ((uint32_t)(N >> 3) << 17)    // N / 8
         | ((uint32_t)(M >> 4) << 24);   // M / 16
}

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once all earlier tcgen05.mma of this thread have completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
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

// 32 consecutive accumulator columns of this warp's 32 TMEM lanes: thread
// lane l gets row (lane base + l), columns col .. col + 31.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, float v[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor core, bulk copies) before it signals them.
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

}  // namespace strata
