// umma.cuh -- the tcgen05 (5th-generation tensor core) pieces the prefill-chunk projections
// share, for sm_100a: shared-memory operand descriptors, the bf16 instruction descriptor, the
// MMA and its commit, tensor-memory loads and the tcgen05 thread-sync fences.
//
// Operand layout used throughout: K-major with the 128-byte swizzle, 8-row groups 1024 bytes
// apart (the layout a 2-D TMA copy with a 64-column bf16 box and SWIZZLE_128B writes, and
// the one the bases are transposed into by hand); M = 128 rows per MMA, N a multiple of 16 up
// to 256, K = 16 per instruction.
#pragma once

#include <cstdint>

#include "stief_device.cuh"

namespace stief {

constexpr int kUmmaRows = 128;  // M of every MMA here

// UMMA shared-memory descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);  // start address
  d |= (uint64_t)1u << 16;                      // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024u >> 4) << 32;            // stride byte offset
  d |= (uint64_t)1u << 46;                      // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;                      // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor: bf16 x bf16 -> fp32, A and B K-major, M = 128, N = n.
__device__ __forceinline__ uint32_t idesc_bf16_f32(int n) {
  return (1u << 4)                      // D format: f32
         | (1u << 7)                    // A format: bf16
         | (1u << 10)                   // B format: bf16
         | ((uint32_t)(n >> 3) << 17)   // N / 8
         | ((uint32_t)(kUmmaRows >> 4) << 24);  // M / 16
}

// D[tmem] (+)= A . B^T over K = 16; accumulate = 0 overwrites D.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// One arrival on `bar` once every tcgen05 operation this thread issued before has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 16 consecutive fp32 columns of the warp's 32 TMEM lanes (lane i reads lane base + i).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, "
      "[%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Warp-wide: allocate `cols` TMEM columns (a power of two >= 32), base address into *slot.
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot)),
               "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(cols)
               : "memory");
}

// Byte offset of element k (0..127) of row n in a K-major SW128 operand of 128-byte rows
// split into two 64-column atoms `atom_bytes` apart: 16-byte chunk (k % 64) / 8 of row n is
// stored at chunk position ((k % 64) / 8) ^ (n % 8).
__device__ __forceinline__ uint32_t sw128_offset(int n, int k, uint32_t atom_bytes) {
  const uint32_t kb = (uint32_t)(k & 63) * 2u;
  return (uint32_t)(k >> 6) * atom_bytes + (uint32_t)n * 128u +
         ((((kb >> 4) ^ (uint32_t)(n & 7)) << 4) | (kb & 15u));
}

// bf16 RNE of 16 fp32 accumulators, stored as 32 contiguous bytes at dst (16-byte aligned).
__device__ __forceinline__ void store_bf16x16(uint16_t* dst, const uint32_t (&v)[16]) {
  uint4 lo, hi;
  lo.x = pack_bf16x2_rn(__uint_as_float(v[0]), __uint_as_float(v[1]));
  lo.y = pack_bf16x2_rn(__uint_as_float(v[2]), __uint_as_float(v[3]));
  lo.z = pack_bf16x2_rn(__uint_as_float(v[4]), __uint_as_float(v[5]));
  lo.w = pack_bf16x2_rn(__uint_as_float(v[6]), __uint_as_float(v[7]));
  hi.x = pack_bf16x2_rn(__uint_as_float(v[8]), __uint_as_float(v[9]));
  hi.y = pack_bf16x2_rn(__uint_as_float(v[10]), __uint_as_float(v[11]));
  hi.z = pack_bf16x2_rn(__uint_as_float(v[12]), __uint_as_float(v[13]));
  hi.w = pack_bf16x2_rn(__uint_as_float(v[14]), __uint_as_float(v[15]));
  *reinterpret_cast<uint4*>(dst) = lo;
  *reinterpret_cast<uint4*>(dst + 8) = hi;
}

}  // namespace stief
