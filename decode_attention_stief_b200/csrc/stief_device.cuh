// stief_device.cuh -- sm_100a device helpers shared by the library's kernels:
// mbarriers, bulk (TMA-engine) copies, programmatic dependent launch, bounded
// waits and bf16 packing.  Inline PTX only; no CUTLASS.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "stief.h"

namespace stief {

// ---------------------------------------------------------------------------- addresses

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------- status word

__device__ __forceinline__ void report(uint32_t* dev_status, uint32_t bits) {
  if (dev_status != nullptr) atomicOr(dev_status, bits);
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// A bounded wait gives up after this long (nanoseconds of the global timer).  The test build
// (STIEF_TEST_HOOKS, a separate library used only by the timeout tests) gives up sooner.
#ifdef STIEF_TEST_HOOKS
constexpr uint64_t kWaitLimitNs = 50000000ull;  // 50 ms
#else
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
#endif

// ---------------------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Make barrier initialisation visible to the asynchronous (TMA / tensor core) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// Plain arrival (count 1) on a barrier.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// One bounded-time wait: the thread may be suspended in hardware (up to about
// kSuspendHintNs) until the phase completes, instead of spinning on issue slots.
constexpr uint32_t kSuspendHintNs = 1000000u;  // 1 ms

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// Non-blocking test: has the phase with the given parity completed?
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete.  Returns false (and
// reports STIEF_DEV_WAIT_TIMEOUT) if it has not completed within kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint32_t* dev_status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      report(dev_status, STIEF_DEV_WAIT_TIMEOUT);
      return false;
    }
  }
  return true;
}

// ---------------------------------------------------------------------------- bulk copies

// 1-D bulk copy global -> shared through the TMA engine; completion is counted
// in bytes on `bar`.  dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Same, with an L2 eviction-priority hint (for data streamed exactly once).
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes,
                                              uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// For data many CTAs read (kept in L2 in preference to streamed data).
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 1-D bulk copy shared -> global (completion tracked with bulk groups).
__device__ __forceinline__ void bulk_s2g(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until all committed bulk stores have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until all committed bulk stores are complete (writes visible).
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// 2-D TMA tensor copy global -> shared of the box at column x, row y of `map`
// (a __grid_constant__ kernel parameter); completion counted in bytes on `bar`.
// x * element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* map, int x, int y,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Bring a tensor map (a __grid_constant__ kernel parameter) into the TMA unit's cache.
__device__ __forceinline__ void prefetch_tensormap(const void* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// ---------------------------------------------------------------------------- named barriers

// Hardware barrier `id` (1..15; 0 is __syncthreads) among `count` threads (a multiple of 32):
// wait for all of them, or arrive without waiting.
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void named_bar_arrive(int id, int count) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ---------------------------------------------------------------------------- PDL

// Block until the preceding grid in the stream has completed and its memory is
// visible (no-op when the kernel was not launched as a programmatic dependent).
// Row of token t of (sequence b, KV head h) in a latent cache.  Contiguous caches hold
// [B][Hkv][L_max] rows; paged caches hold [num_pages][Hkv][page_size] rows and map token t
// through the sequence's block table (page block_table[b][t / page_size]).  Returns -1 for a
// token whose page is not mapped (past max_pages, or an id outside [0, num_pages)).
// `coherent` reads the block table through L2 only (for reads that may precede the
// dependency wait: the read-only path could keep a line that the preceding kernel rewrites).
struct CacheRows {
  const int32_t* block_table;  // [B][max_pages], or null for a contiguous cache
  int max_pages, page_size, num_pages, Hkv, L_max;
};
__device__ __forceinline__ long long cache_row(const CacheRows& c, int b, int h, int t,
                                              bool coherent = false) {
  if (c.block_table == nullptr) return ((long long)b * c.Hkv + h) * c.L_max + t;
  const int pi = t / c.page_size;
  if (pi >= c.max_pages) return -1;
  const int* e = c.block_table + (size_t)b * c.max_pages + pi;
  const int pg = coherent ? __ldcg(e) : __ldg(e);
  if (pg < 0 || pg >= c.num_pages) return -1;
  return ((long long)pg * c.Hkv + h) * c.page_size + (t - pi * c.page_size);
}
// Whether every page holding tokens [t0, t1) of sequence b is mapped (always, contiguous).
__device__ __forceinline__ bool pages_mapped(const CacheRows& c, int b, int t0, int t1) {
  if (c.block_table == nullptr || t1 <= t0) return true;
  for (int pi = t0 / c.page_size; pi <= (t1 - 1) / c.page_size; ++pi) {
    if (pi >= c.max_pages) return false;
    const int pg = __ldg(c.block_table + (size_t)b * c.max_pages + pi);
    if (pg < 0 || pg >= c.num_pages) return false;
  }
  return true;
}

__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Allow the next grid in the stream (if launched as a programmatic dependent)
// to start its prologue now.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------- tagged words

// Values passed between CTAs without a fence: each 64-bit word holds an fp32 value in its
// low half and a tag in its high half.  An aligned 64-bit access is single-copy atomic, so
// a reader that sees the tag also sees the value written with it; a vector access of two
// words is two such accesses (each word is checked on its own).
__device__ __forceinline__ uint64_t tagged(float v, uint32_t tag) {
  return ((uint64_t)tag << 32) | (uint64_t)__float_as_uint(v);
}
__device__ __forceinline__ float tagged_value(uint64_t w) { return __uint_as_float((uint32_t)w); }
__device__ __forceinline__ uint32_t tagged_tag(uint64_t w) { return (uint32_t)(w >> 32); }

// Store two tagged words (16-byte aligned) at GPU scope, bypassing L1.
__device__ __forceinline__ void st_tagged2(uint64_t* p, uint64_t w0, uint64_t w1) {
  asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %2};" ::"l"(p), "l"(w0), "l"(w1)
               : "memory");
}
// Load two tagged words (16-byte aligned) at GPU scope (every call reads L2 again).
__device__ __forceinline__ void ld_tagged2(const uint64_t* p, uint64_t& w0, uint64_t& w1) {
  asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(w0), "=l"(w1) : "l"(p)
               : "memory");
}

// ---------------------------------------------------------------------------- loads

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// Explicit shared-memory accesses (32-bit shared addresses).  Issued in program order and
// free of any generic-address handling, so a batch of them is in flight at once (the
// compiler was found to serialise the equivalent pointer loads in code that runs once).
__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ float2 lds_f32x2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void sts_f32x2(uint32_t addr, float x, float y) {
  asm volatile("st.shared.v2.f32 [%0], {%1,%2};" ::"r"(addr), "f"(x), "f"(y) : "memory");
}

__device__ __forceinline__ float4 lds128f(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

// ---------------------------------------------------------------------------- bf16

// The two bf16 values packed in a 32-bit word, widened exactly to fp32.
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float bf16_to_f32(uint16_t h) {
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

// fp32 -> bf16 bits, round to nearest even (NaN kept quiet).
__device__ __forceinline__ uint16_t f32_to_bf16_rn(float f) {
  uint16_t r;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(f));
  return r;
}

// x rounded to the nearest bf16 (ties to even), as fp32.
__device__ __forceinline__ float bf16_round(float x) {
  return __uint_as_float((uint32_t)f32_to_bf16_rn(x) << 16);
}
// The integer code of x under a row scale: RNE(x / scale) in [-qmax, qmax] (IEEE fp32
// division; qmax 127 for int8, 7 for 4-bit codes); a zero scale (a zero row) gives 0.
__device__ __forceinline__ int quantize_code(float x, float scale, int qmax = 127) {
  if (!(scale > 0.f)) return 0;
  const int c = __float2int_rn(__fdiv_rn(x, scale));
  return c > qmax ? qmax : (c < -qmax ? -qmax : c);
}
__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

}  // namespace stief
