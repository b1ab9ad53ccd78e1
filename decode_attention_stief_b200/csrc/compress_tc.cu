// compress_tc.cu -- compressed storage of prefill-sized chunks on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory), for sm_100a.
//
// Operation (StiefAttention technical summary, "Mecanismo Central" item 5): keys and
// values are stored compressed, K_down = K P_K and V_down = V P_V.  For one (sequence b,
// KV head h) and a tile of 128 new rows, both products are one MMA chain each:
//     D_K[128 x rK] = X_K[128 x 128] . P_K[h][128 x rK]     (bf16 x bf16 -> fp32)
//     D_V[128 x rV] = X_V[128 x 128] . P_V[h][128 x rV]
// with M = 128 rows (tokens), N = r, K = d = 128 in 8 steps of 16.
//   - X tiles arrive by 2-D TMA tensor copies with the 128-byte swizzle, in two 64-column
//     atoms: exactly the canonical K-major SW128 operand layout of the MMA;
//   - P[h] is written once per CTA, transposed into the same K-major SW128 layout
//     (rows n = latent column, 128 bytes of k per row and atom);
//   - one thread issues tcgen05.mma; completion is signalled by tcgen05.commit on an
//     mbarrier; the accumulators live in 256 columns of tensor memory (D_K at column
//     0, D_V at column 128);
//   - epilogue: each of 4 warps reads its 32 TMEM lanes (rows) with tcgen05.ld, rounds
//     to bf16 (RNE) and stores its rows into the latent cache at seq_lens[b] + row.
// A CTA loops over m-tiles of one (b, h) so P is staged once.  Every wait is bounded;
// tensor memory is always released before the CTA exits.
#include <cstdint>

#include "stief_device.cuh"
#include "stief_internal.h"

namespace stief {

namespace {

constexpr int kTcRows = 128;     // M: rows (tokens) per MMA tile
constexpr int kTcThreads = 128;  // 4 warps: TMEM lanes 32w .. 32w + 31
constexpr uint32_t kTmemCols = 256;

// Shared-memory layout (byte offsets, all swizzled operands 1 KiB aligned).
struct TcSmem {
  uint32_t xk[2], xv[2];  // X tiles, two 64-column atoms each: 128 rows x 128 B
  uint32_t pk[2], pv[2];  // transposed bases, two atoms each: r rows x 128 B
  uint32_t bars;          // tma, mma
  uint32_t tmem_slot;     // tcgen05.alloc writes the TMEM base address here
  uint32_t total;
};

__host__ __device__ inline TcSmem tc_smem_layout(int rK, int rV) {
  TcSmem s;
  uint32_t off = 0;
  for (int i = 0; i < 2; ++i) { s.xk[i] = off; off += kTcRows * 128; }
  for (int i = 0; i < 2; ++i) { s.xv[i] = off; off += kTcRows * 128; }
  for (int i = 0; i < 2; ++i) { s.pk[i] = off; off += (uint32_t)rK * 128; off = (off + 1023) & ~1023u; }
  for (int i = 0; i < 2; ++i) { s.pv[i] = off; off += (uint32_t)rV * 128; off = (off + 1023) & ~1023u; }
  s.bars = off;
  off += 16;
  s.tmem_slot = off;
  off += 16;
  s.total = off;
  return s;
}

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
         | ((uint32_t)(kTcRows >> 4) << 24);  // M / 16
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

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

// P[h] ([128][r] row-major in global) -> shared [r rows][128 k] K-major SW128, two atoms.
__device__ __forceinline__ void stage_basis(uint8_t* smem, const uint32_t (&atom)[2],
                                            const uint16_t* P, int r, int tid) {
  // thread = row k of P (128 threads, d = 128); each writes its k into every row n
  const int k = tid;
  const uint16_t* src = P + (size_t)k * r;
  const uint32_t at = atom[k >> 6];
  const uint32_t kb = (uint32_t)(k & 63) * 2u;  // byte of k inside the 128-byte row
  for (int n0 = 0; n0 < r; n0 += 8) {
    const uint4 w = *reinterpret_cast<const uint4*>(src + n0);
    const uint16_t v[8] = {(uint16_t)(w.x & 0xFFFF), (uint16_t)(w.x >> 16), (uint16_t)(w.y & 0xFFFF),
                           (uint16_t)(w.y >> 16),    (uint16_t)(w.z & 0xFFFF), (uint16_t)(w.z >> 16),
                           (uint16_t)(w.w & 0xFFFF), (uint16_t)(w.w >> 16)};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + j;
      const uint32_t off = at + (uint32_t)n * 128u + ((((kb >> 4) ^ (uint32_t)(n & 7)) << 4) | (kb & 15u));
      *reinterpret_cast<uint16_t*>(smem + off) = v[j];
    }
  }
}

}  // namespace

struct CompressTcArgs {
  CUtensorMap mk;  // k_new as [B*Hkv*T rows][128] bf16, box 64 x 128, 128-byte swizzle
  CUtensorMap mv;  // v_new, same
  CompressArgs a;
  int tiles;       // m-tiles per (b, h)
};

__global__ void __launch_bounds__(kTcThreads, 1)
    stief_compress_tc_kernel(const __grid_constant__ CompressTcArgs ta) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const CompressArgs& a = ta.a;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int rK = a.rK, rV = a.rV, T = a.T;
  const TcSmem L = tc_smem_layout(rK, rV);
  uint64_t* tma_bar = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* mma_bar = tma_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.tmem_slot);

  pdl_launch_dependents();
  const int Lb = a.seq_lens[b];
  const bool bad = Lb < 0 || Lb > a.L_max;
  const bool full = !bad && (long long)Lb + T > a.L_max;
  if (tid == 0 && blockIdx.x == 0 && h == 0) {
    if (bad) report(a.dev_status, STIEF_DEV_BAD_LENGTH);
    if (full) report(a.dev_status, STIEF_DEV_CAPACITY_OVERFLOW);
  }
  if (bad || full) return;
  if ((smem_u32(smem) & 1023u) != 0) {  // swizzled operands need 1 KiB alignment
    if (tid == 0) report(a.dev_status, STIEF_DEV_SMEM_ALIGN);
    return;
  }

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    mbar_init(tma_bar, 1);
    mbar_init(mma_bar, 1);
    fence_barrier_init();
  }
  stage_basis(smem, L.pk, a.P_K + (size_t)h * 128 * rK, rK, tid);
  stage_basis(smem, L.pv, a.P_V + (size_t)h * 128 * rV, rV, tid);
  fence_proxy_async_smem();  // the generic-proxy basis writes must be seen by the MMA
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t idK = idesc_bf16_f32(rK), idV = idesc_bf16_f32(rV);
  const int64_t head_row = ((int64_t)b * a.Hkv + h) * T;
  bool ok = true;
  int phase = 0;

  for (int mt = blockIdx.x; mt < ta.tiles && ok; mt += gridDim.x) {
    const int m0 = mt * kTcRows;
    if (tid == 0) {
      const uint64_t pol = l2_policy_evict_first();
      mbar_arrive_expect_tx(tma_bar, 4u * kTcRows * 128u);
      const int y = (int)(head_row + m0);
      for (int i = 0; i < 2; ++i) {
        tma_load_2d(smem + L.xk[i], &ta.mk, 64 * i, y, tma_bar, pol);
        tma_load_2d(smem + L.xv[i], &ta.mv, 64 * i, y, tma_bar, pol);
      }
    }
    // a timed-out wait ends the loop for the whole CTA (tcgen05 ops below are warp-wide)
    if (__syncthreads_or(!mbar_wait_bounded(tma_bar, phase, a.dev_status))) {
      ok = false;
      break;
    }
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {  // K = 128 in steps of 16 (32 bytes inside an atom)
        const uint32_t koff = (uint32_t)(kk & 3) * 32u;
        umma_bf16(tmem, sw128_desc(smem_u32(smem + L.xk[kk >> 2]) + koff),
                  sw128_desc(smem_u32(smem + L.pk[kk >> 2]) + koff), idK, kk > 0);
        umma_bf16(tmem + 128u, sw128_desc(smem_u32(smem + L.xv[kk >> 2]) + koff),
                  sw128_desc(smem_u32(smem + L.pv[kk >> 2]) + koff), idV, kk > 0);
      }
      umma_commit(mma_bar);
    }
    if (__syncthreads_or(!mbar_wait_bounded(mma_bar, phase, a.dev_status))) {
      ok = false;
      break;
    }
    tc_fence_after();
    phase ^= 1;

    // epilogue: warp w owns rows 32w .. 32w + 31 (TMEM lanes); lane = row
    const int row = warp * 32 + lane;
    const bool live = m0 + row < T;
    const size_t cache_row = ((size_t)b * a.Hkv + h) * a.L_max + Lb + m0 + row;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    for (int which = 0; which < 2; ++which) {
      const int r = which ? rV : rK;
      uint16_t* dst = (which ? a.v_lat : a.k_lat) + cache_row * r;
      for (int c0 = 0; c0 < r; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(lane_base + (which ? 128u : 0u) + (uint32_t)c0, v);
        tmem_wait_ld();
        if (live) {
          uint4 lo, hi;
          lo.x = pack_bf16x2_rn(__uint_as_float(v[0]), __uint_as_float(v[1]));
          lo.y = pack_bf16x2_rn(__uint_as_float(v[2]), __uint_as_float(v[3]));
          lo.z = pack_bf16x2_rn(__uint_as_float(v[4]), __uint_as_float(v[5]));
          lo.w = pack_bf16x2_rn(__uint_as_float(v[6]), __uint_as_float(v[7]));
          hi.x = pack_bf16x2_rn(__uint_as_float(v[8]), __uint_as_float(v[9]));
          hi.y = pack_bf16x2_rn(__uint_as_float(v[10]), __uint_as_float(v[11]));
          hi.z = pack_bf16x2_rn(__uint_as_float(v[12]), __uint_as_float(v[13]));
          hi.w = pack_bf16x2_rn(__uint_as_float(v[14]), __uint_as_float(v[15]));
          *reinterpret_cast<uint4*>(dst + c0) = lo;
          *reinterpret_cast<uint4*>(dst + c0 + 8) = hi;
        }
      }
    }
    // every warp is done reading the accumulators before the next tile overwrites them
    tc_fence_before();
    __syncthreads();
  }

  if (!ok && tid == 0) {
    // give an outstanding copy or MMA a bounded chance to finish before memory is released
    mbar_wait_bounded(tma_bar, phase, nullptr);
    mbar_wait_bounded(mma_bar, phase, nullptr);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

uint32_t compress_tc_smem_bytes(int rK, int rV) { return tc_smem_layout(rK, rV).total; }

cudaError_t launch_compress_tc(const CompressArgs& a, cudaStream_t stream) {
  CompressTcArgs ta{};
  ta.a = a;
  ta.tiles = (a.T + kTcRows - 1) / kTcRows;
  const uint64_t rows = (uint64_t)a.B * a.Hkv * a.T;
  if (rows >= (1ull << 31)) return cudaErrorInvalidValue;  // TMA row coordinates are int32
  if (!encode_tiled_bf16_2d(&ta.mk, a.k_new, 128, rows, 256, 64, kTcRows, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tiled_bf16_2d(&ta.mv, a.v_new, 128, rows, 256, 64, kTcRows, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  bool sm100 = false;
  if (!query_device(&dev, &sms, &sm100)) return cudaErrorInvalidDevice;
  const int heads = a.B * a.Hkv;
  int gx = heads >= sms ? 1 : sms / heads;
  if (gx > ta.tiles) gx = ta.tiles;
  // at least 80 KiB so no more than two CTAs (2 x 256 TMEM columns) share an SM
  uint32_t smem = tc_smem_layout(a.rK, a.rV).total;
  if (smem < 80u * 1024u) smem = 80u * 1024u;
  static SmemLimit limit;
  cudaError_t e = limit.ensure(reinterpret_cast<const void*>(stief_compress_tc_kernel), dev, (int)smem);
  if (e != cudaSuccess) return e;
  stief_compress_tc_kernel<<<dim3(gx, a.Hkv, a.B), kTcThreads, smem, stream>>>(ta);
  return cudaGetLastError();
}

}  // namespace stief
