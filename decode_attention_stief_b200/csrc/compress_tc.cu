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
//     (rows n = latent column, 128 bytes of k per row and atom), all its loads in flight
//     at once;
//   - the keys and the values run as two halves of the CTA (warps 0-3 and 4-7), each with
//     its own copies, barriers and MMAs, issued by the half's first thread; completion is
//     signalled by tcgen05.commit on an mbarrier; the accumulators live in tensor memory
//     (D_K at column 0, D_V at column 128 of an accumulator set);
//   - epilogue: each of a half's 4 warps reads 32 TMEM lanes (rows) of its half's columns
//     with tcgen05.ld, rounds to bf16 (RNE) and stores its rows into the latent cache at
//     seq_lens[b] + row; the halves meet only at the start and at the end.
// A CTA loops over m-tiles of one (b, h) so P is staged once.  The kernel is launched as a
// programmatic dependent: barrier set-up, the tensor-memory allocation and the staging of
// the bases (weights, which the preceding kernel must not write) overlap the preceding
// kernel's tail; the new rows and the lengths are read only after the dependency wait.  Its
// X tiles stream through a two-stage ring: the first two are requested right after the wait
// (the length is read while they fly), and the copy of tile i + 2 is issued as soon as tile
// i's MMA has consumed its stage, so loads overlap the MMA and the epilogue.  Two accumulator
// sets (all 512 TMEM columns): tile i + 1's MMAs are issued into the other set before tile
// i's epilogue when its copy is already in, so they run during that epilogue; the epilogue
// requests up to four 16-column TMEM loads before each wait.
// Every wait is bounded; every requested copy lands and tensor memory is released before
// the CTA exits.
#include <cstdint>

#include "stief_device.cuh"
#include "stief_internal.h"
#include "umma.cuh"

namespace stief {

namespace {

constexpr int kTcRows = kUmmaRows;  // M: rows (tokens) per MMA tile
constexpr int kTcStages = 2;     // X tiles in flight per CTA
// 8 warps: warp w reads TMEM lanes 32 (w & 3) .. + 31 (rows), the keys' columns for w < 4 and
// the values' for w >= 4
constexpr int kTcThreads = 256;
// two accumulator sets of 256 columns (keys at 0, values at 128): tile i + 1's MMAs run into
// one while tile i's epilogue reads the other.  All 512 columns of the SM: the shared memory
// keeps this kernel at one CTA per SM
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = 256;

// Shared-memory layout (byte offsets, all swizzled operands 1 KiB aligned).
struct TcSmem {
  uint32_t xk[kTcStages][2], xv[kTcStages][2];  // X tiles per stage, two 64-column atoms:
                                                // 128 rows x 128 B each
  uint32_t pk[2], pv[2];  // transposed bases, two atoms each: r rows x 128 B
  uint32_t bars;          // per half (keys, values): tma[kTcStages], mma[2], drain
  uint32_t tmem_slot;     // tcgen05.alloc writes the TMEM base address here
  uint32_t total;
};

__host__ __device__ inline TcSmem tc_smem_layout(int rK, int rV) {
  TcSmem s;
  uint32_t off = 0;
  for (int st = 0; st < kTcStages; ++st) {
    for (int i = 0; i < 2; ++i) { s.xk[st][i] = off; off += kTcRows * 128; }
    for (int i = 0; i < 2; ++i) { s.xv[st][i] = off; off += kTcRows * 128; }
  }
  for (int i = 0; i < 2; ++i) { s.pk[i] = off; off += (uint32_t)rK * 128; off = (off + 1023) & ~1023u; }
  for (int i = 0; i < 2; ++i) { s.pv[i] = off; off += (uint32_t)rV * 128; off = (off + 1023) & ~1023u; }
  s.bars = off;
  off += 8 * 2 * (kTcStages + 3);  // per half: copies landed [stages], MMAs done [2], drain
  off = (off + 15) & ~15u;
  s.tmem_slot = off;
  off += 16;
  s.total = off;
  return s;
}

// P[h] ([128][r] row-major in global) -> shared [r rows][128 k] K-major SW128, two atoms.
// Threads 0-127 stage P_K and threads 128-255 P_V; thread = row k of its basis (d = 128): it
// reads its row first (all loads in flight together), then writes its k into every row n.
__device__ __forceinline__ void stage_bases(uint8_t* smem, const uint32_t (&atk)[2],
                                            const uint32_t (&atv)[2], const uint16_t* PK,
                                            const uint16_t* PV, int rK, int rV, int tid) {
  constexpr int kMaxChunks = 16;  // r <= 128: 16 chunks of 8 columns
  const int k = tid & 127;
  const bool vals = tid >= 128;
  const int r = vals ? rV : rK;
  const uint16_t* P = vals ? PV : PK;
  const uint32_t(&atom)[2] = vals ? atv : atk;
  uint4 w[kMaxChunks];
#pragma unroll
  for (int q = 0; q < kMaxChunks; ++q)
    if (8 * q < r) w[q] = __ldg(reinterpret_cast<const uint4*>(P + (size_t)k * r) + q);
  const uint32_t kb = (uint32_t)(k & 63) * 2u;  // byte of k inside the 128-byte row
  const uint32_t at = atom[k >> 6];
#pragma unroll
  for (int q = 0; q < kMaxChunks; ++q) {
    if (8 * q >= r) continue;
    const uint32_t v[4] = {w[q].x, w[q].y, w[q].z, w[q].w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = 8 * q + j;
      const uint32_t off = at + (uint32_t)n * 128u + ((((kb >> 4) ^ (uint32_t)(n & 7)) << 4) | (kb & 15u));
      *reinterpret_cast<uint16_t*>(smem + off) = (uint16_t)(v[j >> 1] >> (16 * (j & 1)));
    }
  }
}

// Named barrier `id` over `count` threads that also returns whether any of them passed true.
__device__ __forceinline__ bool bar_red_or(int id, int count, bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)p), "r"(id), "r"(count)
      : "memory");
  return r != 0;
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
  // The keys (warps 0-3) and the values (warps 4-7) run as two halves with their own copies,
  // MMAs, barriers and epilogue; each half's first thread issues its copies and MMAs.
  const int half = warp >> 2;            // 0: keys, 1: values
  const bool issuer = (tid & 127) == 0;
  const int bar_id = 1 + half;           // the half's named barrier (128 threads)
  uint64_t* bars0 = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* tma_bar = bars0 + half * (kTcStages + 3);  // [kTcStages]: the half's copy landed
  uint64_t* mma_bar = tma_bar + kTcStages;  // [2]: the half's MMAs of tile i are done (set i & 1)
  uint64_t* drain_bar = mma_bar + 2;        // exit after a failed wait: every MMA is done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.tmem_slot);
  const int64_t head_row = ((int64_t)b * a.Hkv + h) * T;
  const int my_tiles = (int)blockIdx.x < ta.tiles ? (ta.tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
  auto tile_m0 = [&](int i) { return ((int)blockIdx.x + i * (int)gridDim.x) * kTcRows; };
  // stage st of this half: two 64-column atoms
  auto x_atom = [&](int st, int at) { return half ? L.xv[st][at] : L.xk[st][at]; };
#ifdef STIEF_TEST_HOOKS
  const uint32_t stall = a.test_stall_bytes;  // test build: tile 0's copy never completes
#else
  constexpr uint32_t stall = 0u;
#endif
  int issued = 0;  // copies requested (issuer only)
  auto issue = [&](int i) {  // issuer: tile i of this half into stage i % kTcStages
    const int st = i % kTcStages;
    const uint64_t pol = l2_policy_evict_first();
    mbar_arrive_expect_tx(&tma_bar[st], 2u * kTcRows * 128u + (i == 0 ? stall : 0u));
    const int y = (int)(head_row + tile_m0(i));
    for (int at = 0; at < 2; ++at)
      tma_load_2d(smem + x_atom(st, at), half ? &ta.mv : &ta.mk, 64 * at, y, &tma_bar[st], pol);
    issued = i + 1;
  };

  pdl_launch_dependents();
  if ((smem_u32(smem) & 1023u) != 0) {  // swizzled operands need 1 KiB alignment
    if (tid == 0) report(a.dev_status, STIEF_DEV_SMEM_ALIGN);
    return;
  }
  if (tid == 0) {
    for (int i = 0; i < 2 * (kTcStages + 3); ++i) mbar_init(&bars0[i], 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  stage_bases(smem, L.pk, L.pv, a.P_K + (size_t)h * 128 * rK, a.P_V + (size_t)h * 128 * rV, rK, rV,
              tid);
  __syncthreads();  // the barriers are initialised
  // the new rows and the lengths may come from the preceding kernel: read nothing before this
  pdl_wait();
  if (issuer)  // the first tiles fly while the length is read
    for (int i = 0; i < kTcStages && i < my_tiles; ++i) issue(i);
  const int Lb = a.seq_lens[b];
  const bool bad = Lb < 0 || Lb > a.L_max;
  const CacheRows cr{a.block_table, a.max_pages, a.page_size, a.num_pages, a.Hkv, a.L_max};
  // no room, or (paged) a page of the new rows is not mapped: the sequence is not appended to
  const bool full = !bad && ((long long)Lb + T > a.L_max || !pages_mapped(cr, b, Lb, Lb + T));
  if (tid == 0 && blockIdx.x == 0 && h == 0) {
    if (bad) report(a.dev_status, STIEF_DEV_BAD_LENGTH);
    if (full) report(a.dev_status, STIEF_DEV_CAPACITY_OVERFLOW);
  }
  fence_proxy_async_smem();  // the generic-proxy basis writes must be seen by the MMA
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int r_h = half ? rV : rK;
  const uint32_t idesc = idesc_bf16_f32(r_h);
  const uint32_t p0 = half ? L.pv[0] : L.pk[0], p1 = half ? L.pv[1] : L.pk[1];
  bool ok = !(bad || full);
  int consumed = 0;  // tiles whose copy has been waited for (issuer)
  int mma_next = 0;  // issuer: tiles [0, mma_next) have their MMAs issued
  // issuer: tile i's MMAs into the half's columns of accumulator set i & 1 (keys at 0, values
  // at 128), once its copy has landed
  auto issue_mma = [&](int i) -> bool {
    const int st = i % kTcStages;
    if (!mbar_wait_bounded(&tma_bar[st], (uint32_t)((i / kTcStages) & 1), a.dev_status)) return false;
    consumed = i + 1;
    tc_fence_after();
    const uint32_t acc = tmem + (uint32_t)(i & 1) * kAccCols + (half ? 128u : 0u);
    const uint32_t x0 = x_atom(st, 0), x1 = x_atom(st, 1);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {  // K = 128 in steps of 16 (32 bytes inside an atom)
      const uint32_t koff = (uint32_t)(kk & 3) * 32u;
      umma_bf16(acc, sw128_desc(smem_u32(smem + (kk < 4 ? x0 : x1)) + koff),
                sw128_desc(smem_u32(smem + (kk < 4 ? p0 : p1)) + koff), idesc, kk > 0);
    }
    umma_commit(&mma_bar[i & 1]);
    mma_next = i + 1;
    return true;
  };

  for (int i = 0; i < my_tiles && ok; ++i) {
    bool fail = false;  // issuer: a copy did not land in time
    if (issuer && mma_next == i) fail = !issue_mma(i);
    // a timed-out wait ends the loop for the whole half (tcgen05 ops below are warp-wide)
    if (bar_red_or(bar_id, 128, fail)) {
      ok = false;
      break;
    }
    if (bar_red_or(bar_id, 128, !mbar_wait_bounded(&mma_bar[i & 1], (uint32_t)((i >> 1) & 1), a.dev_status))) {
      ok = false;
      break;
    }
    tc_fence_after();
    if (issuer) {
      // the MMAs have read stage i % kTcStages: refill it with tile i + kTcStages
      if (i + kTcStages < my_tiles) issue(i + kTcStages);
      // the next tile's MMAs run during this tile's epilogue (into the other accumulator set,
      // whose tile's epilogue ended with the previous iteration) if its copy is already in
      if (i + 1 < my_tiles &&
          mbar_test(&tma_bar[(i + 1) % kTcStages], (uint32_t)(((i + 1) / kTcStages) & 1)))
        issue_mma(i + 1);
    }

    // epilogue: warp w owns rows 32 (w & 3) .. + 31 (TMEM lanes; lane = row) of the keys
    // (w < 4) or of the values (w >= 4)
    const int m0 = tile_m0(i);
    const int row = (warp & 3) * 32 + lane;
    const int which = half;
    const bool live = m0 + row < T;
    const long long crow = live ? cache_row(cr, b, h, Lb + m0 + row) : 0;  // mapped (checked)
    const uint32_t lane_base = tmem + (uint32_t)(i & 1) * kAccCols + ((uint32_t)((warp & 3) * 32) << 16);
    if (a.k_scale != nullptr) {
      // int8 / 4-bit cache: the row rounded to bf16, then one fp32 scale (max / 127, or max / 7)
      // and RNE codes, divisions in IEEE fp32; the accumulators are read twice (maximum, then
      // codes).  4-bit codes go two per byte, column 2 j in the low nibble of byte j.
      const int r = which ? rV : rK;
      const uint32_t col0 = which ? 128u : 0u;
      const int qmax = a.q4 ? 7 : 127;
      float amax = 0.f;
      for (int c0 = 0; c0 < r; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(lane_base + col0 + (uint32_t)c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(bf16_round(__uint_as_float(v[e]))));
      }
      const float scale = __fdiv_rn(amax, (float)qmax);
      uint8_t* dst = reinterpret_cast<uint8_t*>(which ? a.v_lat : a.k_lat) + crow * (a.q4 ? r / 2 : r);
      for (int c0 = 0; c0 < r; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(lane_base + col0 + (uint32_t)c0, v);
        tmem_wait_ld();
        int code[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) code[e] = quantize_code(bf16_round(__uint_as_float(v[e])), scale, qmax);
        if (a.q4) {
          uint32_t w0 = 0u, w1 = 0u;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            w0 |= (uint32_t)(code[e] & 0xF) << (4 * e);
            w1 |= (uint32_t)(code[8 + e] & 0xF) << (4 * e);
          }
          if (live) *reinterpret_cast<uint2*>(dst + c0 / 2) = make_uint2(w0, w1);
        } else {
          uint32_t packed[4];
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            uint32_t word = 0u;
#pragma unroll
            for (int e = 0; e < 4; ++e) word |= (uint32_t)(uint8_t)code[4 * g + e] << (8 * e);
            packed[g] = word;
          }
          if (live) *reinterpret_cast<uint4*>(dst + c0) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
      }
      if (live) (which ? a.v_scale : a.k_scale)[crow] = scale;
    }
    if (a.k_scale == nullptr) {
      const int r = which ? rV : rK;
      uint16_t* dst = (which ? a.v_lat : a.k_lat) + crow * r;
      const uint32_t col0 = lane_base + (which ? 128u : 0u);
      for (int g0 = 0; g0 < r; g0 += 64) {  // up to four 16-column loads in flight, one wait
        uint32_t v[4][16];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (g0 + 16 * q < r) tmem_ld16(col0 + (uint32_t)(g0 + 16 * q), v[q]);
        tmem_wait_ld();
        if (live) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (g0 + 16 * q < r) store_bf16x16(dst + g0 + 16 * q, v[q]);
        }
      }
    }
    // every warp of the half is done reading the accumulators before its next tile
    // overwrites them
    tc_fence_before();
    named_bar_sync(bar_id, 128);
  }

  if (issuer) {
    // every requested copy must land before the shared memory is released (bounded waits;
    // on the normal path nothing is outstanding)
    for (int j = consumed; j < issued; ++j)
      mbar_wait_bounded(&tma_bar[j % kTcStages], (uint32_t)((j / kTcStages) & 1), nullptr);
    if (!ok && mma_next > 0) {  // MMAs left by a timeout get a bounded chance to finish
      umma_commit(drain_bar);
      mbar_wait_bounded(drain_bar, 0u, nullptr);
    }
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
#ifdef STIEF_TEST_HOOKS
  ta.a.test_stall_bytes = test_stall_bytes();
#endif
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
  // more than half an SM's shared memory: one CTA per SM (it holds all 512 TMEM columns)
  uint32_t smem = tc_smem_layout(a.rK, a.rV).total;
  if (smem < 120u * 1024u) smem = 120u * 1024u;
  static SmemLimit limit;
  cudaError_t e = limit.ensure(reinterpret_cast<const void*>(stief_compress_tc_kernel), dev, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(gx, a.Hkv, a.B);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  // programmatic dependent launch: the CTAs may start while the preceding kernel drains and
  // wait for it (griddepcontrol.wait) before reading the new rows or the lengths
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, stief_compress_tc_kernel, ta);
}

}  // namespace stief
