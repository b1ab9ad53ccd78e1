// compress_joint_tc.cu -- the joint-value compress of prefill-sized chunks on the
// 5th-generation tensor cores (tcgen05, accumulators in tensor memory), for sm_100a.
//
// Operation (STAR-KV technical summary, "Metodologia" item 2, the hybrid decomposition):
// keys per KV head, values of all KV heads of a token together.  For sequence b and a tile of
// 128 new rows (tokens):
//     D_K[h][128 x rK] = X_K[b][h][128 x d] . P_K[h][d x rK]                  (K = d = 128)
//     D_V[128 x rV]    = [X_V[b][0] | ... | X_V[b][Hkv-1]][128 x Hkv d] . P_VJ[Hkv d x rV]
// bf16 x bf16 -> fp32, each row rounded once to bf16 (RNE) and written at seq_lens[b] + row of
// k_lat [B][Hkv][L_max][rK] and of v_joint [B][L_max][rV].  The value product is a
// K = Hkv * d contraction: 128 reduction columns (one KV head's values) per chunk, Hkv chunks
// accumulated into one TMEM accumulator.
//
// One 1-D grid, two kinds of CTA (value CTAs first, so they are scheduled first: each of
// their tiles takes Hkv chunks against a key tile's one):
//   value CTA (b, x): tiles x, x + gv, ... of sequence b; its chunks of the joint basis staged
//                     once;
//   key CTA (b, h, x): tiles x, x + gk, ... of head h; P_K[h] staged once.
// With an even Hkv (when it fits) the value tiles are split over CTA pairs (thread-block
// clusters of two): the pair's rank-0 CTA takes the chunks of KV heads 0 .. Hkv/2 - 1, rank 1
// the rest, each into its own TMEM accumulator; rank 1 then moves its partial sums into rank
// 0's shared memory (distributed shared memory) and rank 0 adds them (fp32, one order) before
// the rounding.  Each CTA of a pair stages half the joint basis and streams half the rows.
// The bases are transposed by the threads into the K-major 128-byte-swizzled operand layout
// (rows n = latent column); the input chunks arrive by 2-D TMA copies (two 64-column atoms of
// 128 rows) through a ring of `stages` buffers.  Thread 0 issues everything asynchronous: for
// each chunk it waits for the copy, issues the 8 MMAs (K = 16 each), commits them to the
// stage's "empty" barrier, and refills the previous chunk's stage once its MMAs are done, so
// the next copies are in flight while the MMAs run.  After a tile's last chunk a commit on the
// accumulator barrier releases the epilogue: warp w reads TMEM lanes 32 (w & 3) .. + 31
// (rows) and every other group of 16 columns (w >> 2 picks which), rounds and stores.  Key
// CTAs (one chunk per tile, several tiles) keep two accumulator sets instead: tile i + 1's
// MMAs are issued before tile i's epilogue when its copy is already in.
//
// Launched as a programmatic dependent: barrier set-up, the TMEM allocation and the basis
// staging (weights, which the preceding kernel must not write) overlap the preceding kernel's
// tail; the new rows and the lengths are read only after the dependency wait.  Every wait is
// bounded; every requested copy lands, every issued MMA completes and tensor memory is
// released before the CTA exits.
#include <cstdint>

#include "stief_device.cuh"
#include "stief_internal.h"
#include "umma.cuh"

namespace stief {

namespace {

constexpr int kJtThreads = 256;
constexpr uint32_t kJtTmemCols = 256;  // two accumulator sets of 128 columns (N = r <= 128)
constexpr int kJtMaxStages = 4;
constexpr uint32_t kAtomBytes = kUmmaRows * 128u;  // 128 rows x 64 bf16 columns
constexpr uint32_t kChunkBytes = 2u * kAtomBytes;  // one 128 x 128 input chunk

struct JtSmem {
  uint32_t x0;         // ring: stage s at x0 + s * kChunkBytes (two atoms each)
  uint32_t basis;      // chunk c atom a at basis + (2 c + a) * r * 128
  uint32_t exch;       // pairs: rank 1's partial sums [rV / 4][128 rows] float4, then a flag
  uint32_t bars;       // full[stages], empty[stages], acc, drain
  uint32_t tmem_slot;  // tcgen05.alloc writes the TMEM base address here
  uint32_t total;
};

// vch: value chunks a CTA stages (Hkv, or Hkv / 2 for pairs); pair: room for the exchange
__host__ __device__ inline JtSmem jt_smem_layout(int vch, int rK, int rV, int stages, bool pair) {
  JtSmem s;
  s.x0 = 0;
  uint32_t off = (uint32_t)stages * kChunkBytes;
  s.basis = off;
  // r is a multiple of 16, so r * 128 bytes per atom keeps every atom 1 KiB aligned
  const uint32_t kb = 2u * (uint32_t)rK * 128u, vb = 2u * (uint32_t)vch * (uint32_t)rV * 128u;
  off += kb > vb ? kb : vb;
  s.exch = off;
  if (pair) off += (uint32_t)kUmmaRows * (uint32_t)rV * 4u + 16u;
  s.bars = off;
  off += 8u * (2u * (uint32_t)stages + 2u);
  off = (off + 15u) & ~15u;
  s.tmem_slot = off;
  off += 16u;
  s.total = off;
  return s;
}

// The largest ring (2 .. kJtMaxStages) that fits one CTA's shared memory; 0 if none does.
int jt_stages(int vch, int rK, int rV, bool pair) {
  for (int st = kJtMaxStages; st >= 2; --st)
    if (jt_smem_layout(vch, rK, rV, st, pair).total <= (uint32_t)kMaxSmemPerBlock) return st;
  return 0;
}
// Value tiles split over CTA pairs: Hkv even and the half basis, the exchange area and two
// stages fit.
bool jt_pair_fits(int Hkv, int rK, int rV) {
  return Hkv >= 2 && Hkv % 2 == 0 && jt_stages(Hkv / 2, rK, rV, true) >= 2;
}

// Every thread of both CTAs of the cluster: release this CTA's shared-memory writes (local
// and remote) and wait for the partner's.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// The address of `saddr` (this CTA's shared memory) in the cluster CTA of the given rank.
__device__ __forceinline__ uint32_t cluster_addr(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint32_t x, uint32_t y, uint32_t z,
                                              uint32_t w) {
  asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(x), "r"(y),
               "r"(z), "r"(w)
               : "memory");
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t x) {
  asm volatile("st.shared::cluster.b32 [%0], %1;" ::"r"(addr), "r"(x) : "memory");
}

struct JointTcArgs {
  CUtensorMap mk;  // k_new as [B*Hkv*T rows][128] bf16, box 64 x 128, 128-byte swizzle
  CUtensorMap mv;  // v_new, same
  CompressArgs a;
  int tiles;       // 128-row tiles per (b, head)
  int stages;      // ring depth
  int gv, gk;      // value CTAs (pairs) per sequence, key CTAs per (sequence, head)
  int pair;        // value tiles split over CTA pairs (launched as clusters of two)
};

}  // namespace

__global__ void __launch_bounds__(kJtThreads, 1)
    stief_compress_joint_tc_kernel(const __grid_constant__ JointTcArgs ja) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const CompressArgs& a = ja.a;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hkv = a.Hkv, T = a.T, S = ja.stages;

  // the length kernel that follows may start now; it waits for this grid before it writes
  pdl_launch_dependents();

  // role of this CTA
  int id = (int)blockIdx.x;
  const int vct = ja.pair ? 2 : 1;  // CTAs per value tile group
  const int nval = a.B * ja.gv * vct;
  const bool values = id < nval;
  const bool paired = values && ja.pair;  // exchanges partial sums with its cluster partner
  int b, h, x, ctas, rank = 0;
  if (values) {
    rank = ja.pair ? (id & 1) : 0;
    const int g = ja.pair ? (id >> 1) : id;
    b = g / ja.gv;
    x = g - b * ja.gv;
    h = 0;
    ctas = ja.gv;
  } else {
    id -= nval;
    const int per_b = Hkv * ja.gk;
    b = id / per_b;
    const int rem = id - b * per_b;
    h = rem / ja.gk;
    x = rem - h * ja.gk;
    ctas = ja.gk;
  }
  // (pairs: both CTAs of a value pair take the same branch; the padding CTA that may end the
  // grid is a key-side CTA and uses no cluster barrier)
  if (b >= a.B || x >= ja.tiles) return;
  const int r = values ? a.rV : a.rK;
  const int vch = ja.pair ? Hkv / 2 : Hkv;  // value chunks per CTA
  const int nch = values ? vch : 1;          // 128-column chunks of the reduction per tile
  const int g0 = rank * vch;                 // this CTA's first value chunk (KV head)
  const int my_tiles = (ja.tiles - x + ctas - 1) / ctas;
  const int steps = my_tiles * nch;  // chunk copies of this CTA, in order
  const uint32_t atom_b = (uint32_t)r * 128u;  // one atom of the staged basis

  const JtSmem L = jt_smem_layout(vch, a.rK, a.rV, S, ja.pair != 0);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);  // [S]: copy landed
  uint64_t* empty = full + S;                                   // [S]: MMAs done reading
  uint64_t* acc_bar = empty + S;                                // tile's accumulator final
  uint64_t* drain_bar = acc_bar + 1;                            // exit: every MMA done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.tmem_slot);
  const CUtensorMap* map = values ? &ja.mv : &ja.mk;
  auto tile_m0 = [&](int i) { return (x + i * ctas) * kUmmaRows; };

#ifdef STIEF_TEST_HOOKS
  const uint32_t stall = a.test_stall_bytes;  // test build: chunk 0's copy never completes
#else
  constexpr uint32_t stall = 0u;
#endif
  int issued = 0;  // chunk copies requested (thread 0 only)
  auto issue = [&](int s) {  // thread 0: chunk s % nch of tile s / nch into stage s % S
    const int st = s % S, i = s / nch, c = s - i * nch;
    const int g = values ? g0 + c : h;  // KV head whose rows this chunk holds
    const int y = (int)(((int64_t)b * Hkv + g) * T + tile_m0(i));
    const uint64_t pol = l2_policy_evict_first();
    uint8_t* dst = smem + L.x0 + (uint32_t)st * kChunkBytes;
    mbar_arrive_expect_tx(&full[st], kChunkBytes + (s == 0 ? stall : 0u));
    tma_load_2d(dst, map, 0, y, &full[st], pol);
    tma_load_2d(dst + kAtomBytes, map, 64, y, &full[st], pol);
    issued = s + 1;
  };

  if ((smem_u32(smem) & 1023u) != 0) {  // swizzled operands need 1 KiB alignment (the same
    if (tid == 0) report(a.dev_status, STIEF_DEV_SMEM_ALIGN);  // for both CTAs of a pair)
    return;
  }
  if (tid == 0) {
    for (int i = 0; i < 2 * S + 2; ++i) mbar_init(&full[i], 1);
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, kJtTmemCols);

  // basis rows k = 0 .. nch*128 - 1 (row (g0 * 128 + k) of P_VJ, or row k of P_K[h]) -> chunk
  // k / 128, element k % 128 of every row n; each thread loads its whole row first
  {
    constexpr int kMaxChunks = 16;  // r <= 128: 16 groups of 8 columns
    const uint16_t* P = values ? a.P_V + (size_t)g0 * 128 * r : a.P_K + (size_t)h * 128 * r;
    for (int k = tid; k < nch * 128; k += kJtThreads) {
      uint4 w[kMaxChunks];
#pragma unroll
      for (int q = 0; q < kMaxChunks; ++q)
        if (8 * q < r) w[q] = __ldg(reinterpret_cast<const uint4*>(P + (size_t)k * r) + q);
      uint8_t* base = smem + L.basis + (uint32_t)(k >> 7) * 2u * atom_b;
#pragma unroll
      for (int q = 0; q < kMaxChunks; ++q) {
        if (8 * q >= r) continue;
        const uint32_t v[4] = {w[q].x, w[q].y, w[q].z, w[q].w};
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint16_t*>(base + sw128_offset(8 * q + j, k & 127, atom_b)) =
              (uint16_t)(v[j >> 1] >> (16 * (j & 1)));
      }
    }
  }
  __syncthreads();  // the barriers are initialised

  // the new rows and the lengths may come from the preceding kernel: read nothing before this
  pdl_wait();
  if (tid == 0)  // the first chunks fly while the length is read
    for (int s = 0; s < S && s < steps; ++s) issue(s);
  const int Lb = a.seq_lens[b];
  const bool bad = Lb < 0 || Lb > a.L_max;
  const bool over = !bad && (long long)Lb + T > a.L_max;
  if (tid == 0 && values && x == 0 && rank == 0) {
    if (bad) report(a.dev_status, STIEF_DEV_BAD_LENGTH);
    if (over) report(a.dev_status, STIEF_DEV_CAPACITY_OVERFLOW);
  }
  fence_proxy_async_smem();  // the generic-proxy basis writes must be seen by the MMA
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t idesc = idesc_bf16_f32(r);
  // the exchange area of the pair's rank-0 CTA (partial sums, then rank 1's status word)
  const uint32_t exch = smem_u32(smem + L.exch);
  const uint32_t flag_off = (uint32_t)kUmmaRows * (uint32_t)a.rV * 4u;
  bool ok = !(bad || over);
  int consumed = 0;  // chunk copies waited for (thread 0)
  bool mma_issued = false;

  // Key CTAs (one chunk per tile): two accumulator sets, so that tile i + 1's MMAs run
  // during tile i's epilogue when its copy is already in; the stages' "empty" barriers serve
  // as the two sets' "MMAs done" barriers (stage i % S is free once tile i's MMAs are done).
  int mma_next = 0;  // thread 0: key tiles [0, mma_next) have their MMAs issued
  auto key_mma = [&](int i) -> bool {
    const int st = i % S;
    if (!mbar_wait_bounded(&full[st], (uint32_t)((i / S) & 1), a.dev_status)) return false;
    consumed = i + 1;
    tc_fence_after();
    const uint32_t xa = smem_u32(smem + L.x0 + (uint32_t)st * kChunkBytes);
    const uint32_t pa = smem_u32(smem + L.basis);
    const uint32_t acc = tmem + (uint32_t)(i & 1) * 128u;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {  // K = 128 in steps of 16 (32 bytes inside an atom)
      const uint32_t koff = (uint32_t)(kk & 3) * 32u;
      umma_bf16(acc, sw128_desc(xa + (uint32_t)(kk >> 2) * kAtomBytes + koff),
                sw128_desc(pa + (uint32_t)(kk >> 2) * atom_b + koff), idesc, kk > 0 ? 1u : 0u);
    }
    mma_issued = true;
    umma_commit(&empty[i & 1]);
    mma_next = i + 1;
    return true;
  };
  for (int i = 0; !values && i < my_tiles && ok; ++i) {
    bool fail = false;
    if (tid == 0 && mma_next == i) fail = !key_mma(i);
    if (__syncthreads_or(fail)) {
      ok = false;
      break;
    }
    if (__syncthreads_or(!mbar_wait_bounded(&empty[i & 1], (uint32_t)((i >> 1) & 1), a.dev_status))) {
      ok = false;
      break;
    }
    tc_fence_after();
    if (tid == 0) {
      if (i + S < my_tiles) issue(i + S);  // tile i's MMAs have read its stage
      if (i + 1 < my_tiles && mbar_test(&full[(i + 1) % S], (uint32_t)(((i + 1) / S) & 1)))
        key_mma(i + 1);
    }
    const int m0 = tile_m0(i);
    const int row = (warp & 3) * 32 + lane;
    const bool live = m0 + row < T;
    const uint32_t lane_base = tmem + (uint32_t)(i & 1) * 128u + ((uint32_t)((warp & 3) * 32) << 16);
    const size_t crow = ((size_t)b * Hkv + h) * a.L_max + (size_t)(Lb + m0 + row);
    uint16_t* dst = a.k_lat + (live ? crow * (size_t)r : 0);
    for (int c0 = 16 * (warp >> 2); c0 < r; c0 += 32) {
      uint32_t v[16];
      tmem_ld16(lane_base + (uint32_t)c0, v);
      tmem_wait_ld();
      if (live) store_bf16x16(dst + c0, v);
    }
    // every warp is done reading this set before tile i + 2 overwrites it
    tc_fence_before();
    __syncthreads();
  }

  // Value CTAs (one accumulator, set 0).
  // A pair runs every iteration (its two cluster barriers per tile must match in both CTAs);
  // after a failed wait a CTA only skips the work.  Other CTAs stop at the first failure.
  for (int i = 0; values && i < my_tiles && (ok || paired); ++i) {
    bool fail = false;
    if (ok && tid == 0) {
      for (int c = 0; c < nch; ++c) {
        const int s = i * nch + c, st = s % S;
        if (!mbar_wait_bounded(&full[st], (uint32_t)((s / S) & 1), a.dev_status)) {
          fail = true;
          break;
        }
        consumed = s + 1;
        tc_fence_after();
        const uint32_t xa = smem_u32(smem + L.x0 + (uint32_t)st * kChunkBytes);
        const uint32_t pa = smem_u32(smem + L.basis + (uint32_t)c * 2u * atom_b);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // K = 128 in steps of 16 (32 bytes inside an atom)
          const uint32_t koff = (uint32_t)(kk & 3) * 32u;
          umma_bf16(tmem, sw128_desc(xa + (uint32_t)(kk >> 2) * kAtomBytes + koff),
                    sw128_desc(pa + (uint32_t)(kk >> 2) * atom_b + koff), idesc,
                    (c > 0 || kk > 0) ? 1u : 0u);
        }
        mma_issued = true;
        umma_commit(&empty[st]);
        // the previous chunk's MMAs are done (they ran while this one was issued): refill its
        // stage with the chunk S steps later
        const int sp = s - 1;
        if (sp >= 0 && sp + S < steps) {
          if (!mbar_wait_bounded(&empty[sp % S], (uint32_t)((sp / S) & 1), a.dev_status)) {
            fail = true;
            break;
          }
          issue(sp + S);
        }
      }
      if (!fail) umma_commit(acc_bar);
    }
    if (__syncthreads_or(fail)) ok = false;
    if (ok && __syncthreads_or(!mbar_wait_bounded(acc_bar, (uint32_t)(i & 1), a.dev_status)))
      ok = false;
    tc_fence_after();

    // epilogue: lane = row of this warp's 32 TMEM lanes; groups of 16 columns alternate
    // between the two warps of a lane quarter
    const int m0 = tile_m0(i);
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    if (paired && rank == 1) {  // partial sums into rank 0's exchange area, then the status word
      const uint32_t rx = cluster_addr(exch, 0u);
      if (ok) {
        for (int c0 = 16 * (warp >> 2); c0 < r; c0 += 32) {
          uint32_t v[16];
          tmem_ld16(lane_base + (uint32_t)c0, v);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 4; ++q)
            st_cluster_v4(rx + 16u * (uint32_t)((c0 / 4 + q) * kUmmaRows + row), v[4 * q],
                          v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      }
      if (tid == 0) st_cluster_u32(rx + flag_off, ok ? 1u : 0u);
    }
    if (paired) cluster_sync_all();  // rank 1's partial sums are in rank 0's shared memory
    if (rank == 0) {
      const bool both = !paired || lds_u32(exch + flag_off) != 0u;
      const bool live = m0 + row < T;
      const size_t crow = values ? (size_t)b * a.L_max + (size_t)(Lb + m0 + row)
                                 : ((size_t)b * Hkv + h) * a.L_max + (size_t)(Lb + m0 + row);
      uint16_t* dst = (values ? a.v_lat : a.k_lat) + (live ? crow * (size_t)r : 0);
      if (ok && both) {
        for (int c0 = 16 * (warp >> 2); c0 < r; c0 += 32) {
          uint32_t v[16];
          tmem_ld16(lane_base + (uint32_t)c0, v);
          tmem_wait_ld();
          if (paired) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float4 p = lds128f(exch + 16u * (uint32_t)((c0 / 4 + q) * kUmmaRows + row));
              v[4 * q] = __float_as_uint(__uint_as_float(v[4 * q]) + p.x);
              v[4 * q + 1] = __float_as_uint(__uint_as_float(v[4 * q + 1]) + p.y);
              v[4 * q + 2] = __float_as_uint(__uint_as_float(v[4 * q + 2]) + p.z);
              v[4 * q + 3] = __float_as_uint(__uint_as_float(v[4 * q + 3]) + p.w);
            }
          }
          if (live) store_bf16x16(dst + c0, v);
        }
      }
    }
    if (paired) cluster_sync_all();  // rank 0 is done with the exchange area
    // every warp is done reading the accumulator before the next tile overwrites it
    tc_fence_before();
    __syncthreads();
  }

  if (tid == 0) {
    // every issued MMA completes and every requested copy lands before the shared memory
    // and the tensor memory are released (bounded waits; on the normal path nothing is
    // outstanding)
    if (!ok && mma_issued) {
      umma_commit(drain_bar);
      mbar_wait_bounded(drain_bar, 0u, nullptr);
    }
    for (int j = consumed; j < issued; ++j)
      mbar_wait_bounded(&full[j % S], (uint32_t)((j / S) & 1), nullptr);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kJtTmemCols);
  }
}

bool compress_joint_tc_fits(int Hkv, int rK, int rV) {
  return jt_pair_fits(Hkv, rK, rV) || jt_stages(Hkv, rK, rV, false) >= 2;
}

cudaError_t launch_compress_joint_tc(const CompressArgs& a, cudaStream_t stream) {
  JointTcArgs ja{};
  ja.a = a;
#ifdef STIEF_TEST_HOOKS
  ja.a.test_stall_bytes = test_stall_bytes();
#endif
  ja.tiles = (a.T + kUmmaRows - 1) / kUmmaRows;
  ja.pair = jt_pair_fits(a.Hkv, a.rK, a.rV) ? 1 : 0;
  const int vch = ja.pair ? a.Hkv / 2 : a.Hkv;
  ja.stages = jt_stages(vch, a.rK, a.rV, ja.pair != 0);
  if (ja.stages < 2 || a.d != 128) return cudaErrorInvalidValue;
  const uint64_t rows = (uint64_t)a.B * a.Hkv * a.T;
  if (rows >= (1ull << 31)) return cudaErrorInvalidValue;  // TMA row coordinates are int32
  if (!encode_tiled_bf16_2d(&ja.mk, a.k_new, 128, rows, 256, 64, kUmmaRows, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tiled_bf16_2d(&ja.mv, a.v_new, 128, rows, 256, 64, kUmmaRows, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  bool sm100 = false;
  if (!query_device(&dev, &sms, &sm100)) return cudaErrorInvalidDevice;
  // one CTA per SM (the shared memory): value CTAs (pairs), Hkv (Hkv / 2) chunks per tile, get
  // up to half the SMs, one tile each where they can; key CTAs share the rest
  const int vct = ja.pair ? 2 : 1;
  ja.gv = (sms / 2) / (a.B * vct);
  if (ja.gv < 1) ja.gv = 1;
  if (ja.gv > ja.tiles) ja.gv = ja.tiles;
  const long long rest = (long long)sms - (long long)a.B * ja.gv * vct;
  long long gk = rest / ((long long)a.B * a.Hkv);
  if (gk < 1) gk = 1;
  if (gk > ja.tiles) gk = ja.tiles;
  ja.gk = (int)gk;
  long long ctas = (long long)a.B * ja.gv * vct + (long long)a.B * a.Hkv * ja.gk;
  if (ja.pair && (ctas & 1)) ++ctas;  // whole clusters (the extra CTA finds no work)
  if (ctas >= (1ll << 31)) return cudaErrorInvalidValue;
  const uint32_t smem = jt_smem_layout(vch, a.rK, a.rV, ja.stages, ja.pair != 0).total;
  static SmemLimit limit;
  cudaError_t e = limit.ensure(reinterpret_cast<const void*>(stief_compress_joint_tc_kernel), dev, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(kJtThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  // programmatic dependent launch: the CTAs may start while the preceding kernel drains and
  // wait for it (griddepcontrol.wait) before reading the new rows or the lengths; pairs run
  // as clusters of two CTAs
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = ja.pair ? 2 : 1;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = ja.pair ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, stief_compress_joint_tc_kernel, ja);
}

}  // namespace stief
